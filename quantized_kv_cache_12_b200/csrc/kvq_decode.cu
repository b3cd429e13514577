// kvq_decode.cu -- split-K decode attention over the packed cache, with the
// dequantization folded into the QK^T and PV tensor-core products
// (TurboQuant page 2.3, last paragraph) and the splits merged by log-sum-exp
// (Cocktail page 3.2.3).
//
// Work decomposition.  A CTA owns one (sequence b, KV head, token split);
// its four warps each stream a contiguous quarter of the split in 16-token
// tiles.  Each warp runs its own ring of shared-memory stages filled by
// one-dimensional bulk copies (the TMA engine, no multicast) that complete
// on per-stage mbarriers, so warps never wait for each other until the
// final in-CTA merge.
//
// Arithmetic.  With g = q_heads / kv_heads query heads on one KV head and
// NG = head_dim / G groups per token, the score of head h and token t is
//   score = scale * sum_gr s_gr * (sum_{j in gr} q_j c_j - z_gr * sum_{j in gr} q_j)
// where c are the raw integer codes, exact in fp16.  One m16n8k16 MMA tile
// computes the inner sums for up to 16 (group, head) rows at once: row
// r = gr * g + h of the A operand holds q_h masked to group gr, the B operand
// holds 8 tokens' codes.  Scales and zero points are applied afterwards in
// fp32, so nothing is rounded to fp16 but the codes themselves.  For PV,
//   o_h[d] = sum_t (p_t * s_gr(d),t) * c_t[d] - sum_t (p_t * s_gr,t) * z_gr,t
// the weights P' = p * s are split into fp16 hi + lo parts that fill the 16
// rows of the A operand (rows h and 8 + h), keeping ~22 bits of P'.
#include <cuda_runtime.h>
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

template <int BITS, int GE>
struct Cfg {
  static constexpr int D = kHeadDim;
  static constexpr int NG = D / GE;                    // groups per token
  static constexpr int RB = D * BITS / 8;              // code bytes per token
  static constexpr int MB = (BITS == 16) ? 0 : NG * 4; // (s, z) bytes per token
  static constexpr int KC = RB / 4;                    // K bytes per lane (32 dims)
  static constexpr int KW = KC / 4;                    // K words per lane
  static constexpr int VC = (GE / 8) * BITS / 8;       // V bytes per lane per group
  static constexpr int VW = VC >= 4 ? VC / 4 : 1;      // V words per lane per group
  static constexpr int NTG = GE / 8;                   // PV n-tiles per group
  static constexpr int STAGE = 2 * kTile * RB + 2 * kTile * MB;
  static constexpr int STAGES_RAW = 20480 / STAGE;
  static constexpr int STAGES = STAGES_RAW < 2 ? 2 : (STAGES_RAW > 16 ? 16 : STAGES_RAW);
  static constexpr int BAR_BYTES = 1024;
  static constexpr int SMEM = BAR_BYTES + kWarps * STAGES * STAGE;
  static constexpr int CROSS = (BITS == 16) ? 2 : (BITS == 8 ? 4 : (BITS == 4 ? 8 : 16));
};

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  return h2_as_u32(__floats2half2_rn(a, b));
}

// Load `n` bytes (1, 2 or a multiple of 4) of a lane's chunk into words.
template <int NBYTES, int NW>
__device__ __forceinline__ void load_chunk(const uint8_t* p, uint32_t (&w)[NW]) {
  if constexpr (NBYTES == 1) {
    w[0] = *p;
  } else if constexpr (NBYTES == 2) {
    w[0] = *reinterpret_cast<const uint16_t*>(p);
  } else if constexpr (NBYTES % 16 == 0) {
#pragma unroll
    for (int i = 0; i < NBYTES / 16; ++i) {
      uint4 v = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (NBYTES == 8) {
    uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

struct SplitParams {
  DecodeArgs a;
  SegView seg;
};

template <int BITS, int GE>
__global__ void __launch_bounds__(kWarps * 32)
decode_split_kernel(const __grid_constant__ SplitParams P) {
  using C = Cfg<BITS, GE>;
  constexpr int D = C::D;
  const DecodeArgs& a = P.a;
  const SegView& seg = P.seg;

  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int g = a.group_ratio;
  const int R = C::NG * g;  // valid MMA rows (group, head)

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem) + warp * C::STAGES;
  uint8_t* stages = smem + C::BAR_BYTES + warp * C::STAGES * C::STAGE;

  // ---- token range of this warp
  int L = seg.seq_lens[b];
  L = max(0, min(L, seg.max_tokens));
  const int per_split = (L + seg.n_split - 1) / seg.n_split;
  const int chunk = ((per_split + 63) / 64) * 64;
  const int c0 = split * chunk;
  const int c1 = min(c0 + chunk, L);
  const int wq = chunk / kWarps;
  const int w0 = c0 + warp * wq;
  const int w1 = min(w0 + wq, c1);
  const int n_tiles = (w1 > w0) ? (w1 - w0 + kTile - 1) / kTile : 0;
  const long long row0 = ((long long)b * a.kv_heads + kvh) * seg.max_tokens;

  const uint64_t policy = l2_evict_first_policy();
  auto issue = [&](int i) {
    const int st = i % C::STAGES;
    uint8_t* dst = stages + st * C::STAGE;
    const long long row = row0 + w0 + (long long)i * kTile;
    mbar_arrive_expect_tx(&bars[st], C::STAGE);
    bulk_load(dst, seg.k_codes + row * C::RB, kTile * C::RB, &bars[st], policy);
    bulk_load(dst + kTile * C::RB, seg.v_codes + row * C::RB, kTile * C::RB, &bars[st], policy);
    if constexpr (C::MB > 0) {
      bulk_load(dst + 2 * kTile * C::RB, seg.k_meta + row * C::MB, kTile * C::MB, &bars[st],
                policy);
      bulk_load(dst + 2 * kTile * C::RB + kTile * C::MB, seg.v_meta + row * C::MB,
                kTile * C::MB, &bars[st], policy);
    }
  };

  if (lane == 0) {
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (lane == 0) {
    const int pre = min(n_tiles, C::STAGES);
    for (int i = 0; i < pre; ++i) issue(i);
  }

  // ---- query fragments: row r = gr * g + h holds q_h masked to group gr
  const __half* qh16 = reinterpret_cast<const __half*>(a.q);
  const __nv_bfloat16* qb16 = reinterpret_cast<const __nv_bfloat16*>(a.q);
  const long long qbase = ((long long)b * a.q_heads + (long long)kvh * g) * D;
  auto qval = [&](int r, int d) -> float {
    if (r >= R || d / GE != r / g) return 0.0f;
    const long long i = qbase + (long long)(r % g) * D + d;
    // bf16 queries are used through fp16 (exact for |q| in [2^-14, 65504])
    return a.q_is_bf16 ? __half2float(__float2half_rn(__bfloat162float(qb16[i])))
                       : __half2float(qh16[i]);
  };
  using WP = WordPairs<BITS>;
  auto kdim = [&](int p, int e) -> int {
    return 32 * tig + (p / WP::kPairs) * WP::kDims + WP::dim(p % WP::kPairs, e);
  };
  uint32_t qf[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int pA = 2 * ks, pB = 2 * ks + 1;
    qf[ks][0] = pack_h2(qval(gid, kdim(pA, 0)), qval(gid, kdim(pA, 1)));
    qf[ks][1] = pack_h2(qval(gid + 8, kdim(pA, 0)), qval(gid + 8, kdim(pA, 1)));
    qf[ks][2] = pack_h2(qval(gid, kdim(pB, 0)), qval(gid, kdim(pB, 1)));
    qf[ks][3] = pack_h2(qval(gid + 8, kdim(pB, 0)), qval(gid + 8, kdim(pB, 1)));
  }
  // sum of q over the row's group (for the zero-point term)
  float qs0 = 0.f, qs1 = 0.f;
  if constexpr (BITS != 16) {
    if (gid < R) {
      const int gr = gid / g;
      for (int d = gr * GE; d < (gr + 1) * GE; ++d) qs0 += qval(gid, d);
    }
    if (gid + 8 < R) {
      const int gr = (gid + 8) / g;
      for (int d = gr * GE; d < (gr + 1) * GE; ++d) qs1 += qval(gid + 8, d);
    }
  }
  const int gr0 = (gid < R) ? gid / g : 0;
  const int gr1 = (gid + 8 < R) ? (gid + 8) / g : 0;
  const bool row0_ok = gid < R, row1_ok = gid + 8 < R;
  const bool head_ok = gid < g;  // this lane's PV rows are a real head

  // ---- running state (head = gid)
  float o_acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float corr[C::NG];
#pragma unroll
  for (int i = 0; i < C::NG; ++i) corr[i] = 0.f;
  float m_run = -INFINITY, l_part = 0.f;
  int failed_at = -1;

  for (int i = 0; i < n_tiles; ++i) {
    const int st = i % C::STAGES;
    if (!mbar_wait_bounded(&bars[st], (i / C::STAGES) & 1, 1u << 22)) {
      failed_at = i;
      break;
    }
    const uint8_t* sK = stages + st * C::STAGE;
    const uint8_t* sV = sK + kTile * C::RB;
    const uint8_t* sKm = sK + 2 * kTile * C::RB;
    const uint8_t* sVm = sKm + kTile * C::MB;
    const int t0 = w0 + i * kTile;
    const int n_valid = min(kTile, w1 - t0);

    // ---- S = Qx * K^T for the two 8-token n-tiles
    float s_acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      s_acc[nt][0] = s_acc[nt][1] = s_acc[nt][2] = s_acc[nt][3] = 0.f;
      uint32_t kw[C::KW];
      load_chunk<C::KC, C::KW>(sK + (nt * 8 + gid) * C::RB + tig * C::KC, kw);
      uint32_t pr[16];
#pragma unroll
      for (int w = 0; w < C::KW; ++w) {
        uint32_t tmp[WP::kPairs];
        WP::run(kw[w], tmp);
#pragma unroll
        for (int j = 0; j < WP::kPairs; ++j) pr[w * WP::kPairs + j] = tmp[j];
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_f16(s_acc[nt], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], pr[2 * ks],
                pr[2 * ks + 1]);
    }

    // ---- scores of head (gid mod g) for tokens nt*8 + 2*tig + e
    float sc[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = nt * 8 + 2 * tig + e;
        float c;
        if constexpr (BITS == 16) {
          c = row0_ok ? s_acc[nt][e] : 0.f;
        } else {
          const __half2* m = reinterpret_cast<const __half2*>(sKm + tok * C::MB);
          c = 0.f;
          if (row0_ok) {
            const float2 sz = __half22float2(m[gr0]);
            c = sz.x * (s_acc[nt][e] - sz.y * qs0);
          }
          if (row1_ok) {
            const float2 sz = __half22float2(m[gr1]);
            c += sz.x * (s_acc[nt][2 + e] - sz.y * qs1);
          }
        }
        sc[nt * 2 + e] = c;
      }
    }
    // sum the group rows of each head: lanes gid and gid ^ m (m >= g)
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
      if (m >= g) {
#pragma unroll
        for (int k = 0; k < 4; ++k) sc[k] += __shfl_xor_sync(0xffffffffu, sc[k], 4 * m);
      }
    }
    float tmax = -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int tok = (k >> 1) * 8 + 2 * tig + (k & 1);
      sc[k] = (tok < n_valid) ? sc[k] * a.scale_log2 : -INFINITY;
      tmax = fmaxf(tmax, sc[k]);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    if (tmax > m_run) {  // new running max: rescale what was accumulated
      const float alpha = exp2f(m_run - tmax);  // 0 when m_run = -inf
#pragma unroll
      for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int c = 0; c < 4; ++c) o_acc[n][c] *= alpha;
#pragma unroll
      for (int gr = 0; gr < C::NG; ++gr) corr[gr] *= alpha;
      l_part *= alpha;
      m_run = tmax;
    }
    float p[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      p[k] = (m_run == -INFINITY) ? 0.f : exp2f(sc[k] - m_run);
      if (!head_ok) p[k] = 0.f;
      l_part += p[k];
    }

    // ---- O += P' * V per group (hi rows gid, lo rows gid + 8)
    const int tokA = 2 * tig, tokB = 2 * tig + 1, tokC = 8 + 2 * tig, tokD = 9 + 2 * tig;
#pragma unroll
    for (int gr = 0; gr < C::NG; ++gr) {
      float pp[4];
      if constexpr (BITS == 16) {
#pragma unroll
        for (int k = 0; k < 4; ++k) pp[k] = p[k];
      } else {
        const int toks[4] = {tokA, tokB, tokC, tokD};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // slots past the valid length may hold any bytes (NaN scales):
          // select, never multiply by a zero weight
          const bool valid = toks[k] < n_valid;
          const float2 sz =
              __half22float2(reinterpret_cast<const __half2*>(sVm + toks[k] * C::MB)[gr]);
          pp[k] = valid ? p[k] * sz.x : 0.f;
          corr[gr] += valid ? pp[k] * sz.y : 0.f;
        }
      }
      __half hi[4];
      float lo[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        hi[k] = __float2half_rn(pp[k]);
        lo[k] = pp[k] - __half2float(hi[k]);
      }
      const uint32_t a0 = h2_as_u32(__halves2half2(hi[0], hi[1]));
      const uint32_t a1 = pack_h2(lo[0], lo[1]);
      const uint32_t a2 = h2_as_u32(__halves2half2(hi[2], hi[3]));
      const uint32_t a3 = pack_h2(lo[2], lo[3]);

      const uint8_t* vbase = sV + gr * (GE * BITS / 8) + gid * C::VC;
      uint32_t wA[C::VW], wB[C::VW], wC[C::VW], wD[C::VW];
      load_chunk<C::VC, C::VW>(vbase + tokA * C::RB, wA);
      load_chunk<C::VC, C::VW>(vbase + tokB * C::RB, wB);
      load_chunk<C::VC, C::VW>(vbase + tokC * C::RB, wC);
      load_chunk<C::VC, C::VW>(vbase + tokD * C::RB, wD);
      if constexpr (BITS == 16) {
        // raw fp16 rows past the valid length may hold anything: zero them
        if (n_valid < kTile) {
#pragma unroll
          for (int w = 0; w < C::VW; ++w) {
            if (tokA >= n_valid) wA[w] = 0u;
            if (tokB >= n_valid) wB[w] = 0u;
            if (tokC >= n_valid) wC[w] = 0u;
            if (tokD >= n_valid) wD[w] = 0u;
          }
        }
      }
#pragma unroll
      for (int w = 0; w < C::VW; ++w) {
        uint32_t x[C::CROSS], y[C::CROSS];
        CrossPairs<BITS>::run(wA[w], wB[w], x);
        CrossPairs<BITS>::run(wC[w], wD[w], y);
        constexpr int PER_W = (C::NTG < C::CROSS) ? C::NTG : C::CROSS;
#pragma unroll
        for (int j = 0; j < PER_W; ++j)
          mma_f16(o_acc[gr * C::NTG + w * PER_W + j], a0, a1, a2, a3, x[j], y[j]);
      }
    }
    __syncwarp();
    if (lane == 0 && i + C::STAGES < n_tiles) issue(i + C::STAGES);
  }

  if (failed_at >= 0) {
    if (lane == 0) atomicOr(a.err, kErrWaitTimeout);
    // drain the copies this warp issued and has not consumed (bounded)
    const int issued_end = min(n_tiles, failed_at + C::STAGES);
    for (int i = failed_at; i < issued_end; ++i)
      (void)mbar_wait_bounded(&bars[i % C::STAGES], (i / C::STAGES) & 1, 1u << 16);
  }

  // ---- per-warp totals over the 4 lanes of a head
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
#pragma unroll
  for (int gr = 0; gr < C::NG; ++gr) {
    corr[gr] += __shfl_xor_sync(0xffffffffu, corr[gr], 1);
    corr[gr] += __shfl_xor_sync(0xffffffffu, corr[gr], 2);
  }

  // ---- merge the 4 warps in shared memory (reusing the stage buffers)
  __syncthreads();
  float* ms = reinterpret_cast<float*>(smem + C::BAR_BYTES);  // [kWarps][8]
  float* ls = ms + kWarps * 8;                                 // [kWarps][8]
  float* os = ls + kWarps * 8;                                 // [kWarps][8][D]
  if (head_ok) {
    if (tig == 0) {
      ms[warp * 8 + gid] = m_run;
      ls[warp * 8 + gid] = l_part;
    }
    float* oh = os + (warp * 8 + gid) * D;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int gr = nt / C::NTG, jj = nt % C::NTG;
      const int d0 = gr * GE + (2 * tig) * C::NTG + jj;
      const int d1 = d0 + C::NTG;
      oh[d0] = o_acc[nt][0] + o_acc[nt][2] - corr[gr];
      oh[d1] = o_acc[nt][1] + o_acc[nt][3] - corr[gr];
    }
  }
  __syncthreads();
  const int t = threadIdx.x;  // one output dim per thread
  const int part = seg.part_base + split;
  for (int h = 0; h < g; ++h) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      if (ls[w * 8 + h] > 0.f) M = fmaxf(M, ms[w * 8 + h]);
    float Ls = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        if (ls[w * 8 + h] > 0.f) {
          const float wt = exp2f(ms[w * 8 + h] - M);
          Ls += wt * ls[w * 8 + h];
          O += wt * os[(w * 8 + h) * D + t];
        }
      }
    }
    const long long bh = (long long)b * a.q_heads + (long long)kvh * g + h;
    if (a.parts == 1) {
      a.out[bh * D + t] = (Ls > 0.f) ? O / Ls : 0.f;
      if (a.lse != nullptr && t == 0)
        a.lse[bh] = (Ls > 0.f) ? (M + log2f(Ls)) * 0.69314718055994531f : -INFINITY;
    } else {
      const long long pi = bh * a.parts + part;
      a.part_o[pi * D + t] = O;
      if (t == 0) {
        a.part_ml[pi * 2 + 0] = M;
        a.part_ml[pi * 2 + 1] = Ls;
      }
    }
  }
}

// Merge the partial (m, l, o) of every split and segment (log-sum-exp).
__global__ void __launch_bounds__(kHeadDim) decode_merge_kernel(const DecodeArgs a) {
  const long long bh = blockIdx.x;
  const int t = threadIdx.x;
  const float* ml = a.part_ml + bh * a.parts * 2;
  const float* po = a.part_o + bh * a.parts * kHeadDim;
  float M = -INFINITY;
  for (int p = 0; p < a.parts; ++p)
    if (ml[2 * p + 1] > 0.f) M = fmaxf(M, ml[2 * p]);
  float L = 0.f, O = 0.f;
  if (M != -INFINITY) {
    for (int p = 0; p < a.parts; ++p) {
      const float l = ml[2 * p + 1];
      if (l > 0.f) {
        const float w = exp2f(ml[2 * p] - M);
        L += w * l;
        O += w * po[(long long)p * kHeadDim + t];
      }
    }
  }
  a.out[bh * kHeadDim + t] = (L > 0.f) ? O / L : 0.f;
  if (a.lse != nullptr && t == 0)
    a.lse[bh] = (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

template <int BITS, int GE>
cudaError_t launch_split(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  using C = Cfg<BITS, GE>;
  static bool attr_set = false;  // per process; harmless to repeat
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<BITS, GE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  SplitParams P{a, seg};
  dim3 grid(seg.n_split, a.kv_heads, a.batch);
  decode_split_kernel<BITS, GE><<<grid, kWarps * 32, C::SMEM, s>>>(P);
  return cudaGetLastError();
}

}  // namespace

bool decode_supported(int bits, int group, int group_ratio) {
  if (!(group_ratio == 1 || group_ratio == 2 || group_ratio == 4 || group_ratio == 8))
    return false;
  if (bits == 16) return true;
  if (!(bits == 2 || bits == 4 || bits == 8)) return false;
  if (!(group == 32 || group == 64 || group == 128)) return false;
  return (kHeadDim / group) * group_ratio <= 16;
}

int decode_smem_bytes(int bits, int group) {
#define KVQ_S(B, G_) \
  if (bits == B && group == G_) return Cfg<B, G_>::SMEM;
  KVQ_S(16, 128)
  KVQ_S(8, 32) KVQ_S(8, 64) KVQ_S(8, 128)
  KVQ_S(4, 32) KVQ_S(4, 64) KVQ_S(4, 128)
  KVQ_S(2, 32) KVQ_S(2, 64) KVQ_S(2, 128)
#undef KVQ_S
  return 0;
}

cudaError_t launch_decode_segment(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  const int bits = seg.bits, group = (seg.bits == 16) ? kHeadDim : seg.group;
#define KVQ_D(B, G_) \
  if (bits == B && group == G_) return launch_split<B, G_>(a, seg, s);
  KVQ_D(16, 128)
  KVQ_D(8, 32) KVQ_D(8, 64) KVQ_D(8, 128)
  KVQ_D(4, 32) KVQ_D(4, 64) KVQ_D(4, 128)
  KVQ_D(2, 32) KVQ_D(2, 64) KVQ_D(2, 128)
#undef KVQ_D
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t s) {
  decode_merge_kernel<<<(unsigned)((long long)a.batch * a.q_heads), kHeadDim, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
