// kvq_oaken.cu -- the Oaken group-shift codec ("大模型KV缓存量化技术：原理、
// 优化与实践" page: section 3.1, thresholds fixed offline and applied online
// with group-shift quantization and a dense-sparse encoding; 3.2.1, the
// outer zone at 5-7 bits, the inner and middle zones at 4 bits; 3.2.2, the
// outer values shifted by the threshold they crossed, Delta = value - T_hi
// or value - T_lo, and dequantized as T + Delta * scale).
//
// Encoding of one token row of head_dim values with the plane's offline
// (s_in, z_in, s_out, b): T_lo = -z_in s_in, T_hi = (15 - z_in) s_in.
//   T_lo <= v <= T_hi: code c = clamp(rne(v / s_in) + z_in, 0, 15);
//   v > T_hi: c = 15, outlier +min(rne((v - T_hi) / s_out), 2^b - 1);
//   v < T_lo: c = 0,  outlier -min(rne((T_lo - v) / s_out), 2^b - 1).
// Dense part: the 4-bit codes, packed two per byte (low nibble first).
// Sparse part: KVQ_OAKEN_SLOTS 16-bit slots per row, the outliers in
// ascending dim order (dim in the low byte, signed magnitude in the high
// byte), zeros after them; outliers past the last slot are dropped.
// x_hat = (c - z_in) s_in + d s_out, d = the element's slot value: for an
// outlier the dense part is its threshold and the slot adds the shift.
//
// Kernels:
//   oaken_quantize_kernel: quantize-on-write, half a warp per row (8 dims a
//     lane), the outliers' slots placed by a shuffle scan of the lanes'
//     counts.  HBM-bound: 256 B read and 96 B written per row.
//   oaken_decode_kernel<G>: split-K decode attention, one CTA per (sequence,
//     KV head, split), four warps taking 32-token tiles in turn.  QK: lane =
//     token, the dense dot sum_j q_j (c_j - z_in) with the codes turned into
//     floats by the 2^23 trick, plus the slots' s_out d q_idx terms.  PV:
//     each lane writes its token's dequantized V row (dense + slots) to a
//     padded fp32 tile in shared memory, then lane = 4 dims accumulates
//     p_t x_hat_t over the tile.  Online softmax in log2 units; the partials
//     go through the same in-CTA merge and workspace as the other decode
//     kernels.  HBM-bound: 2 x (64 + 32) bytes per KV-head token.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>

#include "kvq_decode_common.cuh"
#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant_core.cuh"

namespace kvq {

namespace {

constexpr int D = kHeadDim;
constexpr int kSlots = KVQ_OAKEN_SLOTS;
constexpr int kRowBytes = D / 2;         // 4-bit codes of one row
constexpr int kSlotBytes = kSlots * 2;   // outlier slots of one row

// One element: its 4-bit code, and its signed outlier magnitude (0 inside).
__device__ __forceinline__ uint32_t oaken_code(float v, const OakenParams& p, int& d,
                                               bool& outlier) {
  if (v > p.t_hi) {
    const float m = fminf(rintf(__fdiv_rn(v - p.t_hi, p.s_out)), p.m_max);
    d = (int)m;
    outlier = true;
    return 15u;
  }
  if (v < p.t_lo) {
    const float m = fminf(rintf(__fdiv_rn(-(v - p.t_lo), p.s_out)), p.m_max);
    d = -(int)m;
    outlier = true;
    return 0u;
  }
  // the IEEE quotient by the fp16 scale (div_rn with its reciprocal), then
  // round half to even and the integer zero point
  const float c = fminf(fmaxf(rintf(div_rn(v, p.s_in, p.r_in)) + p.z, 0.0f), 15.0f);
  d = 0;
  outlier = false;
  return (uint32_t)c;
}

// Half a warp per row: lane li of the half owns dims 8 li .. 8 li + 7.
__global__ void __launch_bounds__(256) oaken_quantize_kernel(const QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const int li = lane & 15;
  const unsigned half_mask = (lane < 16) ? 0x0000FFFFu : 0xFFFF0000u;
  const long long per_plane = (long long)a.batch * a.kv_heads * a.n_new;
  const long long rows = 2 * per_plane;
  const long long stride = (long long)gridDim.x * (blockDim.x / 16);
  for (long long r = (long long)blockIdx.x * (blockDim.x / 16) + (threadIdx.x >> 4); r < rows;
       r += stride) {
    const int plane = r >= per_plane;
    const long long rr = plane ? r - per_plane : r;
    const int i = (int)(rr % a.n_new);
    const long long bh = rr / a.n_new;
    const int b = (int)(bh / a.kv_heads);
    const int pos = a.seq_lens[b] + i;
    if (pos >= a.max_tokens) continue;  // the whole half-warp skips together
    const OakenParams& p = plane ? a.v_oaken : a.k_oaken;
    const __half* src = (plane ? a.v_new : a.k_new) + rr * D;
    const long long dst_row = bh * a.max_tokens + pos;
    uint8_t* codes = (plane ? a.v_codes : a.k_codes) + dst_row * kRowBytes;
    uint16_t* slots =
        reinterpret_cast<uint16_t*>((plane ? a.v_meta : a.k_meta) + dst_row * kSlotBytes);

    const uint4 raw = reinterpret_cast<const uint4*>(src)[li];
    const __half* hv = reinterpret_cast<const __half*>(&raw);
    uint32_t word = 0, flags = 0;
    int dv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      bool o;
      word |= oaken_code(__half2float(hv[e]), p, dv[e], o) << (4 * e);
      flags |= (uint32_t)o << e;
    }
    reinterpret_cast<uint32_t*>(codes)[li] = word;
    // slot positions: exclusive prefix of the lanes' outlier counts
    const int cnt = __popc(flags);
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) {
      const int t = __shfl_up_sync(half_mask, incl, off, 16);
      if (li >= off) incl += t;
    }
    const int total = __shfl_sync(half_mask, incl, 15, 16);
    int k = incl - cnt;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if ((flags >> e) & 1u) {
        if (k < kSlots)
          slots[k] = (uint16_t)((uint32_t)(8 * li + e) | ((uint32_t)(uint8_t)(int8_t)dv[e] << 8));
        ++k;
      }
    if (li >= total) slots[li] = 0;  // kSlots == 16 lanes: one empty slot each
  }
}

__global__ void oaken_advance_kernel(int32_t* seq_lens, int batch, int n_new, int max_tokens) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch) seq_lens[b] = min(seq_lens[b] + n_new, max_tokens);
}

// Decode attention.  Shared memory (floats): per warp a V tile of 32 rows
// of D + 4 (a stride of 4 mod 32 banks: a lane's row stores and the slot
// adds stay spread) and the tile's weights [32][G]; the query rows as fp32
// [D][G]; the merge scratch.
constexpr int kTileTok = 32;
constexpr int kVStride = D + 4;

template <int G>
struct OakenCfg {
  static constexpr int WARP_FLOATS = kTileTok * kVStride + kTileTok * G;
  static constexpr int Q_OFF = kWarps * WARP_FLOATS;
  static constexpr int QH_OFF = Q_OFF + D * G;       // fp16 query rows (D * G halves)
  static constexpr int MISC_OFF = QH_OFF + D * G / 2;
  // merge: ms, ls [kWarps * 8], scratch [8 * (kWarps + 2)]; os reuses the tiles
  static constexpr int FLOATS = MISC_OFF + 2 * kWarps * 8 + 8 * (kWarps + 2);
  static constexpr int SMEM = FLOATS * 4;
  static_assert(kWarps * 8 * D <= kWarps * WARP_FLOATS, "merge outputs fit the tiles");
};

template <int G>
__global__ void __launch_bounds__(kWarps * 32) oaken_decode_kernel(const __grid_constant__ SplitParams P) {
  using C = OakenCfg<G>;
  const DecodeArgs& a = P.a;
  const SegView& seg = P.seg;
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

  const int n_split = seg.n_split;
  const int unit = blockIdx.x;
  const int split = unit % n_split;
  const int bh = unit / n_split;
  const int b = bh / a.kv_heads, kvh = bh % a.kv_heads;

  // the query rows as fp32 [D][G], straight from the fp16 or bf16 inputs
  // (exact; this kernel's arithmetic is fp32 throughout)
  float* qf = sm + C::Q_OFF;
  {
    const uint16_t* qg = static_cast<const uint16_t*>(a.q) +
                         ((long long)b * a.q_heads + (long long)kvh * G) * D;
    for (int i = t; i < D * G; i += kWarps * 32) {
      const int j = i / G, h = i % G;
      const uint16_t u = qg[h * D + j];
      qf[i] = a.q_is_bf16 ? __uint_as_float((uint32_t)u << 16)
                          : __half2float(__ushort_as_half(u));
    }
  }
  __syncthreads();

  const int L = seg.seq_lens[b];
  int c0, c1;
  split_range(L, n_split, split, c0, c1);

  const OakenParams kp = seg.k_oaken, vp = seg.v_oaken;
  const float kz = 8388608.0f + kp.z;  // (2^23 | c) - (2^23 + z) = c - z exactly
  const long long row0 = (long long)bh * seg.max_tokens;
  float* vt = sm + warp * C::WARP_FLOATS;   // [32][kVStride]
  float* pw = vt + kTileTok * kVStride;     // [32][G]

  float m[G], lsum[G], acc[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    lsum[h] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[h][k] = 0.f;
  }

  for (int tile = c0 + warp * kTileTok; tile < c1; tile += kWarps * kTileTok) {
    const int tok = tile + lane;
    const bool valid = tok < c1;
    uint4 kc[4], vc[4], ks[2], vs[2];
    if (valid) {
      const long long row = row0 + tok;
      const uint4* kr = reinterpret_cast<const uint4*>(seg.k_codes + row * kRowBytes);
      const uint4* vr = reinterpret_cast<const uint4*>(seg.v_codes + row * kRowBytes);
      const uint4* ksr = reinterpret_cast<const uint4*>(seg.k_meta + row * kSlotBytes);
      const uint4* vsr = reinterpret_cast<const uint4*>(seg.v_meta + row * kSlotBytes);
#pragma unroll
      for (int i = 0; i < 4; ++i) kc[i] = kr[i];
#pragma unroll
      for (int i = 0; i < 4; ++i) vc[i] = vr[i];
      ks[0] = ksr[0]; ks[1] = ksr[1];
      vs[0] = vsr[0]; vs[1] = vsr[1];
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) kc[i] = vc[i] = make_uint4(0, 0, 0, 0);
      ks[0] = ks[1] = vs[0] = vs[1] = make_uint4(0, 0, 0, 0);
    }

    // ---- QK: dense dot over the codes, then the slots
    float dot[G], sp[G];
#pragma unroll
    for (int h = 0; h < G; ++h) dot[h] = sp[h] = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w4[4] = {kc[i].x, kc[i].y, kc[i].z, kc[i].w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = (i * 4 + wi) * 8 + e;
          const float cz = __uint_as_float(0x4B000000u | ((w4[wi] >> (4 * e)) & 15u)) - kz;
#pragma unroll
          for (int h = 0; h < G; ++h) dot[h] = fmaf(qf[j * G + h], cz, dot[h]);
        }
      }
    }
    {
      const uint32_t sw[8] = {ks[0].x, ks[0].y, ks[0].z, ks[0].w, ks[1].x, ks[1].y, ks[1].z, ks[1].w};
#pragma unroll
      for (int s = 0; s < kSlots; ++s) {
        const uint32_t w = (sw[s / 2] >> (16 * (s % 2))) & 0xFFFFu;
        const int d = (int)(int8_t)(uint8_t)(w >> 8);
        const int idx = (int)(w & 0x7Fu);
        if (d != 0) {
#pragma unroll
          for (int h = 0; h < G; ++h) sp[h] = fmaf(qf[idx * G + h], (float)d, sp[h]);
        }
      }
    }
    float sc[G];
#pragma unroll
    for (int h = 0; h < G; ++h)
      sc[h] = valid ? a.scale_log2 * fmaf(kp.s_in, dot[h], kp.s_out * sp[h]) : -INFINITY;

    // ---- V row of this lane's token: dense part, then the slots
    float* vrow = vt + lane * kVStride;
    const float vz = 8388608.0f + vp.z;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w4[4] = {vc[i].x, vc[i].y, vc[i].z, vc[i].w};
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          x[e] = (__uint_as_float(0x4B000000u | ((w4[wi] >> (4 * e)) & 15u)) - vz) * vp.s_in;
        float4* dst = reinterpret_cast<float4*>(vrow + (i * 4 + wi) * 8);
        dst[0] = make_float4(x[0], x[1], x[2], x[3]);
        dst[1] = make_float4(x[4], x[5], x[6], x[7]);
      }
    }
    {
      const uint32_t sw[8] = {vs[0].x, vs[0].y, vs[0].z, vs[0].w, vs[1].x, vs[1].y, vs[1].z, vs[1].w};
#pragma unroll
      for (int s = 0; s < kSlots; ++s) {
        const uint32_t w = (sw[s / 2] >> (16 * (s % 2))) & 0xFFFFu;
        const int d = (int)(int8_t)(uint8_t)(w >> 8);
        if (d != 0) vrow[w & 0x7Fu] += (float)d * vp.s_out;
      }
    }

    // ---- online softmax over the tile (log2 units)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = sc[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[h], mx);  // finite: the tile has a valid token
      const float alpha = exp2f(m[h] - m_new);
      m[h] = m_new;
      const float p = valid ? exp2f(sc[h] - m_new) : 0.f;
      pw[lane * G + h] = p;
      lsum[h] = lsum[h] * alpha + p;
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[h][k] *= alpha;
    }
    __syncwarp();

    // ---- PV: lane = dims 4 lane .. 4 lane + 3
    const int n_tok = min(kTileTok, c1 - tile);
    for (int tt = 0; tt < n_tok; ++tt) {
      const float4 xv = reinterpret_cast<const float4*>(vt + tt * kVStride)[lane];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float p = pw[tt * G + h];
        acc[h][0] = fmaf(p, xv.x, acc[h][0]);
        acc[h][1] = fmaf(p, xv.y, acc[h][1]);
        acc[h][2] = fmaf(p, xv.z, acc[h][2]);
        acc[h][3] = fmaf(p, xv.w, acc[h][3]);
      }
    }
    __syncwarp();  // the next tile rewrites vt and pw
  }

  // ---- warp results to shared memory, then the CTA merge and the store
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum[h] += __shfl_xor_sync(0xffffffffu, lsum[h], off);
  __syncthreads();  // every warp is done with its tile before os overwrites them
  float* os = sm;
  float* ms = sm + C::MISC_OFF;
  float* ls = ms + kWarps * 8;
  float* scratch = ls + kWarps * 8;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    reinterpret_cast<float4*>(os + (warp * 8 + h) * D)[lane] =
        make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
    if (lane == 0) {
      ms[warp * 8 + h] = m[h];
      ls[warp * 8 + h] = lsum[h];
    }
  }
  __syncthreads();
  cta_merge_store<G>(a, ms, ls, os, scratch, b, kvh, seg.part_base + split, t);
}

template <int G>
cudaError_t launch_oaken_g(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  using C = OakenCfg<G>;
  // the shared-memory opt-in is per device (bit i of the mask = device i)
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(oaken_decode_kernel<G>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  const long long units = (long long)seg.n_split * a.kv_heads * a.batch;
  if (units <= 0) return cudaSuccess;
  oaken_decode_kernel<G><<<(unsigned)units, kWarps * 32, C::SMEM, s>>>(SplitParams{a, seg});
  return cudaGetLastError();
}

}  // namespace

OakenParams make_oaken_params(float s_in, int z_in, float s_out, int outer_bits) {
  OakenParams p;
  p.s_in = s_in;
  p.r_in = 1.0f / s_in;  // host IEEE division: the correctly rounded reciprocal
  p.z = (float)z_in;
  p.t_lo = -p.z * s_in;
  p.t_hi = (15.0f - p.z) * s_in;
  p.s_out = s_out;
  p.m_max = (float)((1 << outer_bits) - 1);
  return p;
}

cudaError_t launch_oaken_quantize(const QuantArgs& a, cudaStream_t s) {
  const long long rows = 2LL * a.batch * a.kv_heads * a.n_new;
  const long long blocks = (rows + 15) / 16;
  const long long cap = (long long)device_sm_count() * 8;
  const unsigned grid = (unsigned)(blocks < cap ? blocks : cap);
  oaken_quantize_kernel<<<grid, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.advance) return e;
  oaken_advance_kernel<<<(a.batch + 127) / 128, 128, 0, s>>>(a.seq_lens, a.batch, a.n_new,
                                                             a.max_tokens);
  return cudaGetLastError();
}

bool decode_oaken_supported(int group_ratio) {
  return group_ratio == 1 || group_ratio == 2 || group_ratio == 4 || group_ratio == 8;
}

int decode_oaken_ctas_per_sm(int group_ratio) {
  const int smem = group_ratio == 8 ? OakenCfg<8>::SMEM : OakenCfg<4>::SMEM;
  return 227 * 1024 / (smem + 1024);
}

cudaError_t launch_decode_oaken(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  switch (a.group_ratio) {
    case 1: return launch_oaken_g<1>(a, seg, s);
    case 2: return launch_oaken_g<2>(a, seg, s);
    case 4: return launch_oaken_g<4>(a, seg, s);
    case 8: return launch_oaken_g<8>(a, seg, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace kvq
