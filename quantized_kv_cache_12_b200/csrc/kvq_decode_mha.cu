// kvq_decode_mha.cu -- split-K decode attention for one query head per KV
// head (multi-head attention), with the tokens on the M dimension of the
// tensor-core tiles.  Same work units, stage ring, arithmetic identities and
// partial-result format as the grouped-query kernel in kvq_decode.cu
// (TurboQuant page 2.3, last paragraph: dequantization inside the attention
// products; Cocktail page 3.2.3: log-sum-exp merge of the pieces).
//
// Why a second kernel.  With a single query row, putting (group, head) rows
// on M (as the grouped kernel does) fills 2 to 8 of the 16 rows of every
// m16n8k16 tile.  Here both products are transposed:
//   S^T = K * Qx^T   rows = 16 tokens, k = 16 dims, columns = the NG groups
//                    (column c holds q masked to group c): 8 MMAs / 16 tokens
//   O^T = V^T * P'^T rows = 16 dims, k = 16 tokens, columns = (group, hi/lo)
//                    parts of P' = p * s_V: 8 MMAs / 16 tokens
// half the MMAs and half the accumulator registers of the grouped kernel at
// g = 1, and the code conversions are shared by all columns.
//
// Lane roles (gid = lane / 4, tig = lane % 4), per 16-token sub-tile:
//   QK: A rows gid, gid + 8 are tokens gid, gid + 8; the lane's k elements are
//       its 32-dim chunk [32 tig, 32 tig + 32) of those tokens; B column gid
//       is q (scaled by the code's power of two) masked to group gid.
//   PV: k positions 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 are tokens tig,
//       tig + 4, tig + 8, tig + 12 (that order makes the 4-byte V loads of a
//       warp one contiguous 128-byte block); A rows gid, gid + 8 of m-tile mt
//       are dims 16 gid + mt and 16 gid + mt + 8, so a lane reads the 16
//       contiguous dims [16 gid, 16 gid + 16) of each of its four tokens; B
//       column gid is the hi (gid even) or lo (gid odd) fp16 part of
//       P' = p * s_V for group gid / 2.
// The output for dim d sits in lane (d / 16, group(d)), columns 2 tig (hi)
// and 2 tig + 1 (lo).
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>
#include <type_traits>

#include "kvq_decode_common.cuh"
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

template <int BITS, int GE>
struct MhaCfg {
  static constexpr int D = kHeadDim;
  static constexpr int NG = D / GE;                    // groups per token (<= 4)
  static constexpr int RB = D * BITS / 8;              // code bytes per token
  static constexpr int MB = (BITS == 16) ? 0 : NG * 4; // (s, z) bytes per token
  static constexpr int KC = RB / 4;                    // K bytes of a lane (32 dims)
  static constexpr int KW = KC / 4;
  static constexpr int VB = RB / 8;                    // V bytes of a lane (16 dims)
  static constexpr int VW = VB / 4;
  static constexpr int SUB = (BITS == 16) ? 1 : 2;     // 16-token sub-tiles per stage
  static constexpr int STOK = SUB * kTile;
  static constexpr int STAGE = 2 * STOK * RB + 2 * STOK * MB;
  // header: mbarriers (<= 512 B), q as fp16 (256 B), group sums of q,
  // unit id and fail flag
  static constexpr int HDR_BARS = 0, HDR_Q = 512, HDR_QS = HDR_Q + D * 2;
  static constexpr int HDR_MISC = HDR_QS + 64;
  static constexpr int HDR_BYTES = 1024;
  // four CTAs per SM where three stages per warp fit in a quarter of the SM's
  // shared memory (4 x (56 KB + 1 KB reserved) <= 228 KB), else three
  static constexpr int MIN_CTAS = (HDR_BYTES + kWarps * 3 * STAGE <= 56 * 1024) ? 4 : 3;
  static constexpr int SMEM_BUDGET = (MIN_CTAS == 4 ? 56 : 74) * 1024;
  static constexpr int STAGES_RAW = (SMEM_BUDGET - HDR_BYTES) / (kWarps * STAGE);
  static constexpr int STAGES = STAGES_RAW < 2 ? 2 : (STAGES_RAW > 16 ? 16 : STAGES_RAW);
  static constexpr int SMEM = HDR_BYTES + kWarps * STAGES * STAGE;
  static constexpr int EMAX = WordPairs<BITS>::kEmax;
  // the warp merge reuses the stage buffers: m, l, o of kWarps x 8 rows
  static constexpr int MERGE_BYTES = (2 * kWarps * 8 + kWarps * 8 * D + 8 * (kWarps + 2)) * 4;
  static_assert(NG <= 4, "at most four groups per token");
  static_assert(kWarps * STAGES * 8 <= HDR_Q, "mbarriers fit the header");
  static_assert(HDR_MISC + 8 <= HDR_BYTES, "header layout");
  static_assert(MERGE_BYTES <= kWarps * STAGES * STAGE, "merge scratch fits the stages");
  static_assert(WordPairs<BITS>::kPairs * KW == 16, "16 K pairs per lane and token");
  static_assert(CrossPairs<BITS>::kOut * VW == 16, "16 V dims per lane and token");
};

template <int BITS, int GE>
__global__ void __launch_bounds__(kWarps * 32, MhaCfg<BITS, GE>::MIN_CTAS)
decode_mha_kernel(const __grid_constant__ SplitParams P) {
  using C = MhaCfg<BITS, GE>;
  using WP = WordPairs<BITS>;
  using XP = CrossPairs<BITS>;
  constexpr int D = C::D, NG = C::NG;
  const DecodeArgs& a = P.a;
  const SegView& seg = P.seg;

  extern __shared__ __align__(128) uint8_t smem[];
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int gid = lane >> 2, tig = lane & 3;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::HDR_BARS) + warp * C::STAGES;
  __half* q_sm = reinterpret_cast<__half*>(smem + C::HDR_Q);
  float* qs_sm = reinterpret_cast<float*>(smem + C::HDR_QS);
  int* unit_sm = reinterpret_cast<int*>(smem + C::HDR_MISC);
  int* fail_sm = unit_sm + 1;
  uint8_t* stages = smem + C::HDR_BYTES + warp * C::STAGES * C::STAGE;
  uint32_t* counters = a.err + 1;  // [0] next unit, [1] CTAs done

  // ---- per-lane constants
  const int kgrp = (32 * tig) / GE;          // group of this lane's K chunk
  const bool colA = 2 * tig < NG;            // QK accumulator columns 2 tig,
  const bool colB = 2 * tig + 1 < NG;        // 2 tig + 1 are real groups
  const int gv = gid >> 1;                   // PV: B column gid = (gv, hi/lo)
  const bool pv_ok = gv < NG;
  const int gvc = pv_ok ? gv : 0;            // clamped for addressing
  const float lo_sel = (gid & 1) ? 1.f : 0.f;
  const bool writer = tig == (16 * gid) / GE;  // holds the output of its 16 dims
  const float score_scale = a.scale_log2 * pow2f(24 - C::EMAX);
  const int vt[4] = {tig, tig + 4, tig + 8, tig + 12};  // PV tokens of this lane

  const uint64_t policy = l2_evict_first_policy();
  int st = 0;  // the stage ring (position and phase) runs on across units
  uint32_t phase = 0;
  if (lane == 0) {
    for (int s2 = 0; s2 < C::STAGES; ++s2) mbar_init(&bars[s2], 1);
    fence_barrier_init();
  }
  if (t == 0) *fail_sm = 0;
  __syncwarp();
  const int units = seg.n_split * a.kv_heads * a.batch;

  for (;;) {
  if (t == 0) *unit_sm = (int)atomicAdd(&counters[0], 1u);
  __syncthreads();
  const int unit = *unit_sm;
  if (unit >= units || *fail_sm) break;
  const int split = unit % seg.n_split;
  const int kvh = (unit / seg.n_split) % a.kv_heads;
  const int b = unit / (seg.n_split * a.kv_heads);

  int L = seg.seq_lens[b];
  L = max(0, min(L, seg.max_tokens));
  int c0, c1;
  split_range(L, seg.n_split, split, c0, c1);
  const int unit_stages = (c1 > c0) ? (c1 - c0 + C::STOK - 1) / C::STOK : 0;
  const int n_tiles = (unit_stages > warp) ? (unit_stages - warp + kWarps - 1) / kWarps : 0;
  const int w0 = c0 + warp * C::STOK;  // first token of this warp's first stage

  const long long row0 = ((long long)b * a.kv_heads + kvh) * seg.max_tokens + w0;
  const uint8_t* kc_src = seg.k_codes + row0 * C::RB;
  const uint8_t* vc_src = seg.v_codes + row0 * C::RB;
  const uint8_t* km_src = seg.k_meta + row0 * C::MB;
  const uint8_t* vm_src = seg.v_meta + row0 * C::MB;
  auto issue = [&](int i, int st) {
    uint8_t* dst = stages + st * C::STAGE;
    mbar_arrive_expect_tx(&bars[st], C::STAGE);
    const size_t tok = (size_t)i * (kWarps * C::STOK);
    bulk_load(dst, kc_src + tok * C::RB, C::STOK * C::RB, &bars[st], policy);
    bulk_load(dst + C::STOK * C::RB, vc_src + tok * C::RB, C::STOK * C::RB, &bars[st], policy);
    if constexpr (C::MB > 0) {
      bulk_load(dst + 2 * C::STOK * C::RB, km_src + tok * C::MB, C::STOK * C::MB, &bars[st],
                policy);
      bulk_load(dst + 2 * C::STOK * C::RB + C::STOK * C::MB, vm_src + tok * C::MB,
                C::STOK * C::MB, &bars[st], policy);
    }
  };
  if (lane == 0) {
    const int pre = min(n_tiles, C::STAGES);
    for (int i = 0; i < pre; ++i) issue(i, (st + i) % C::STAGES);
  }

  // ---- the query of this head, once per unit
  stage_queries<1>(a, b, kvh, q_sm, t);
  __syncthreads();
  // group sums of q in the QK MMA's units (it returns 2^(EMAX - 24) sum q c)
  if constexpr (BITS != 16) {
    if (t < 32) {
      const int r = t >> 3, part = t & 7;
      float acc = 0.f;
      if (r < NG) {
        const __half* qr = q_sm + r * GE + part * (GE / 8);
#pragma unroll 4
        for (int i = 0; i < GE / 8; ++i) acc += __half2float(qr[i]);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (r < NG && part == 0) qs_sm[r] = acc * pow2f(C::EMAX - 24);
    }
  }
  __syncthreads();
  // B fragments of QK: pair p = 2 ks + h of this lane's chunk, column gid;
  // each element scaled by 2^(EMAX - e) for the exponent e of its code
  uint32_t qb[8][2];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = 2 * ks + h;
      const int j = p % WP::kPairs;
      const int d0 = 32 * tig + (p / WP::kPairs) * WP::kDims + WP::dim(j, 0);
      const int d1 = 32 * tig + (p / WP::kPairs) * WP::kDims + WP::dim(j, 1);
      const float f = pow2f(C::EMAX - WP::exp(j));
      qb[ks][h] = (gid == kgrp) ? pack_h2(__half2float(q_sm[d0]) * f, __half2float(q_sm[d1]) * f)
                                : 0u;
    }
  }
  const float qsA = (BITS != 16 && colA) ? qs_sm[2 * tig] : 0.f;
  const float qsB = (BITS != 16 && colB) ? qs_sm[2 * tig + 1] : 0.f;

  // ---- running state.  m_ref is a reference point at least as large as
  // every score seen, so p = 2^(x - m_ref) <= 1 and P' = p * s_V stays
  // within fp16 range; it moves (with a rescale) only when a stage's max
  // exceeds it, and then to that max + kLazy.
  float o_acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float corr = 0.f;  // sum of P' * z_V for group gv
  constexpr float kLazy = 4.0f;
  float m_ref = -INFINITY, l_part = 0.f;
  int failed_at = -1;
  const int st0 = st;
  const uint32_t phase0 = phase;

  auto stage_body = [&](auto full_tag, const uint8_t* sK, const uint8_t* sV, const uint8_t* sKm,
                        const uint8_t* sVm, int n_valid) {
    constexpr bool FULL = decltype(full_tag)::value;
    constexpr int NS = C::SUB;
    auto valid = [&](int tok) { return FULL || tok < n_valid; };  // tok: 0 .. STOK-1

    // ---- S^T = K * Qx^T per sub-tile: this lane's rows are tokens gid, gid + 8
    float sc[NS][2];
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
      float s_acc[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t k0[C::KW], k1[C::KW];
      load_chunk<C::KC, C::KW>(sK + (sub * kTile + gid) * C::RB + tig * C::KC, k0);
      load_chunk<C::KC, C::KW>(sK + (sub * kTile + gid + 8) * C::RB + tig * C::KC, k1);
      uint32_t p0[16], p1[16];
#pragma unroll
      for (int w = 0; w < C::KW; ++w) {
        uint32_t x0[WP::kPairs], x1[WP::kPairs];
        WP::run(k0[w], x0);
        WP::run(k1[w], x1);
#pragma unroll
        for (int j = 0; j < WP::kPairs; ++j) {
          p0[w * WP::kPairs + j] = x0[j];
          p1[w * WP::kPairs + j] = x1[j];
        }
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_f16(s_acc, p0[2 * ks], p1[2 * ks], p0[2 * ks + 1], p1[2 * ks + 1], qb[ks][0],
                qb[ks][1]);
      // score = sum over this lane's group columns of s_K * (S - z_K * qs);
      // rows past the valid length may hold any bytes: masked below by select
      if constexpr (BITS == 16) {
        sc[sub][0] = s_acc[0];
        sc[sub][1] = s_acc[2];
      } else {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint8_t* m = sKm + (sub * kTile + gid + 8 * r) * C::MB;
          float v = 0.f;
          if constexpr (NG == 1) {
            if (colA) {
              const float2 sz = __half22float2(*reinterpret_cast<const __half2*>(m));
              v = sz.x * fmaf(-sz.y, qsA, s_acc[2 * r]);
            }
          } else {
            if (colA) {
              const uint2 u = *reinterpret_cast<const uint2*>(m + 8 * tig);
              const float2 szA = __half22float2(u32_as_h2(u.x));
              const float2 szB = __half22float2(u32_as_h2(u.y));
              v = fmaf(szB.x, fmaf(-szB.y, qsB, s_acc[2 * r + 1]),
                       szA.x * fmaf(-szA.y, qsA, s_acc[2 * r]));
            }
          }
          sc[sub][r] = v;
        }
        if constexpr (NG == 4) {
#pragma unroll
          for (int r = 0; r < 2; ++r) sc[sub][r] += __shfl_xor_sync(0xffffffffu, sc[sub][r], 1);
        }
      }
    }

    // ---- to the PV layout: lane (., tig) takes tokens tig, tig + 4, tig + 8,
    // tig + 12 from the tig = 0 lanes of rows tig and tig + 4
    float x[NS][4];
    float tmax = -INFINITY;
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
      x[sub][0] = __shfl_sync(0xffffffffu, sc[sub][0], 4 * tig);
      x[sub][1] = __shfl_sync(0xffffffffu, sc[sub][0], 4 * tig + 16);
      x[sub][2] = __shfl_sync(0xffffffffu, sc[sub][1], 4 * tig);
      x[sub][3] = __shfl_sync(0xffffffffu, sc[sub][1], 4 * tig + 16);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        x[sub][k] = valid(sub * kTile + vt[k]) ? x[sub][k] * score_scale : -INFINITY;
        tmax = fmaxf(tmax, x[sub][k]);
      }
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    if (tmax > m_ref) {  // warp-uniform
      const float m_new = tmax + kLazy;
      if (m_ref != -INFINITY) {
        const float alpha = fast_exp2(m_ref - m_new);
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int c = 0; c < 4; ++c) o_acc[n][c] *= alpha;
        corr *= alpha;
        l_part *= alpha;
      }
      m_ref = m_new;
    }

    // ---- O^T += V^T * P'^T per sub-tile
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
      float pp[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float p = fast_exp2(x[sub][k] - m_ref);  // 0 for masked tokens
        l_part += p;
        if constexpr (BITS == 16) {
          pp[k] = pv_ok ? p : 0.f;
        } else {
          // slots past the valid length may hold any bytes (NaN scales):
          // select, never multiply by a zero weight
          const bool ok = pv_ok && valid(sub * kTile + vt[k]);
          const float2 sz = __half22float2(*reinterpret_cast<const __half2*>(
              sVm + (sub * kTile + vt[k]) * C::MB + gvc * 4));
          pp[k] = ok ? p * sz.x : 0.f;
          corr = ok ? fmaf(pp[k], sz.y, corr) : corr;
        }
      }
      // hi part in even columns, lo = P' - hi in odd ones
      const float2 h01 = __half22float2(__floats2half2_rn(pp[0], pp[1]));
      const float2 h23 = __half22float2(__floats2half2_rn(pp[2], pp[3]));
      const uint32_t b0 = pack_h2(fmaf(-lo_sel, h01.x, pp[0]), fmaf(-lo_sel, h01.y, pp[1]));
      const uint32_t b1 = pack_h2(fmaf(-lo_sel, h23.x, pp[2]), fmaf(-lo_sel, h23.y, pp[3]));

      const uint8_t* vb = sV + sub * kTile * C::RB + gid * C::VB;
      uint32_t wA[C::VW], wB[C::VW], wC[C::VW], wD[C::VW];
      load_chunk<C::VB, C::VW>(vb + vt[0] * C::RB, wA);
      load_chunk<C::VB, C::VW>(vb + vt[1] * C::RB, wB);
      load_chunk<C::VB, C::VW>(vb + vt[2] * C::RB, wC);
      load_chunk<C::VB, C::VW>(vb + vt[3] * C::RB, wD);
      if constexpr (BITS == 16 && !FULL) {
        // raw fp16 rows past the valid length may hold anything: zero them
#pragma unroll
        for (int w = 0; w < C::VW; ++w) {
          wA[w] = valid(sub * kTile + vt[0]) ? wA[w] : 0u;
          wB[w] = valid(sub * kTile + vt[1]) ? wB[w] : 0u;
          wC[w] = valid(sub * kTile + vt[2]) ? wC[w] : 0u;
          wD[w] = valid(sub * kTile + vt[3]) ? wD[w] : 0u;
        }
      }
      uint32_t xa[16], xc[16];
#pragma unroll
      for (int w = 0; w < C::VW; ++w) {
        uint32_t ya[XP::kOut], yc[XP::kOut];
        XP::run(wA[w], wB[w], ya);
        XP::run(wC[w], wD[w], yc);
#pragma unroll
        for (int i = 0; i < XP::kOut; ++i) {
          xa[w * XP::kOut + i] = ya[i];
          xc[w * XP::kOut + i] = yc[i];
        }
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) mma_f16(o_acc[mt], xa[mt], xa[mt + 8], xc[mt], xc[mt + 8], b0, b1);
    }
  };

  for (int i = 0; i < n_tiles; ++i) {
    if (!mbar_wait_bounded(&bars[st], phase, 1u << 22)) {
      failed_at = i;
      break;
    }
    const uint8_t* sK = stages + st * C::STAGE;
    const uint8_t* sV = sK + C::STOK * C::RB;
    const uint8_t* sKm = sK + 2 * C::STOK * C::RB;
    const uint8_t* sVm = sKm + C::STOK * C::MB;
    const int n_stage = min(C::STOK, c1 - (w0 + i * kWarps * C::STOK));
    if (n_stage == C::STOK)
      stage_body(std::integral_constant<bool, true>(), sK, sV, sKm, sVm, C::STOK);
    else
      stage_body(std::integral_constant<bool, false>(), sK, sV, sKm, sVm, n_stage);
    __syncwarp();
    if (lane == 0 && i + C::STAGES < n_tiles) issue(i + C::STAGES, st);
    if (++st == C::STAGES) {
      st = 0;
      phase ^= 1u;
    }
  }

  if (failed_at >= 0) {
    if (lane == 0) {
      atomicOr(a.err, kErrWaitTimeout);
      *fail_sm = 1;  // the CTA stops after this unit
    }
    // drain the copies this warp issued and has not consumed (bounded)
    const int issued_end = min(n_tiles, failed_at + C::STAGES);
    for (int i = failed_at; i < issued_end; ++i) {
      const int pos = st0 + i;
      const uint32_t ph = phase0 ^ (uint32_t)((pos / C::STAGES) & 1);
      (void)mbar_wait_bounded(&bars[pos % C::STAGES], ph, 1u << 16);
    }
  }

  // ---- warp totals: every row gid holds the same tokens, so sum over tig
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
  corr += __shfl_xor_sync(0xffffffffu, corr, 1);
  corr += __shfl_xor_sync(0xffffffffu, corr, 2);
  // the correction of group tig, from the hi lane of column 2 tig
  const float corr_t = __shfl_sync(0xffffffffu, corr, 8 * tig);

  __syncthreads();
  float* ms = reinterpret_cast<float*>(smem + C::HDR_BYTES);  // [kWarps][8]
  float* ls = ms + kWarps * 8;                                 // [kWarps][8]
  float* os = ls + kWarps * 8;                                 // [kWarps][8][D]
  if (lane == 0) {
    ms[warp * 8] = m_ref;
    ls[warp * 8] = l_part;
  }
  if (writer) {
    float* oh = os + warp * 8 * D + 16 * gid;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      // undo the subnormal code scale 2^(e - 24) of the row's dim
      const float f0 = pow2f(24 - XP::exp(mt % XP::kOut));
      const float f1 = pow2f(24 - XP::exp((mt + 8) % XP::kOut));
      oh[mt] = fmaf(o_acc[mt][0] + o_acc[mt][1], f0, -corr_t);
      oh[mt + 8] = fmaf(o_acc[mt][2] + o_acc[mt][3], f1, -corr_t);
    }
  }
  __syncthreads();
  cta_merge_store<1>(a, ms, ls, os, os + kWarps * 8 * D, b, kvh, seg.part_base + split, t);
  }  // unit loop

  if (t == 0) release_counters(counters);
}

template <int BITS, int GE>
cudaError_t launch_mha(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  using C = MhaCfg<BITS, GE>;
  // the shared-memory opt-in is a per-device function attribute: set it once
  // per device (bit i of the mask = device i)
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(decode_mha_kernel<BITS, GE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  SplitParams P{a, seg};
  const long long units = (long long)seg.n_split * a.kv_heads * a.batch;
  const long long slots = 148LL * C::MIN_CTAS;  // one wave of persistent CTAs
  const unsigned grid = (unsigned)(units < slots ? units : slots);
  decode_mha_kernel<BITS, GE><<<grid, kWarps * 32, C::SMEM, s>>>(P);
  return cudaGetLastError();
}

}  // namespace

int decode_mha_ctas_per_sm(int bits, int group) {
#define KVQ_S(B, G_) \
  if (bits == B && group == G_) return MhaCfg<B, G_>::MIN_CTAS;
  KVQ_S(16, 128)
  KVQ_S(8, 32) KVQ_S(8, 64) KVQ_S(8, 128)
  KVQ_S(4, 32) KVQ_S(4, 64) KVQ_S(4, 128)
  KVQ_S(2, 32) KVQ_S(2, 64) KVQ_S(2, 128)
#undef KVQ_S
  return 0;
}

cudaError_t launch_decode_mha(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  const int bits = seg.bits, group = (seg.bits == 16) ? kHeadDim : seg.group;
#define KVQ_D(B, G_) \
  if (bits == B && group == G_) return launch_mha<B, G_>(a, seg, s);
  KVQ_D(16, 128)
  KVQ_D(8, 32) KVQ_D(8, 64) KVQ_D(8, 128)
  KVQ_D(4, 32) KVQ_D(4, 64) KVQ_D(4, 128)
  KVQ_D(2, 32) KVQ_D(2, 64) KVQ_D(2, 128)
#undef KVQ_D
  return cudaErrorInvalidValue;
}

}  // namespace kvq
