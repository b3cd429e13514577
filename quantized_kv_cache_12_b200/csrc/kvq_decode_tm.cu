// kvq_decode_tm.cu -- split-K decode attention with the tokens on the M
// dimension of the tensor-core tiles, for query groups of g heads per KV head
// with NG * g <= 8 (NG = head_dim / G groups per token).  Same work units,
// stage ring, arithmetic identities and partial-result format as the kernel
// in kvq_decode.cu, which covers NG * g = 16 (TurboQuant page 2.3, last
// paragraph: dequantization inside the attention products; Cocktail page
// 3.2.3: log-sum-exp merge of the pieces).
//
// Both products are transposed with respect to the textbook form:
//   S^T = K * Qx^T   rows = 16 tokens, k = 16 dims, columns c = h * NG + gr
//                    (query head h masked to group gr): 8 MMAs / 16 tokens
//   O^T = V^T * P'^T rows = 16 dims, k = 16 tokens, columns (h, gr, hi/lo)
//                    of P' = p_h * s_V,gr split into two fp16 parts:
//                    8 MMAs per 8 columns / 16 tokens
// so the code conversions (the bulk of the instruction count) are done once
// per token for all heads and groups, and no MMA row is padding.
//
// Lane roles (gid = lane / 4, tig = lane % 4), per 16-token sub-tile:
//   QK: A rows gid, gid + 8 are tokens gid, gid + 8; the lane's k elements are
//       its 32-dim chunk [32 tig, 32 tig + 32) of those tokens.  Accumulator
//       columns 2 tig, 2 tig + 1 give the lane, for its two tokens, either the
//       scores of heads 2 tig and 2 tig + 1 (NG = 1: two head slots), of head
//       tig (NG = 2), or half of the score of head tig / 2 (NG = 4, completed
//       by one shuffle).  The softmax runs here, per head slot.
//   PV: k positions 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 are tokens tig,
//       tig + 4, tig + 8, tig + 12 (that order makes a warp's V loads one
//       contiguous block); A rows gid, gid + 8 of m-tile mt are dims
//       16 gid + mt and 16 gid + mt + 8, so a lane reads the 16 contiguous dims
//       [16 gid, 16 gid + 16) of each of its four tokens; B column gid of
//       n-tile nt is column nt * 8 + gid = (h, gr, part) of P'.
// The output for head h and dim d sits in n-tile (h * 2NG + 2 group(d)) / 8,
// lane (d / 16, (h * 2NG + 2 group(d)) % 8 / 2), columns hi + lo.
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>
#include <type_traits>

#include "kvq_decode_common.cuh"
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

template <int BITS, int GE, int GR>
struct TmCfg {
  static constexpr int D = kHeadDim;
  static constexpr int NG = D / GE;                    // groups per token
  static constexpr int RB = D * BITS / 8;              // code bytes per token
  static constexpr int MB = (BITS == 16) ? 0 : NG * 4; // (s, z) bytes per token
  static constexpr int KC = RB / 4;                    // K bytes of a lane (32 dims)
  static constexpr int KW = KC / 4;
  static constexpr int VB = RB / 8;                    // V bytes of a lane (16 dims)
  static constexpr int VW = VB / 4;
  static constexpr int NCQ = NG * GR;                  // QK columns (h, gr)
  static constexpr int NCP = 2 * NCQ;                  // PV columns (h, gr, part)
  static constexpr int NP = (NCP + 7) / 8;             // PV n-tiles
  static constexpr int HS = (NG == 1 && GR > 1) ? 2 : 1;  // head slots of a QK lane
  static constexpr int SUB = (BITS == 16) ? 1 : 2;     // 16-token sub-tiles per stage
  static constexpr int STOK = SUB * kTile;
  static constexpr int STAGE = 2 * STOK * RB + 2 * STOK * MB;
  // header: mbarriers (<= 512 B), the g query rows as fp16, the column sums
  // of q, unit id and fail flag
  static constexpr int HDR_BARS = 0, HDR_Q = 512, HDR_QS = HDR_Q + GR * D * 2;
  static constexpr int HDR_MISC = HDR_QS + 64;
  static constexpr int HDR_BYTES = ((HDR_MISC + 8 + 127) / 128) * 128;
  // four CTAs per SM where the registers allow it (one PV n-tile) and three
  // stages per warp fit in a quarter of the SM's shared memory
  // (4 x (56 KB + 1 KB reserved) <= 228 KB), else three
  static constexpr int MIN_CTAS =
      (NP == 1 && HDR_BYTES + kWarps * 3 * STAGE <= 56 * 1024) ? 4 : 3;
  static constexpr int SMEM_BUDGET = (MIN_CTAS == 4 ? 56 : 74) * 1024;
  static constexpr int STAGES_RAW = (SMEM_BUDGET - HDR_BYTES) / (kWarps * STAGE);
  static constexpr int STAGES = STAGES_RAW < 2 ? 2 : (STAGES_RAW > 16 ? 16 : STAGES_RAW);
  static constexpr int SMEM = HDR_BYTES + kWarps * STAGES * STAGE;
  static constexpr int EMAX = WordPairs<BITS>::kEmax;
  // the warp merge reuses the stage buffers: m, l, o of kWarps x 8 rows
  static constexpr int MERGE_BYTES = (2 * kWarps * 8 + kWarps * 8 * D + 8 * (kWarps + 2)) * 4;
  static_assert(NCQ <= 8, "at most eight (head, group) columns");
  static_assert(kWarps * STAGES * 8 <= HDR_Q, "mbarriers fit the header");
  static_assert(MERGE_BYTES <= kWarps * STAGES * STAGE, "merge scratch fits the stages");
  static_assert(WordPairs<BITS>::kPairs * KW == 16, "16 K pairs per lane and token");
  static_assert(CrossPairs<BITS>::kOut * VW == 16, "16 V dims per lane and token");
};

template <int BITS, int GE, int GR>
__global__ void __launch_bounds__(kWarps * 32, TmCfg<BITS, GE, GR>::MIN_CTAS)
decode_tm_kernel(const __grid_constant__ SplitParams P) {
  using C = TmCfg<BITS, GE, GR>;
  using WP = WordPairs<BITS>;
  using XP = CrossPairs<BITS>;
  constexpr int D = C::D, NG = C::NG, NP = C::NP, HS = C::HS;
  const DecodeArgs& a = P.a;
  const SegView& seg = P.seg;

  extern __shared__ __align__(128) uint8_t smem[];
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int gid = lane >> 2, tig = lane & 3;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::HDR_BARS) + warp * C::STAGES;
  __half* q_sm = reinterpret_cast<__half*>(smem + C::HDR_Q);      // [GR][D]
  float* qs_sm = reinterpret_cast<float*>(smem + C::HDR_QS);      // [NCQ]
  int* unit_sm = reinterpret_cast<int*>(smem + C::HDR_MISC);
  int* fail_sm = unit_sm + 1;
  uint8_t* stages = smem + C::HDR_BYTES + warp * C::STAGES * C::STAGE;
  uint32_t* counters = a.err + 1;  // [0] next unit, [1] CTAs done

  // ---- per-lane constants
  // QK B column gid = (head qh, group qg); this lane's K chunk is in group kgrp
  const int kgrp = (32 * tig) / GE;
  const bool qb_ok = gid < C::NCQ && (gid % NG) == kgrp;
  const int qh = (gid < C::NCQ) ? gid / NG : 0;
  // QK accumulator columns 2 tig, 2 tig + 1
  const bool colA = 2 * tig < C::NCQ, colB = 2 * tig + 1 < C::NCQ;
  const int meta_off = 4 * ((2 * tig) % NG);  // (s, z) of column 2 tig's group
  // head of QK slot s of this lane (valid if < GR)
  auto slot_head = [&](int s) { return NG == 1 ? 2 * tig + s : (2 * tig) / NG; };
  // PV B column nt * 8 + gid: head hb, group gv (the same in every n-tile),
  // part gid & 1; its head's scores sit in QK lanes with tig = ts
  const int gv = (gid >> 1) % NG;
  const float lo_sel = (gid & 1) ? 1.f : 0.f;
  bool pv_ok[NP];
  int ts[NP], sl[NP];
#pragma unroll
  for (int nt = 0; nt < NP; ++nt) {
    const int col = nt * 8 + gid;
    const int hb = col / (2 * NG);
    pv_ok[nt] = col < C::NCP;
    ts[nt] = pv_ok[nt] ? (hb * NG) / 2 : 0;
    sl[nt] = (HS == 2) ? (hb & 1) : 0;
  }
  // PV accumulator columns nt * 8 + 2 tig (+1): head ho, group tig % NG; the
  // lane holds outputs where that group is the group of its 16 dims
  int ho[NP];
  bool writer[NP];
#pragma unroll
  for (int nt = 0; nt < NP; ++nt) {
    ho[nt] = (nt * 8 + 2 * tig) / (2 * NG);
    writer[nt] = ho[nt] < GR && (tig % NG) == (16 * gid) / GE;
  }
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

  // ---- the g query rows of this KV head, once per unit
  stage_queries<GR>(a, b, kvh, q_sm, t);
  __syncthreads();
  // column sums of q in the QK MMA's units (it returns 2^(EMAX - 24) sum q c)
  if constexpr (BITS != 16) {
    if (t < 64) {
      const int r = t >> 3, part = t & 7;
      float acc = 0.f;
      if (r < C::NCQ) {
        const __half* qr = q_sm + (r / NG) * D + (r % NG) * GE + part * (GE / 8);
#pragma unroll 4
        for (int i = 0; i < GE / 8; ++i) acc += __half2float(qr[i]);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (r < C::NCQ && part == 0) qs_sm[r] = acc * pow2f(C::EMAX - 24);
    }
  }
  __syncthreads();
  // B fragments of QK: pair p = 2 ks + h of this lane's chunk, column gid;
  // each element scaled by 2^(EMAX - e) for the exponent e of its code
  uint32_t qb[8][2];
  {
    const __half* qrow = q_sm + qh * D + 32 * tig;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int p = 2 * ks + h;
        const int j = p % WP::kPairs;
        const int d0 = (p / WP::kPairs) * WP::kDims + WP::dim(j, 0);
        const int d1 = (p / WP::kPairs) * WP::kDims + WP::dim(j, 1);
        const float f = pow2f(C::EMAX - WP::exp(j));
        qb[ks][h] = qb_ok ? pack_h2(__half2float(qrow[d0]) * f, __half2float(qrow[d1]) * f) : 0u;
      }
    }
  }
  const float qsA = (BITS != 16 && colA) ? qs_sm[2 * tig] : 0.f;
  const float qsB = (BITS != 16 && colB) ? qs_sm[2 * tig + 1] : 0.f;

  // ---- running state.  m_ref (per head slot) is a reference point at least
  // as large as every score seen, so p = 2^(x - m_ref) <= 1 and P' = p * s_V
  // stays within fp16 range; it moves (with a rescale) only when a stage's
  // max exceeds it, and then to that max + kLazy.
  float o_acc[NP][8][4];
#pragma unroll
  for (int nt = 0; nt < NP; ++nt)
#pragma unroll
    for (int i = 0; i < 8; ++i) o_acc[nt][i][0] = o_acc[nt][i][1] = o_acc[nt][i][2] = o_acc[nt][i][3] = 0.f;
  float corr[NP];  // sum of P' * z_V for B column nt * 8 + gid
#pragma unroll
  for (int nt = 0; nt < NP; ++nt) corr[nt] = 0.f;
  constexpr float kLazy = 4.0f;
  float m_ref[HS], l_part[HS];
#pragma unroll
  for (int s = 0; s < HS; ++s) {
    m_ref[s] = -INFINITY;
    l_part[s] = 0.f;
  }
  int failed_at = -1;
  const int st0 = st;
  const uint32_t phase0 = phase;

  auto stage_body = [&](auto full_tag, const uint8_t* sK, const uint8_t* sV, const uint8_t* sKm,
                        const uint8_t* sVm, int n_valid) {
    constexpr bool FULL = decltype(full_tag)::value;
    constexpr int NS = C::SUB;
    auto valid = [&](int tok) { return FULL || tok < n_valid; };  // tok: 0 .. STOK-1

    // ---- S^T = K * Qx^T per sub-tile: this lane's rows are tokens gid, gid + 8
    float x[NS][HS][2];
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
      float s_acc[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t k0[C::KW], k1[C::KW];
      load_chunk<C::KC, C::KW>(sK + (sub * kTile + gid) * C::RB + tig * C::KC, k0);
      load_chunk<C::KC, C::KW>(sK + (sub * kTile + gid + 8) * C::RB + tig * C::KC, k1);
      uint32_t p0[16], p1[16];
#pragma unroll
      for (int w = 0; w < C::KW; ++w) {
        uint32_t y0[WP::kPairs], y1[WP::kPairs];
        WP::run(k0[w], y0);
        WP::run(k1[w], y1);
#pragma unroll
        for (int j = 0; j < WP::kPairs; ++j) {
          p0[w * WP::kPairs + j] = y0[j];
          p1[w * WP::kPairs + j] = y1[j];
        }
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_f16(s_acc, p0[2 * ks], p1[2 * ks], p0[2 * ks + 1], p1[2 * ks + 1], qb[ks][0],
                qb[ks][1]);
      // score = sum over the head's group columns of s_K * (S - z_K * qs);
      // rows past the valid length may hold any bytes: masked below by select
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float v[HS];
        if constexpr (BITS == 16) {
          v[0] = s_acc[2 * r];
          if constexpr (HS == 2) v[1] = s_acc[2 * r + 1];
        } else {
          const uint8_t* m = sKm + (sub * kTile + gid + 8 * r) * C::MB + meta_off;
          if constexpr (NG == 1) {
            const float2 sz = __half22float2(*reinterpret_cast<const __half2*>(m));
            v[0] = colA ? sz.x * fmaf(-sz.y, qsA, s_acc[2 * r]) : 0.f;
            if constexpr (HS == 2) v[1] = colB ? sz.x * fmaf(-sz.y, qsB, s_acc[2 * r + 1]) : 0.f;
          } else {
            v[0] = 0.f;
            if (colA) {
              const uint2 u = *reinterpret_cast<const uint2*>(m);
              const float2 szA = __half22float2(u32_as_h2(u.x));
              const float2 szB = __half22float2(u32_as_h2(u.y));
              v[0] = fmaf(szB.x, fmaf(-szB.y, qsB, s_acc[2 * r + 1]),
                          szA.x * fmaf(-szA.y, qsA, s_acc[2 * r]));
            }
            if constexpr (NG == 4) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
          }
        }
        const bool ok = valid(sub * kTile + gid + 8 * r);
#pragma unroll
        for (int s = 0; s < HS; ++s) x[sub][s][r] = ok ? v[s] * score_scale : -INFINITY;
      }
    }

    // ---- online softmax per head slot: max over the stage's tokens (rows
    // gid and gid + 8 of every sub-tile, then across gid)
    bool any_rescale = false;
    float alpha[HS];
#pragma unroll
    for (int s = 0; s < HS; ++s) {
      float tmax = -INFINITY;
#pragma unroll
      for (int sub = 0; sub < NS; ++sub) tmax = fmaxf(tmax, fmaxf(x[sub][s][0], x[sub][s][1]));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
      alpha[s] = 1.f;
      if (tmax > m_ref[s]) {
        const float m_new = tmax + kLazy;
        if (m_ref[s] != -INFINITY) {
          alpha[s] = fast_exp2(m_ref[s] - m_new);
          any_rescale = true;
        }
        m_ref[s] = m_new;
      }
      l_part[s] *= alpha[s];
    }
    if (__any_sync(0xffffffffu, any_rescale)) {
      // the PV accumulators (columns of head ho) and corrections (B column
      // of head hb) take the factor of their head from its QK lane
#pragma unroll
      for (int nt = 0; nt < NP; ++nt) {
        const int src_o = 4 * gid + (ho[nt] < GR ? (ho[nt] * NG) / 2 : 0);
        const int src_b = 4 * gid + ts[nt];
        float ao = __shfl_sync(0xffffffffu, alpha[0], src_o);
        float ab = __shfl_sync(0xffffffffu, alpha[0], src_b);
        if constexpr (HS == 2) {
          const float ao1 = __shfl_sync(0xffffffffu, alpha[1], src_o);
          const float ab1 = __shfl_sync(0xffffffffu, alpha[1], src_b);
          ao = (ho[nt] & 1) ? ao1 : ao;
          ab = sl[nt] ? ab1 : ab;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) o_acc[nt][i][c] *= ao;
        corr[nt] *= ab;
      }
    }
    // p in the QK layout (0 for masked tokens)
#pragma unroll
    for (int sub = 0; sub < NS; ++sub)
#pragma unroll
      for (int s = 0; s < HS; ++s)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          x[sub][s][r] = fast_exp2(x[sub][s][r] - m_ref[s]);
          l_part[s] += x[sub][s][r];
        }

    // ---- O^T += V^T * P'^T per sub-tile
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
      // V (s, z) of this lane's four tokens for group gv
      [[maybe_unused]] float2 szv[4];
      if constexpr (BITS != 16) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          szv[k] = __half22float2(*reinterpret_cast<const __half2*>(
              sVm + (sub * kTile + vt[k]) * C::MB + gv * 4));
      }
      uint32_t b0[NP], b1[NP];
#pragma unroll
      for (int nt = 0; nt < NP; ++nt) {
        // p of head hb for tokens tig, tig + 4 (row 0 of QK lanes tig, tig + 4)
        // and tig + 8, tig + 12 (row 1)
        const int la = 4 * tig + ts[nt], lb = 4 * (tig + 4) + ts[nt];
        float pv[4];
        pv[0] = __shfl_sync(0xffffffffu, x[sub][0][0], la);
        pv[1] = __shfl_sync(0xffffffffu, x[sub][0][0], lb);
        pv[2] = __shfl_sync(0xffffffffu, x[sub][0][1], la);
        pv[3] = __shfl_sync(0xffffffffu, x[sub][0][1], lb);
        if constexpr (HS == 2) {
          const float q0 = __shfl_sync(0xffffffffu, x[sub][HS - 1][0], la);
          const float q1 = __shfl_sync(0xffffffffu, x[sub][HS - 1][0], lb);
          const float q2 = __shfl_sync(0xffffffffu, x[sub][HS - 1][1], la);
          const float q3 = __shfl_sync(0xffffffffu, x[sub][HS - 1][1], lb);
          if (sl[nt]) {
            pv[0] = q0; pv[1] = q1; pv[2] = q2; pv[3] = q3;
          }
        }
        float pp[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if constexpr (BITS == 16) {
            pp[k] = pv_ok[nt] ? pv[k] : 0.f;
          } else {
            // slots past the valid length may hold any bytes (NaN scales):
            // select, never multiply by a zero weight
            const bool ok = pv_ok[nt] && valid(sub * kTile + vt[k]);
            pp[k] = ok ? pv[k] * szv[k].x : 0.f;
            corr[nt] = ok ? fmaf(pp[k], szv[k].y, corr[nt]) : corr[nt];
          }
        }
        // hi part in even columns, lo = P' - hi in odd ones
        const float2 h01 = __half22float2(__floats2half2_rn(pp[0], pp[1]));
        const float2 h23 = __half22float2(__floats2half2_rn(pp[2], pp[3]));
        b0[nt] = pack_h2(fmaf(-lo_sel, h01.x, pp[0]), fmaf(-lo_sel, h01.y, pp[1]));
        b1[nt] = pack_h2(fmaf(-lo_sel, h23.x, pp[2]), fmaf(-lo_sel, h23.y, pp[3]));
      }

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
      for (int nt = 0; nt < NP; ++nt)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
          mma_f16(o_acc[nt][mt], xa[mt], xa[mt + 8], xc[mt], xc[mt + 8], b0[nt], b1[nt]);
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

  // ---- warp totals: l over the token rows (gid), corrections over tig
#pragma unroll
  for (int s = 0; s < HS; ++s) {
    l_part[s] += __shfl_xor_sync(0xffffffffu, l_part[s], 4);
    l_part[s] += __shfl_xor_sync(0xffffffffu, l_part[s], 8);
    l_part[s] += __shfl_xor_sync(0xffffffffu, l_part[s], 16);
  }
  float corr_t[NP];  // the correction of accumulator column nt * 8 + 2 tig
#pragma unroll
  for (int nt = 0; nt < NP; ++nt) {
    corr[nt] += __shfl_xor_sync(0xffffffffu, corr[nt], 1);
    corr[nt] += __shfl_xor_sync(0xffffffffu, corr[nt], 2);
    corr_t[nt] = __shfl_sync(0xffffffffu, corr[nt], 8 * tig);
  }

  __syncthreads();
  float* ms = reinterpret_cast<float*>(smem + C::HDR_BYTES);  // [kWarps][8]
  float* ls = ms + kWarps * 8;                                 // [kWarps][8]
  float* os = ls + kWarps * 8;                                 // [kWarps][8][D]
  if (gid == 0 && (NG != 4 || (tig & 1) == 0)) {
#pragma unroll
    for (int s = 0; s < HS; ++s) {
      const int h = slot_head(s);
      if (h < GR) {
        ms[warp * 8 + h] = m_ref[s];
        ls[warp * 8 + h] = l_part[s];
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NP; ++nt) {
    if (writer[nt]) {
      float* oh = os + (warp * 8 + ho[nt]) * D + 16 * gid;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        // undo the subnormal code scale 2^(e - 24) of the row's dim
        const float f0 = pow2f(24 - XP::exp(mt % XP::kOut));
        const float f1 = pow2f(24 - XP::exp((mt + 8) % XP::kOut));
        oh[mt] = fmaf(o_acc[nt][mt][0] + o_acc[nt][mt][1], f0, -corr_t[nt]);
        oh[mt + 8] = fmaf(o_acc[nt][mt][2] + o_acc[nt][mt][3], f1, -corr_t[nt]);
      }
    }
  }
  __syncthreads();
  cta_merge_store<GR>(a, ms, ls, os, os + kWarps * 8 * D, b, kvh, seg.part_base + split, t);
  }  // unit loop

  if (t == 0) release_counters(counters);
}

template <int BITS, int GE, int GR>
cudaError_t launch_tm(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  using C = TmCfg<BITS, GE, GR>;
  // the shared-memory opt-in is a per-device function attribute: set it once
  // per device (bit i of the mask = device i)
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(decode_tm_kernel<BITS, GE, GR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  SplitParams P{a, seg};
  const long long units = (long long)seg.n_split * a.kv_heads * a.batch;
  const long long slots = 148LL * C::MIN_CTAS;  // one wave of persistent CTAs
  const unsigned grid = (unsigned)(units < slots ? units : slots);
  decode_tm_kernel<BITS, GE, GR><<<grid, kWarps * 32, C::SMEM, s>>>(P);
  return cudaGetLastError();
}

// Every (bits, G, g) with NG * g <= 8 that the cache formats allow.
#define KVQ_TM_FORMATS(X)                                              \
  X(16, 128, 1) X(16, 128, 2) X(16, 128, 4) X(16, 128, 8)              \
  X(8, 128, 1) X(8, 128, 2) X(8, 128, 4) X(8, 128, 8)                  \
  X(4, 128, 1) X(4, 128, 2) X(4, 128, 4) X(4, 128, 8)                  \
  X(2, 128, 1) X(2, 128, 2) X(2, 128, 4) X(2, 128, 8)                  \
  X(8, 64, 1) X(8, 64, 2) X(8, 64, 4)                                  \
  X(4, 64, 1) X(4, 64, 2) X(4, 64, 4)                                  \
  X(2, 64, 1) X(2, 64, 2) X(2, 64, 4)                                  \
  X(8, 32, 1) X(8, 32, 2) X(4, 32, 1) X(4, 32, 2) X(2, 32, 1) X(2, 32, 2)

}  // namespace

bool decode_tm_supported(int bits, int group, int group_ratio) {
#define KVQ_X(B, G_, R) \
  if (bits == B && group == G_ && group_ratio == R) return true;
  KVQ_TM_FORMATS(KVQ_X)
#undef KVQ_X
  return false;
}

int decode_tm_ctas_per_sm(int bits, int group, int group_ratio) {
#define KVQ_X(B, G_, R) \
  if (bits == B && group == G_ && group_ratio == R) return TmCfg<B, G_, R>::MIN_CTAS;
  KVQ_TM_FORMATS(KVQ_X)
#undef KVQ_X
  return 0;
}

cudaError_t launch_decode_tm(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  const int bits = seg.bits, group = (seg.bits == 16) ? kHeadDim : seg.group;
  const int g = a.group_ratio;
#define KVQ_X(B, G_, R) \
  if (bits == B && group == G_ && g == R) return launch_tm<B, G_, R>(a, seg, s);
  KVQ_TM_FORMATS(KVQ_X)
#undef KVQ_X
  return cudaErrorInvalidValue;
}

}  // namespace kvq
