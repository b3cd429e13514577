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

#include <atomic>
#include <type_traits>

#include "kvq_decode_common.cuh"
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
  // CTAs kept on one SM: four for the 2- and 4-bit formats (the query
  // fragments live in shared memory, not registers), three otherwise
  static constexpr int MIN_CTAS = 3;
  // 16-token sub-tiles per stage: two side by side, except where the
  // registers of two would not fit (fp16 rows, 4 groups)
  static constexpr int SUB = (BITS == 16 || NG == 4) ? 1 : 2;
  static constexpr int STOK = SUB * kTile;                   // tokens per stage
  static constexpr int STAGE = 2 * STOK * RB + 2 * STOK * MB;
  static constexpr int MF_FLOATS = 2 * STOK * NG * 2;        // fp32 (s, z) of a stage
  // header: mbarriers (<= 512 B), q rows as fp16 (<= 8 x 128), group sums,
  // the A fragments of all 32 lane positions (8 x 32 x 16 B)
  static constexpr int HDR_BARS = 0, HDR_Q = 512, HDR_QS = 512 + 8 * kHeadDim * 2;
  static constexpr int HDR_QF = HDR_QS + 128;
  static constexpr int HDR_MF = HDR_QF + 8 * 32 * 16;        // per-warp fp32 meta
  static constexpr int HDR_MISC = HDR_MF + kWarps * MF_FLOATS * 4;  // unit id, fail flag
  static constexpr int HDR_BYTES = HDR_MISC + 128;
  // as many stages as fit in a budget that keeps MIN_CTAS CTAs on an SM
  // (3 x (74 KB + 1 KB reserved) and 4 x (56 KB + 1 KB) <= 228 KB)
  static constexpr int SMEM_BUDGET = (MIN_CTAS == 4 ? 56 : 74) * 1024;
  static constexpr int STAGES_RAW = (SMEM_BUDGET - HDR_BYTES) / (kWarps * STAGE);
  static constexpr int STAGES = STAGES_RAW < 2 ? 2 : (STAGES_RAW > 16 ? 16 : STAGES_RAW);
  static constexpr int SMEM = HDR_BYTES + kWarps * STAGES * STAGE;
  static constexpr int CROSS = (BITS == 16) ? 2 : (BITS == 8 ? 4 : (BITS == 4 ? 8 : 16));
  static constexpr int PER_W = (NTG < CROSS) ? NTG : CROSS;  // V n-tiles per word
  static constexpr int EMAX = WordPairs<BITS>::kEmax;
};

// Token order inside an 8-token n-tile: MMA column n reads token row
// rho(n) = n ^ ((n >> 1) & 1) = 0 1 3 2 4 5 7 6.  Softmax and attention do
// not depend on token order; this order keeps the 16-byte K loads free of
// shared-memory bank conflicts and halves those of the V loads (the four
// rows a V load instruction touches alternate between the two 64-byte
// halves of a bank window).
__device__ __forceinline__ int rho(int n) { return n ^ ((n >> 1) & 1); }

template <int BITS, int GE, int GR>
__global__ void __launch_bounds__(kWarps * 32, Cfg<BITS, GE>::MIN_CTAS)
decode_split_kernel(const __grid_constant__ SplitParams P) {
  using C = Cfg<BITS, GE>;
  using WP = WordPairs<BITS>;
  using XP = CrossPairs<BITS>;
  constexpr int D = C::D;
  const DecodeArgs& a = P.a;
  const SegView& seg = P.seg;

  extern __shared__ __align__(128) uint8_t smem[];
  grid_dependents_may_launch();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  constexpr int g = GR;                  // query heads per KV head: 1, 2, 4 or 8
  constexpr int lg = GR == 1 ? 0 : (GR == 2 ? 1 : (GR == 4 ? 2 : 3));
  constexpr int R = C::NG * g;           // valid MMA rows (group, head)
  static_assert(R <= 16, "at most 16 (group, head) rows");

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::HDR_BARS) + warp * C::STAGES;
  __half* q_sm = reinterpret_cast<__half*>(smem + C::HDR_Q);      // [g][D]
  float* qs_sm = reinterpret_cast<float*>(smem + C::HDR_QS);      // [R]
  uint4* qf_sm = reinterpret_cast<uint4*>(smem + C::HDR_QF);      // [8][32 lanes]
  float2* mf = reinterpret_cast<float2*>(smem + C::HDR_MF) + warp * (C::MF_FLOATS / 2);
  uint8_t* stages = smem + C::HDR_BYTES + warp * C::STAGES * C::STAGE;
  int* unit_sm = reinterpret_cast<int*>(smem + C::HDR_MISC);
  int* fail_sm = unit_sm + 1;
  int* qexp_sm = unit_sm + 8;  // [8] power-of-two shift of each staged query row
  uint32_t* counters = a.err + seg.ctr;  // [0] next unit, [1] CTAs done

  const uint64_t policy = l2_evict_first_policy();
  // the stage ring (position and mbarrier phase) runs on across units
  int st = 0;
  uint32_t phase = 0;
  if (lane == 0) {
    for (int s2 = 0; s2 < C::STAGES; ++s2) mbar_init(&bars[s2], 1);
    fence_barrier_init();
  }
  if (threadIdx.x == 0) *fail_sm = 0;
  __syncwarp();
  const int t = threadIdx.x;
  const int units = seg.n_split * a.kv_heads * a.batch;

  // Persistent CTA: take (sequence, KV head, split) units from a counter in
  // the workspace until none is left.  The barrier after the fetch also
  // orders the previous unit's reads of the merge scratch before this
  // unit's copies into the stage buffers.
  for (;;) {
  if (t == 0) *unit_sm = (int)atomicAdd(&counters[0], 1u);
  __syncthreads();
  const int unit = *unit_sm;
  if (unit >= units || *fail_sm) break;
  const int split = unit % seg.n_split;
  const int kvh = (unit / seg.n_split) % a.kv_heads;
  const int b = unit / (seg.n_split * a.kv_heads);

  // ---- token range of this warp (a multiple of the stage size, so a
  // stage's copy never runs past round_up(seq_len, 32) <= max_tokens)
  int L = seg.seq_lens[b];
  L = max(0, min(L, seg.max_tokens));
  // a unit is a whole number of 32-token stages; its stages go to the four
  // warps round-robin: warp w takes stages w, w + 4, ...
  int c0, c1;
  split_range(L, seg.n_split, split, c0, c1);
  const int unit_stages = (c1 > c0) ? (c1 - c0 + C::STOK - 1) / C::STOK : 0;
  const int n_tiles = (unit_stages > warp) ? (unit_stages - warp + kWarps - 1) / kWarps : 0;
  const int w0 = c0 + warp * C::STOK;  // first token of this warp's first stage

  const uint8_t* kc_src = seg.k_codes + (((long long)b * a.kv_heads + kvh) * seg.max_tokens + w0) * C::RB;
  const uint8_t* vc_src = seg.v_codes + (((long long)b * a.kv_heads + kvh) * seg.max_tokens + w0) * C::RB;
  const uint8_t* km_src = seg.k_meta + (((long long)b * a.kv_heads + kvh) * seg.max_tokens + w0) * C::MB;
  const uint8_t* vm_src = seg.v_meta + (((long long)b * a.kv_heads + kvh) * seg.max_tokens + w0) * C::MB;
  // copy tile `i` into stage `st` (lane 0 only)
  auto issue = [&](int i, int st) {
    uint8_t* dst = stages + st * C::STAGE;
    mbar_arrive_expect_tx(&bars[st], C::STAGE);
    const size_t tok = (size_t)i * (kWarps * C::STOK);  // stage i of this warp
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

  // ---- the g query rows of this KV head, once per unit, as fp16 in smem
  stage_queries<g, C::EMAX - WP::exp(0)>(a, b, kvh, q_sm, qexp_sm, t);
  __syncthreads();
  // sum of q over each (group, head) row, in the MMA's units (the QK MMA
  // returns 2^(EMAX - 24) * sum(q * c))
  if constexpr (BITS != 16) {
    const int r = t >> 3, part = t & 7;
    float acc = 0.f;
    if (r < R) {
      const __half* qr = q_sm + (r & (g - 1)) * D + (r >> lg) * GE + part * (GE / 8);
#pragma unroll 4
      for (int i = 0; i < GE / 8; ++i) acc += __half2float(qr[i]);
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (r < R && part == 0) qs_sm[r] = acc * pow2f(C::EMAX - 24);
  }
  // A fragments, built once per CTA for every lane position: row r =
  // gr * g + h holds q_h masked to group gr, each element scaled by
  // 2^(EMAX - e) for the subnormal exponent e of the code it meets.
  // Thread t builds 8 of the 32 registers of lane position t / 4.
  {
    const int fl = t >> 2;                 // lane position
    const int fg = fl >> 2, ft = fl & 3;   // its gid, tig
    auto qx = [&](int r, int d, int e) -> float {
      if (r >= R || d / GE != (r >> lg)) return 0.0f;
      return __half2float(q_sm[(r & (g - 1)) * D + d]) * pow2f(C::EMAX - e);
    };
    auto kdim = [&](int pidx, int e) -> int {
      return 32 * ft + (pidx / WP::kPairs) * WP::kDims + WP::dim(pidx % WP::kPairs, e);
    };
#pragma unroll
    for (int u = 0; u < 2; ++u) {          // this thread: k-steps 2 * (t & 3) + u
      const int ks = 2 * (t & 3) + u;
      const int pA = 2 * ks, pB = 2 * ks + 1;
      const int eA = WP::exp(pA % WP::kPairs), eB = WP::exp(pB % WP::kPairs);
      uint4 v;
      v.x = pack_h2(qx(fg, kdim(pA, 0), eA), qx(fg, kdim(pA, 1), eA));
      v.y = pack_h2(qx(fg + 8, kdim(pA, 0), eA), qx(fg + 8, kdim(pA, 1), eA));
      v.z = pack_h2(qx(fg, kdim(pB, 0), eB), qx(fg, kdim(pB, 1), eB));
      v.w = pack_h2(qx(fg + 8, kdim(pB, 0), eB), qx(fg + 8, kdim(pB, 1), eB));
      qf_sm[ks * 32 + fl] = v;
    }
  }
  __syncthreads();
  // query fragments: kept in registers for the 3-CTA formats, re-read from
  // shared memory (once per stage and k-step) for the 4-CTA ones
  constexpr bool kQfRegs = C::MIN_CTAS == 3;
  uint32_t qf[kQfRegs ? 8 : 1][4];
  if constexpr (kQfRegs) {
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint4 v = qf_sm[ks * 32 + lane];
      qf[ks][0] = v.x; qf[ks][1] = v.y; qf[ks][2] = v.z; qf[ks][3] = v.w;
    }
  }
  const bool row0_ok = gid < R, row1_ok = gid + 8 < R;
  const float qs0 = (BITS != 16 && row0_ok) ? qs_sm[gid] : 0.f;
  const float qs1 = (BITS != 16 && row1_ok) ? qs_sm[gid + 8] : 0.f;
  const int gr0 = row0_ok ? (gid >> lg) : 0;
  const int gr1 = row1_ok ? ((gid + 8) >> lg) : 0;
  const bool head_ok = gid < g;  // this lane's PV rows are a real head
  // log2-domain softmax scale including the MMA's 2^(24 - EMAX), and the
  // query row's shift: every score of this lane is head gid % g's
  const float score_scale = a.scale_log2 * pow2f(24 - C::EMAX) * unshift(qexp_sm[gid & (g - 1)]);
  // this lane's token rows within a tile: MMA columns 2*tig, 2*tig+1 of the
  // two n-tiles, in the rho order
  const int tokA = rho(2 * tig), tokB = rho(2 * tig + 1);
  const int tokC = 8 + tokA, tokD = 8 + tokB;
  const int tok4[4] = {tokA, tokB, tokC, tokD};
  const int krow = rho(gid);  // K row this lane feeds into MMA column gid

  // ---- running state (head = gid)
  float o_acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float corr[C::NG];
#pragma unroll
  for (int i = 0; i < C::NG; ++i) corr[i] = 0.f;
  // m_run is a reference point at least as large as every score seen, so
  // p = 2^(x - m_run) <= 1 and P' = p * s_V stays within fp16 range; it
  // moves (with a rescale) only when a stage's max exceeds it, and then to
  // that max + kLazy
  constexpr float kLazy = 4.0f;
  float m_run = -INFINITY, l_part = 0.f;
  int failed_at = -1;
  const int st0 = st;
  const uint32_t phase0 = phase;

  // One stage (SUB sub-tiles of 16 tokens): QK^T of every sub-tile, one
  // online-softmax update, then PV of every sub-tile.  Working on the
  // sub-tiles side by side gives the scheduler independent MMA chains and
  // conversions to interleave.  FULL = all STOK tokens valid (no masking).
  auto stage_body = [&](auto full_tag, const uint8_t* sK, const uint8_t* sV, const uint8_t* sKm,
                        const uint8_t* sVm, int n_valid) {
    constexpr bool FULL = decltype(full_tag)::value;
    constexpr int NS = C::SUB;
    auto valid = [&](int tok) { return FULL || tok < n_valid; };  // tok: 0 .. STOK-1

    // (s, z) of the stage's K and V rows to fp32, once per warp: each lane
    // converts SUB * NG pairs, every lane then reads the ones it needs
    if constexpr (BITS != 16) {
      __syncwarp();
#pragma unroll
      for (int j = 0; j < NS * C::NG; ++j) {
        const int idx = lane * (NS * C::NG) + j;  // 0 .. 2 * STOK * NG - 1
        const int plane = idx >= C::STOK * C::NG;
        const __half2* src = reinterpret_cast<const __half2*>(plane ? sVm : sKm);
        mf[idx] = __half22float2(src[idx - plane * C::STOK * C::NG]);
      }
      __syncwarp();
    }

    // ---- S = Qx * K^T for every 8-token n-tile of the stage
    float s_acc[NS][2][4];
    if constexpr (kQfRegs) {
#pragma unroll
      for (int sub = 0; sub < NS; ++sub) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          s_acc[sub][nt][0] = s_acc[sub][nt][1] = s_acc[sub][nt][2] = s_acc[sub][nt][3] = 0.f;
          uint32_t kw[C::KW];
          load_chunk<C::KC, C::KW>(sK + ((sub * 2 + nt) * 8 + krow) * C::RB + tig * C::KC, kw);
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
            mma_f16(s_acc[sub][nt], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], pr[2 * ks],
                    pr[2 * ks + 1]);
        }
      }
    } else {
      // k-step outermost: one shared-memory read of each query fragment
      // feeds the MMAs of all n-tiles of the stage
      uint32_t kw[NS][2][C::KW];
#pragma unroll
      for (int sub = 0; sub < NS; ++sub)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          s_acc[sub][nt][0] = s_acc[sub][nt][1] = s_acc[sub][nt][2] = s_acc[sub][nt][3] = 0.f;
          load_chunk<C::KC, C::KW>(sK + ((sub * 2 + nt) * 8 + krow) * C::RB + tig * C::KC,
                                   kw[sub][nt]);
        }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint4 q4 = qf_sm[ks * 32 + lane];
        constexpr int P = WP::kPairs;
#pragma unroll
        for (int sub = 0; sub < NS; ++sub)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = WP::one(kw[sub][nt][(2 * ks) / P], (2 * ks) % P);
            const uint32_t b1 = WP::one(kw[sub][nt][(2 * ks + 1) / P], (2 * ks + 1) % P);
            mma_f16(s_acc[sub][nt], q4.x, q4.y, q4.z, q4.w, b0, b1);
          }
      }
    }

    // ---- scores of head (gid mod g) for this lane's tokens.  Rows past R
    // hold zero queries (S = 0, qs = 0), so they add nothing.
    float sc[NS][4];
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int nt = k >> 1, e = k & 1;
        const float S0 = s_acc[sub][nt][e];
        if constexpr (BITS == 16) {
          sc[sub][k] = S0;
        } else {
          const float S1 = s_acc[sub][nt][2 + e];
          const float2* m = mf + (sub * kTile + tok4[k]) * C::NG;
          const float2 sz0 = m[gr0];
          const float2 sz1 = m[gr1];
          sc[sub][k] = fmaf(sz1.x, fmaf(-sz1.y, qs1, S1), sz0.x * fmaf(-sz0.y, qs0, S0));
        }
      }
    }
    // sum the group rows of each head: lanes gid and gid ^ m (m >= g)
#pragma unroll
    for (int m = 1; m < 8; m <<= 1) {
      if (m >= g) {
#pragma unroll
        for (int sub = 0; sub < NS; ++sub)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            sc[sub][k] += __shfl_xor_sync(0xffffffffu, sc[sub][k], 4 * m);
      }
    }
    float tmax = -INFINITY;
#pragma unroll
    for (int sub = 0; sub < NS; ++sub)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        sc[sub][k] = valid(sub * kTile + tok4[k]) ? sc[sub][k] * score_scale : -INFINITY;
        tmax = fmaxf(tmax, sc[sub][k]);
      }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    if (tmax > m_run) {
      const float m_new = tmax + kLazy;
      if (m_run != -INFINITY) {  // nothing accumulated yet: no rescale needed
        const float alpha = fast_exp2(m_run - m_new);
#pragma unroll
        for (int n = 0; n < 16; ++n)
#pragma unroll
          for (int c = 0; c < 4; ++c) o_acc[n][c] *= alpha;
#pragma unroll
        for (int gr = 0; gr < C::NG; ++gr) corr[gr] *= alpha;
        l_part *= alpha;
      }
      m_run = m_new;
    }
    float p[NS][4];
#pragma unroll
    for (int sub = 0; sub < NS; ++sub)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        p[sub][k] = head_ok ? fast_exp2(sc[sub][k] - m_run) : 0.f;  // 0 for masked tokens
        l_part += p[sub][k];
      }

    // ---- O += P' * V per group and sub-tile (hi rows gid, lo rows gid + 8)
#pragma unroll
    for (int gr = 0; gr < C::NG; ++gr) {
#pragma unroll
      for (int sub = 0; sub < NS; ++sub) {
        float pp[4];
        if constexpr (BITS == 16) {
#pragma unroll
          for (int k = 0; k < 4; ++k) pp[k] = p[sub][k];
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            // slots past the valid length may hold any bytes (NaN scales):
            // select, never multiply by a zero weight
            const bool ok = valid(sub * kTile + tok4[k]);
            const float2 sz = mf[(C::STOK + sub * kTile + tok4[k]) * C::NG + gr];
            pp[k] = ok ? p[sub][k] * sz.x : 0.f;
            corr[gr] = ok ? fmaf(pp[k], sz.y, corr[gr]) : corr[gr];
          }
        }
        const __half2 h01 = __floats2half2_rn(pp[0], pp[1]);
        const __half2 h23 = __floats2half2_rn(pp[2], pp[3]);
        const float2 f01 = __half22float2(h01);
        const float2 f23 = __half22float2(h23);
        const uint32_t a0 = h2_as_u32(h01);
        const uint32_t a1 = pack_h2(pp[0] - f01.x, pp[1] - f01.y);
        const uint32_t a2 = h2_as_u32(h23);
        const uint32_t a3 = pack_h2(pp[2] - f23.x, pp[3] - f23.y);

        const uint8_t* vbase = sV + sub * kTile * C::RB + gr * (GE * BITS / 8) + gid * C::VC;
        uint32_t wA[C::VW], wB[C::VW], wC[C::VW], wD[C::VW];
        load_chunk<C::VC, C::VW>(vbase + tokA * C::RB, wA);
        load_chunk<C::VC, C::VW>(vbase + tokB * C::RB, wB);
        load_chunk<C::VC, C::VW>(vbase + tokC * C::RB, wC);
        load_chunk<C::VC, C::VW>(vbase + tokD * C::RB, wD);
        if constexpr (BITS == 16 && !FULL) {
          // raw fp16 rows past the valid length may hold anything: zero them
#pragma unroll
          for (int w = 0; w < C::VW; ++w) {
            wA[w] = valid(sub * kTile + tokA) ? wA[w] : 0u;
            wB[w] = valid(sub * kTile + tokB) ? wB[w] : 0u;
            wC[w] = valid(sub * kTile + tokC) ? wC[w] : 0u;
            wD[w] = valid(sub * kTile + tokD) ? wD[w] : 0u;
          }
        }
#pragma unroll
        for (int w = 0; w < C::VW; ++w) {
          uint32_t x[C::CROSS], y[C::CROSS];
          XP::run(wA[w], wB[w], x);
          XP::run(wC[w], wD[w], y);
#pragma unroll
          for (int j = 0; j < C::PER_W; ++j)
            mma_f16(o_acc[gr * C::NTG + w * C::PER_W + j], a0, a1, a2, a3, x[j], y[j]);
        }
      }
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
  float* ms = reinterpret_cast<float*>(smem + C::HDR_BYTES);  // [kWarps][8]
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
      // undo the subnormal code scale 2^(e - 24) of this column
      const float f = pow2f(24 - XP::exp(jj));
      oh[d0] = fmaf(o_acc[nt][0] + o_acc[nt][2], f, -corr[gr]);
      oh[d1] = fmaf(o_acc[nt][1] + o_acc[nt][3], f, -corr[gr]);
    }
  }
  __syncthreads();
  cta_merge_store<g>(a, ms, ls, os, os + kWarps * 8 * D, b, kvh, seg.part_base + split, t);
  // the merge wrote the stage buffers: order that before the next unit's copies
  fence_proxy_async_smem();
  }  // unit loop

  if (t == 0) release_counters(counters);
  grid_dependency_wait();  // after the previous segment's kernel (see decode_tm_kernel)
}

// Merge the partial (m, l, o) of every split and segment (log-sum-exp).
// One CTA of 128 x PG threads per (sequence, query head): all threads
// reduce the max and the weights over the partials together; thread
// (group j, dim d) then sums dim d over the partials j, j + PG, j + 2 PG, ...
// eight loads in flight at a time, and group 0 adds the groups' sums.  At
// 512 threads of 32 registers a CTA still fits on an SM beside three CTAs
// of the split kernel, so it can be resident before they end (a
// 1024-thread CTA cannot, and measured slower).  It is launched as a programmatic dependent of the split-K
// kernels: the launch overlaps their tail, and griddepcontrol.wait holds
// every thread until they have completed and their stores are visible.
template <int PG>
__global__ void __launch_bounds__(kHeadDim * PG) decode_merge_kernel(const DecodeArgs a) {
  extern __shared__ float w_sm[];  // [parts] weights 2^(m_p - M), then [PG][D] sums
  __shared__ float red[4 * PG];
  grid_dependency_wait();
  constexpr int NT = kHeadDim * PG, NW = NT / 32;
  const long long bh = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int d = t % kHeadDim, grp = t / kHeadDim;
  const int P = a.parts;
  const float* ml = a.part_ml + bh * P * 2;
  const float* po = a.part_o + bh * P * kHeadDim;
  float m = -INFINITY;
  for (int p = t; p < P; p += NT)
    if (ml[2 * p + 1] > 0.f) m = fmaxf(m, ml[2 * p]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float M = red[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  float l = 0.f;
  for (int p = t; p < P; p += NT) {
    const float lp = ml[2 * p + 1];
    const float w = (lp > 0.f && M != -INFINITY) ? exp2f(ml[2 * p] - M) : 0.f;
    w_sm[p] = w;
    l += w * lp;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) L += red[w];
  // every partial's o is finite (a split with no tokens stores 0), so a
  // weight of 0 contributes exactly nothing; the loads stay independent of
  // the weights
  // the thread's partials grp, grp + PG, ... eight at a time, all eight
  // loads issued before the first is used
  float O = 0.f;
  for (int p0 = grp; p0 < P; p0 += 8 * PG) {
    float v[8], wv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int p = p0 + j * PG;
      v[j] = p < P ? po[(long long)p * kHeadDim + d] : 0.f;
      wv[j] = p < P ? w_sm[p] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) O = fmaf(wv[j], v[j], O);
  }
  if constexpr (PG > 1) {
    float* osm = w_sm + P;
    osm[grp * kHeadDim + d] = O;
    __syncthreads();
    if (grp != 0) return;
#pragma unroll
    for (int j = 1; j < PG; ++j) O += osm[j * kHeadDim + d];
  }
  a.out[bh * kHeadDim + d] = (L > 0.f) ? O / L : 0.f;
  if (a.lse != nullptr && t == 0)
    a.lse[bh] = (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

template <int BITS, int GE, int GR>
cudaError_t launch_split_g(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  using C = Cfg<BITS, GE>;
  // the shared-memory opt-in is a per-device function attribute: set it once
  // per device (bit i of the mask = device i)
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<BITS, GE, GR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  SplitParams P{a, seg};
  const long long units = (long long)seg.n_split * a.kv_heads * a.batch;
  const long long slots = (long long)seg.sms * C::MIN_CTAS;  // one wave of persistent CTAs
  const unsigned grid = (unsigned)(units < slots ? units : slots);
  return launch_segment_kernel(decode_split_kernel<BITS, GE, GR>, grid, kWarps * 32, C::SMEM, s,
                               seg.after_prev != 0, P);
}

}  // namespace

bool decode_supported(int bits, int group, int group_ratio, bool kpc) {
  if (kpc || bits == kE4M3 || bits == kE5M2 || bits == kSym8 || bits == kOaken)
    return decode_tm_supported(bits, group, group_ratio, kpc);
  if (!(group_ratio == 1 || group_ratio == 2 || group_ratio == 4 || group_ratio == 8))
    return false;
  if (bits == 16) return true;
  if (!(bits == 2 || bits == 4 || bits == 8)) return false;
  if (!(group == 32 || group == 64 || group == 128)) return false;
  return (kHeadDim / group) * group_ratio <= 16;
}

int decode_ctas_per_sm(int bits, int group, int group_ratio, bool kpc) {
  if (decode_tm_supported(bits, group, group_ratio, kpc))
    return decode_tm_ctas_per_sm(bits, group, group_ratio, kpc);
  return Cfg<4, 64>::MIN_CTAS;  // the same for every format
}

cudaError_t launch_decode_segment(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  const int bits = seg.bits, group = (seg.bits == 16) ? kHeadDim : seg.group;
  // (group, head) columns that fit one 8-wide tile: tokens-on-M kernel
  if (decode_tm_supported(bits, group, a.group_ratio, seg.k_channels))
    return launch_decode_tm(a, seg, s);
  if (seg.k_channels) return cudaErrorInvalidValue;
  // 16 (group, head) rows: this file's kernel
#define KVQ_D(B, G_, R) \
  if (bits == B && group == G_ && a.group_ratio == R) return launch_split_g<B, G_, R>(a, seg, s);
  KVQ_D(8, 64, 8) KVQ_D(4, 64, 8) KVQ_D(2, 64, 8)
  KVQ_D(8, 32, 4) KVQ_D(4, 32, 4) KVQ_D(2, 32, 4)
#undef KVQ_D
  return cudaErrorInvalidValue;
}

// The merge for up to kSmallParts partials: one thread per output dim
// issues every load it needs at once -- all (m, l) pairs of its head (the
// same for the head's threads) and its dim of every partial's o -- and
// reduces in registers: a single round trip to L2, no barrier.
constexpr int kSmallParts = 16;

__global__ void __launch_bounds__(kHeadDim) decode_merge_small_kernel(const DecodeArgs a) {
  grid_dependency_wait();
  const long long bh = blockIdx.x;
  const int d = threadIdx.x;
  const int P = a.parts;
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + bh * P;
  const float* po = a.part_o + bh * P * kHeadDim + d;
  float2 v[kSmallParts];
  float x[kSmallParts];
#pragma unroll
  for (int p = 0; p < kSmallParts; ++p) {
    v[p] = p < P ? ml[p] : make_float2(-INFINITY, 0.f);
    x[p] = p < P ? po[(long long)p * kHeadDim] : 0.f;
  }
  float M = -INFINITY;
#pragma unroll
  for (int p = 0; p < kSmallParts; ++p)
    if (v[p].y > 0.f) M = fmaxf(M, v[p].x);
  float L = 0.f, O = 0.f;
#pragma unroll
  for (int p = 0; p < kSmallParts; ++p) {
    // a partial with no tokens (l = 0, o = 0) weighs 0
    const float w = (v[p].y > 0.f) ? exp2f(v[p].x - M) : 0.f;
    L = fmaf(w, v[p].y, L);
    O = fmaf(w, x[p], O);
  }
  a.out[bh * kHeadDim + d] = (L > 0.f) ? O / L : 0.f;
  if (a.lse != nullptr && d == 0)
    a.lse[bh] = (L > 0.f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

cudaError_t launch_merge_small(const DecodeArgs& a, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)a.batch * a.q_heads));
  cfg.blockDim = dim3(kHeadDim);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_merge_small_kernel, a);
}

template <int PG>
cudaError_t launch_merge_pg(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = ((size_t)a.parts + (PG > 1 ? PG * kHeadDim : 0)) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(decode_merge_kernel<PG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((long long)a.batch * a.q_heads));
  cfg.blockDim = dim3(kHeadDim * PG);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel<PG>, a);
}

cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t s) {
  // more partials: more thread groups, so that each thread's chain of
  // dependent loads stays short
  if (a.parts >= 48) return launch_merge_pg<4>(a, s);
  if (a.parts > kSmallParts) return launch_merge_pg<2>(a, s);
  return launch_merge_small(a, s);
}

}  // namespace kvq
