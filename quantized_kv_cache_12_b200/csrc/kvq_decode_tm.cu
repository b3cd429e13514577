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
// Lane roles (gid = lane / 4, tig = lane % 4), per 16-token sub-tile.  A
// sub-tile's MMA rows r = 0 .. 15 are its tokens perm(r) = r ^ ((r >> 2) & 1)
// (an order that keeps the shared-memory loads below free of bank
// conflicts for the 2- and 4-bit formats).
//   QK: A rows gid, gid + 8; the lane's k elements are its 32-dim chunk
//       [32 tig, 32 tig + 32) of those two tokens.  B column c holds query
//       head (c / CPH) mod g masked to group c mod NG, where CPH (columns per
//       head) is chosen so that the two accumulator columns 2 tig, 2 tig + 1
//       of a lane give it whole heads: the scores of heads 2 tig and 2 tig + 1
//       (g = 8, NG = 1), or of one head, complete (NG <= 2) or in two halves
//       added by one shuffle (NG = 4).  Unused columns repeat a head.  The
//       online softmax and the weights P' = p * s_V (split into an fp16 high
//       part and the negated fp16 remainder) are computed here, per owned
//       head, for the lane's two tokens.
//   PV: the weights go to the B operand by 8x8 transposes (movmatrix): B
//       column 2 tig + part of n-tile b is (head, V group) combination (b, tig)
//       of QK lane tig, so the accumulator columns 2 tig, 2 tig + 1 of a PV
//       lane belong to the same lane position that owns their head: rescale
//       factors and zero-point corrections never cross lanes.  A rows gid,
//       gid + 8 of m-tile mt are dims 16 gid + mt and 16 gid + mt + 8; the k
//       positions 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 are rows 2 tig, 2 tig + 1,
//       2 tig + 8, 2 tig + 9 of the sub-tile, whose V codes the lane converts.
#include <cuda_runtime.h>
#include <math.h>

#include <atomic>
#include <type_traits>

#include "kvq_decode_common.cuh"
#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant_core.cuh"

namespace kvq {

namespace {

template <int BITS, int GE, int GR, bool KPC = false>
struct TmCfg {
  static constexpr int D = kHeadDim;
  // the Oaken codec: 4-bit dense codes with one (s, z) per plane, and a
  // row's outlier slots in place of per-token (s, z) pairs
  static constexpr bool OAK = BITS == kOaken;
  static constexpr int NG = D / GE;                    // V groups per token (and K's, per token)
  static constexpr int RB = D * code_bits(BITS) / 8;   // code bytes per token
  static constexpr int MB =                            // (s, z) (or slot) bytes per token
      (BITS == 16) ? 0 : (OAK ? KVQ_OAKEN_SLOTS * 2 : NG * 4);
  // K meta bytes per token: per-channel K (KPC) stores D (s, z) pairs per
  // block of kChannelBlock tokens, i.e. 16 bytes per token, and a stage is
  // one block
  static constexpr int MBK = KPC ? D * 4 / kChannelBlock : MB;
  static constexpr int KC = RB / 4;                    // K bytes of a lane (32 dims)
  static constexpr int KW = KC / 4;
  static constexpr int VB = RB / 8;                    // V bytes of a lane (16 dims)
  static constexpr int VW = VB / 4;
  // QK columns per head (see the file comment), head slots of a QK lane,
  // PV n-tiles, and lane positions whose (head, V group) combinations are
  // distinct
  static constexpr int CPH = (NG == 1 && GR == 8) ? 1 : ((NG == 4 || (NG == 2 && GR <= 2)) ? 4 : 2);
  static constexpr int HS = CPH == 1 ? 2 : 1;
  static constexpr int NP = (NG * GR + 3) / 4;
  static constexpr int W = NG * GR < 4 ? NG * GR : 4;
  // grouped PV (two groups, four heads): the m-tiles are split between the
  // groups, and each multiplies only its own group's weights; a lane then
  // reads CH = G / 8 contiguous dims of each group
  static constexpr bool GPV = NG == 2 && GR == 4;
  static constexpr int NO = GPV ? 1 : NP;              // accumulator n-tiles
  static constexpr int SUB = (BITS == 16) ? 1 : 2;     // 16-token sub-tiles per stage
  static constexpr int STOK = SUB * kTile;
  static constexpr int STAGE = 2 * STOK * RB + STOK * (MBK + MB);
  // header: mbarriers (<= 512 B), the g query rows as fp16, the column sums
  // of q, unit id and fail flag
  static constexpr int HDR_BARS = 0, HDR_Q = 512, HDR_QS = HDR_Q + GR * D * 2;
  static constexpr int HDR_MISC = HDR_QS + 64;
  // decode step: the new token's K and V rows (codes, then meta), each at a
  // 16-byte aligned stride (the quantizer stores up to 8 bytes at a time)
  static constexpr int NEW_STRIDE = ((RB + MB + 15) / 16) * 16;
  static constexpr int HDR_NEW = HDR_MISC + 64;
  // with two PV n-tiles the QK query fragments are read from shared memory
  // (8 x 32 lanes x 8 B) instead of being held in 16 registers per thread
  static constexpr bool QB_SMEM = false;
  static constexpr int HDR_QF = HDR_NEW + 2 * NEW_STRIDE;
  // per-channel K: the g query rows times each dim's 2^(EMAX - e), fp16;
  // Oaken: the query table [D][GR] fp32 of the K slots' products, and each
  // warp's slot scores [32 tokens][GR] fp32
  static constexpr int QF_BYTES =
      QB_SMEM ? 8 * 32 * 8 : (KPC ? GR * D * 2 : (OAK ? (D + kWarps * 32) * GR * 4 : 0));
  static constexpr int HDR_BYTES = ((HDR_QF + QF_BYTES + 127) / 128) * 128;
  // four CTAs per SM (128 registers a thread) where three stages per warp
  // fit in a quarter of the SM's shared memory (4 x (56 KB + 1 KB reserved)
  // <= 228 KB), else three
  static constexpr int MIN_CTAS =
      (NO == 1 && HDR_BYTES + kWarps * 3 * STAGE <= 56 * 1024) ? 4 : 3;
  static constexpr int SMEM_BUDGET = (MIN_CTAS == 4 ? 56 : 74) * 1024;
  static constexpr int STAGES_RAW = (SMEM_BUDGET - HDR_BYTES) / (kWarps * STAGE);
  static constexpr int STAGES = STAGES_RAW < 2 ? 2 : (STAGES_RAW > 16 ? 16 : STAGES_RAW);
  static constexpr int SMEM = HDR_BYTES + kWarps * STAGES * STAGE;
  static constexpr int EMAX = WordPairs<BITS>::kEmax;
  // FP8 weights P' = p * s_V carry an exact 2^8 (E4M3) or 2^14 (E5M2): their
  // scales (|max| / 448, / 57344) would otherwise put small weights among the
  // fp16 subnormals, where the (hi, lo) split loses its bits; the largest
  // scale times the factor stays below 65504.  The output undoes it.
  static constexpr float PSCALE = BITS == kE4M3 ? 256.0f : (BITS == kE5M2 ? 16384.0f : 1.0f);
  static constexpr float INV_PSCALE = 1.0f / PSCALE;
  // the warp merge reuses the stage buffers: m, l, o of kWarps x 8 rows
  static constexpr int MERGE_BYTES = (2 * kWarps * 8 + kWarps * 8 * D + 8 * (kWarps + 2)) * 4;
  static_assert(NG * GR <= 8, "at most eight (head, group) combinations");
  static_assert(kWarps * STAGES * 8 <= HDR_Q, "mbarriers fit the header");
  static_assert(MERGE_BYTES <= kWarps * STAGES * STAGE, "merge scratch fits the stages");
  static_assert(HDR_NEW % 16 == 0 && NEW_STRIDE % 16 == 0, "aligned new-token rows");
  static_assert(WordPairs<BITS>::kPairs * KW == 16, "16 K pairs per lane and token");
  static_assert(CrossPairs<BITS>::kOut * VW == 16, "16 V dims per lane and token");
  // per-channel K: a stage is one block, and lane tig owns head tig % g with
  // its QK columns 2 tig (hi part) and 2 tig + 1 (lo part)
  static_assert(!KPC || ((BITS == 2 || BITS == 4 || BITS == 8) && STOK == kChannelBlock &&
                         CPH == 2 && HS == 1),
                "per-channel K: integer codes, one block per stage, two columns per head");
  // Oaken: one group per token (the plane's (s, z)), and the V slots'
  // scatter tile of one 16-token sub-tile (128 dims x 16 tokens of fp16)
  // fits the stage's code bytes
  static_assert(!OAK || (NG == 1 && !GPV && 2 * STOK * RB >= D * kTile * 2 && SUB == 2),
                "Oaken: one group per token, scatter tile inside the stage's codes");
};

// Token of MMA row r (0 .. 15) of a 16-token sub-tile.
__device__ __forceinline__ int tok_perm(int r) { return r ^ ((r >> 2) & 1); }

// 8x8 transpose of 16-bit elements across the warp: lane (gid, tig) gets
// elements (2 tig, gid) and (2 tig + 1, gid) of the matrix whose row gid,
// columns 2 tig, 2 tig + 1 it passed in.
__device__ __forceinline__ uint32_t transpose8x8(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// Two weights as (hi, -lo) pairs: hi = fp16(x), -lo = fp16(hi - x), the
// remainder formed exactly in fp32 from the fp16 hi.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& r0, uint32_t& r1) {
  const uint32_t hh = pack_h2(x0, x1);
  float n0, n1;
  asm("{.reg .f16 l, h;\n mov.b32 {l, h}, %2;\n sub.rn.f32.f16 %0, l, %3;\n"
      " sub.rn.f32.f16 %1, h, %4;\n}"
      : "=f"(n0), "=f"(n1)
      : "r"(hh), "f"(x0), "f"(x1));
  r0 = pack_h2(x0, n0);
  r1 = pack_h2(x1, n1);
}

// Centre two 8-bit codes held as fp16 subnormals c * 2^-24: c - 128, exact
// (|c - 128| <= 128).
__device__ __forceinline__ uint32_t center8(uint32_t v) {
  return h2_as_u32(__hsub2(u32_as_h2(v), u32_as_h2(0x00800080u)));
}

template <int BITS, int GE, int GR, bool KPC>
__global__ void __launch_bounds__(kWarps * 32, TmCfg<BITS, GE, GR, KPC>::MIN_CTAS)
decode_tm_kernel(const __grid_constant__ SplitParams P) {
  using C = TmCfg<BITS, GE, GR, KPC>;
  using WP = WordPairs<BITS>;
  using XP = CrossPairs<BITS>;
  constexpr bool OAK = C::OAK;
  // the zero point the codes are read against: symmetric INT8 codes are read
  // as offset binary (c + 128) with a stored zero point of 0.  On the V side
  // 8-bit codes enter the tensor cores centred (c - 128, so symmetric INT8
  // codes end up as c itself, with z = 0): the PV products are summed over
  // a whole split, and offset codes near 128 would make those sums large
  // while the output is their small difference
  constexpr bool CENTER8 = BITS == 8 || BITS == kSym8;
  auto zero_of = [](float z) {
    if constexpr (BITS == kSym8)
      return z + 128.0f;
    else
      return z;
  };
  auto zero_of_v = [](float z) {
    if constexpr (BITS == 8)
      return z - 128.0f;
    else
      return z;
  };
  auto cen = [](uint32_t v) {
    if constexpr (CENTER8)
      return center8(v);
    else
      return v;
  };
  constexpr int D = C::D, NG = C::NG, NP = C::NP, HS = C::HS, CPH = C::CPH;
  // grouped PV: dims of each group per lane, and their V bytes and words
  constexpr int CH = GE / 8, VBG = CH * code_bits(BITS) / 8, VWG = VBG >= 4 ? VBG / 4 : 1;
  const DecodeArgs& a = P.a;
  const SegView& seg = P.seg;

  extern __shared__ __align__(128) uint8_t smem[];
  grid_dependents_may_launch();
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int gid = lane >> 2, tig = lane & 3;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::HDR_BARS) + warp * C::STAGES;
  __half* q_sm = reinterpret_cast<__half*>(smem + C::HDR_Q);      // [GR][D]
  float* qs_sm = reinterpret_cast<float*>(smem + C::HDR_QS);      // [8] per QK column
  float* hsc_sm = qs_sm + 8;  // [8] score scale of each query head
  int* unit_sm = reinterpret_cast<int*>(smem + C::HDR_MISC);
  int* fail_sm = unit_sm + 1;
  int* qexp_sm = unit_sm + 8;  // [8] power-of-two shift of each staged query row
  // decode step: the new token's quantized K and V rows (codes, then meta)
  uint8_t* new_sm = smem + C::HDR_NEW;
  uint2* qf_sm = reinterpret_cast<uint2*>(smem + C::HDR_QF);     // [8 ks][32 lanes]
  uint8_t* stages = smem + C::HDR_BYTES + warp * C::STAGES * C::STAGE;
  uint32_t* counters = a.err + seg.ctr;  // [0] next unit, [1] CTAs done

  // ---- per-lane constants
  // QK B column gid: head (gid / CPH) mod g, group gid mod NG; the lane's K
  // chunk lies in group kgrp
  const int kgrp = (32 * tig) / GE;
  const bool qb_ok = (gid % NG) == kgrp;
  const int qh = (gid / CPH) % GR;
  // heads owned by this lane (slot s) and the group of each PV block b
  int own_h[HS];
#pragma unroll
  for (int s = 0; s < HS; ++s) own_h[s] = (CPH == 1) ? 2 * tig + s : ((2 * tig) / CPH) % GR;
  auto slot_of = [](int b) { return HS == 2 ? b : 0; };
  int gv[NP];
#pragma unroll
  for (int b = 0; b < NP; ++b)
    gv[b] = NG == 1 ? 0 : (NG == 2 ? (NP == 2 ? b : (tig & 1)) : (NP == 2 ? 2 * b + (tig & 1) : tig));
  const bool distinct = tig < C::W;        // this lane's combinations are not repeats
  const int dgrp = (16 * gid) / GE;        // group of the lane's 16 output dims
  const float score_scale = a.scale_log2 * pow2f(24 - C::EMAX);
  // the largest power of two a query element is lifted by before it becomes
  // an fp16 operand: 2^(EMAX - e) for the code exponent e = 0
  constexpr int QUP = C::EMAX - WP::exp(0);
  // tokens of the lane's QK rows and PV k positions within a sub-tile
  const int tq0 = tok_perm(gid);
  const int tvA = tok_perm(2 * tig), tvB = tok_perm(2 * tig + 1);

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

  // a decode step appends one token at position L_old (dropped when the
  // cache is full) and attends over it too
  const int L_old = max(0, min(seg.seq_lens[b], seg.max_tokens));
  const bool step = a.k_new != nullptr;
  const int L = (step && L_old < seg.max_tokens) ? L_old + 1 : L_old;
  int c0, c1;
  split_range(L, seg.n_split, split, c0, c1);
  const int unit_stages = (c1 > c0) ? (c1 - c0 + C::STOK - 1) / C::STOK : 0;
  const int n_tiles = (unit_stages > warp) ? (unit_stages - warp + kWarps - 1) / kWarps : 0;
  const int w0 = c0 + warp * C::STOK;  // first token of this warp's first stage
  // this unit writes the new token; the warp holding its stage patches the
  // stage in shared memory after the copy lands (the copy may read the row
  // before or after the global store)
  const bool append_here = step && L > L_old && c0 <= L_old && L_old < c1;
  const int patch_stage = (L_old - c0) / C::STOK;
  const int patch_i = (append_here && patch_stage % kWarps == warp) ? patch_stage / kWarps : -1;
  const int patch_row = (L_old - c0) % C::STOK;

  // A stage is filled by one bulk copy per plane (K codes, V codes, K meta,
  // V meta), issued side by side by lanes 0 .. NCOPY-1: lane j holds its
  // plane's source for this warp's first stage, its per-stage stride, its
  // byte count and its offset inside a stage.
  constexpr int NCOPY = C::MB > 0 ? 4 : 2;
  const long long row0 = ((long long)b * a.kv_heads + kvh) * seg.max_tokens + w0;
  const int cp_j = lane < NCOPY ? lane : 0;
  const int cp_rb = (cp_j < 2) ? C::RB : (cp_j == 2 ? C::MBK : C::MB);  // bytes per token
  const uint8_t* cp_src = (cp_j == 0 ? seg.k_codes : cp_j == 1 ? seg.v_codes
                           : cp_j == 2 ? seg.k_meta : seg.v_meta) + row0 * cp_rb;
  const uint32_t cp_off = cp_j == 0 ? 0u : cp_j == 1 ? (uint32_t)(C::STOK * C::RB)
                          : cp_j == 2 ? (uint32_t)(2 * C::STOK * C::RB)
                                      : (uint32_t)(2 * C::STOK * C::RB + C::STOK * C::MBK);
  const uint32_t cp_bytes = (uint32_t)(C::STOK * cp_rb);
  const size_t cp_stride = (size_t)(kWarps * C::STOK) * cp_rb;
  // stage i of this warp into ring slot st (all lanes call it together)
  auto issue = [&](int i, int st) {
    if (lane == 0) mbar_arrive_expect_tx(&bars[st], C::STAGE);
    __syncwarp();
    if (lane < NCOPY)
      bulk_load(stages + st * C::STAGE + cp_off, cp_src + (size_t)i * cp_stride, cp_bytes,
                &bars[st], policy);
  };
  {
    const int pre = min(n_tiles, C::STAGES);
    for (int i = 0; i < pre; ++i) issue(i, (st + i) % C::STAGES);
  }

  // ---- decode step: quantize the new K (lanes 0-15) and V (16-31) rows of
  // this KV head into shared memory, then copy them to the cache (the
  // Oaken codec appends with its own kernel before the attention)
  if constexpr (BITS != 16 && !KPC && !OAK) {
    if (append_here && warp == 0) {
      const int vh = lane >> 4, l16 = lane & 15;
      const __half* src = (vh ? a.v_new : a.k_new) + ((long long)b * a.kv_heads + kvh) * D;
      uint8_t* row = new_sm + vh * C::NEW_STRIDE;
      quantize_slice<BITS, GE>(src, row, row + C::RB, l16, true);
      __syncwarp();
      const long long dst = ((long long)b * a.kv_heads + kvh) * seg.max_tokens + L_old;
      uint8_t* gc = const_cast<uint8_t*>(vh ? seg.v_codes : seg.k_codes) + dst * C::RB;
      uint8_t* gm = const_cast<uint8_t*>(vh ? seg.v_meta : seg.k_meta) + dst * C::MB;
      for (int i = l16; i < C::RB / 4; i += 16)
        reinterpret_cast<uint32_t*>(gc)[i] = reinterpret_cast<const uint32_t*>(row)[i];
      if (l16 < C::MB / 4)
        reinterpret_cast<uint32_t*>(gm)[l16] = reinterpret_cast<const uint32_t*>(row + C::RB)[l16];
    }
  }

  // ---- the g query rows of this KV head, once per unit, and each head's
  // score scale (undoing its row's power-of-two shift), read from shared
  // memory where it is used rather than held in registers across the loop
  stage_queries<GR, QUP>(a, b, kvh, q_sm, qexp_sm, t);
  __syncthreads();
  if (t >= 64 && t < 64 + GR) hsc_sm[t - 64] = score_scale * unshift(qexp_sm[t - 64]);
  // column sums of q in the QK MMA's units (it returns 2^(EMAX - 24) sum q c)
  if constexpr (BITS != 16 && !KPC) {
    if (t < 64) {
      const int r = t >> 3, part = t & 7;
      const __half* qr = q_sm + ((r / CPH) % GR) * D + (r % NG) * GE + part * (GE / 8);
      float acc = 0.f;
#pragma unroll 4
      for (int i = 0; i < GE / 8; ++i) acc += __half2float(qr[i]);
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (part == 0) qs_sm[r] = acc * pow2f(C::EMAX - 24);
    }
  }
  // Oaken: the K slots' query table, otab[j][h] = q_h,j s_out in the QK
  // MMA's units (2^(EMAX - 24) times the staged, shifted query)
  float* otab = reinterpret_cast<float*>(smem + C::HDR_QF);             // [D][GR]
  float* spx = otab + D * GR + warp * 32 * GR;                          // [32][GR]
  if constexpr (OAK) {
    const float f = pow2f(C::EMAX - 24) * seg.k_oaken.s_out;
    for (int i = t; i < D * GR; i += kWarps * 32)
      otab[i] = __half2float(q_sm[(i % GR) * D + i / GR]) * f;
  }
  __syncthreads();
  // B fragments of QK: pair p = 2 ks + h of this lane's chunk, column gid;
  // each element scaled by 2^(EMAX - e) for the exponent e of its code
  uint32_t qb[C::QB_SMEM ? 1 : 8][2];
  if constexpr (!KPC) {
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
        const uint32_t v =
            qb_ok ? pack_h2(__half2float(qrow[d0]) * f, __half2float(qrow[d1]) * f) : 0u;
        if constexpr (C::QB_SMEM) {
          if (warp == 0) reinterpret_cast<uint32_t*>(&qf_sm[ks * 32 + lane])[h] = v;
        } else {
          qb[ks][h] = v;
        }
      }
    }
    if constexpr (C::QB_SMEM) __syncthreads();
  }
  const float qsA = (BITS != 16 && !KPC) ? qs_sm[2 * tig] : 0.f;
  const float qsB = (BITS != 16 && !KPC) ? qs_sm[2 * tig + 1] : 0.f;
  // Oaken planes' parameters (unused for the other formats)
  const float ks_in = seg.k_oaken.s_in, kz_in = seg.k_oaken.z;
  const float vs_in = seg.v_oaken.s_in, vz_in = seg.v_oaken.z;
  const float v_ratio = seg.v_oaken.s_out / seg.v_oaken.s_in;

  // Per-channel K: the QK B fragments of a block are q * s_d for the block's
  // channel scales, in two fp16 parts (hi in the even columns, lo = the fp32
  // remainder in the odd ones: q * s is exact in fp32, hi + lo keeps 22
  // bits), each element times 2^(EMAX - e) as above; the zero points enter
  // as the block's bias sum_d q_d s_d z_d per head, in the MMA's units.
  float kbias = 0.f;
  __half* qf_tab = reinterpret_cast<__half*>(smem + C::HDR_QF);  // [GR][D] (per-channel K)
  if constexpr (KPC) {
    // q * 2^(EMAX - e) of each dim, once per unit (lanes of one head and
    // chunk write the same values)
    const __half* qrow = q_sm + qh * D + 32 * tig;
    __half* qfrow = qf_tab + qh * D + 32 * tig;
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const int j = p % WP::kPairs;
      const int blk = (p / WP::kPairs) * WP::kDims;
      const float f = pow2f(C::EMAX - WP::exp(j));
      qfrow[blk + WP::dim(j, 0)] = __float2half_rn(__half2float(qrow[blk + WP::dim(j, 0)]) * f);
      qfrow[blk + WP::dim(j, 1)] = __float2half_rn(__half2float(qrow[blk + WP::dim(j, 1)]) * f);
    }
    __syncthreads();
  }
  // d = fp32 a * b + c for fp16 a, b (the product is exact)
  auto fma_h = [](__half a, __half b, float c) {
    float d;
    asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(__half_as_ushort(a)),
        "h"(__half_as_ushort(b)), "f"(c));
    return d;
  };
  auto kpc_rebuild = [&](const uint8_t* sKm) {
    if constexpr (KPC) {
      constexpr int KD = WP::kDims;  // dims of one code word
      const __half* qfrow = qf_tab + qh * D + 32 * tig;
      const __half2* szr = reinterpret_cast<const __half2*>(sKm) + 32 * tig;  // (s, z) of its channels
      const bool lo_part = gid & 1;
      // the chunk's zero points as A rows of the bias MMA: pair p holds
      // (z_d0, z_d1) 2^(e_j - 24), exact in fp16 (z is an integer), the
      // units of the codes
      uint32_t zf[16];
#pragma unroll
      for (int wb = 0; wb < 32 / KD; ++wb) {
        // this word block's query values and (s, z) pairs, in vector loads
        __half qd[KD];
        __half2 szd[KD];
#pragma unroll
        for (int i = 0; i < KD; i += 8)
          *reinterpret_cast<uint4*>(&qd[i]) = *reinterpret_cast<const uint4*>(qfrow + wb * KD + i);
        if constexpr (KD == 4)
          *reinterpret_cast<uint2*>(&qd[0]) = *reinterpret_cast<const uint2*>(qfrow + wb * KD);
#pragma unroll
        for (int i = 0; i < KD; i += 4)
          *reinterpret_cast<uint4*>(&szd[i]) = *reinterpret_cast<const uint4*>(szr + wb * KD + i);
#pragma unroll
        for (int j = 0; j < WP::kPairs; ++j) {
          const int p = wb * WP::kPairs + j;
          const __half2 sz0 = szd[WP::dim(j, 0)], sz1 = szd[WP::dim(j, 1)];
          const __half q0 = qd[WP::dim(j, 0)], q1 = qd[WP::dim(j, 1)];
          const __half2 hi = __hmul2(__halves2half2(q0, q1), __lows2half2(sz0, sz1));
          const float r0 = fma_h(q0, __low2half(sz0), -__low2float(hi));
          const float r1 = fma_h(q1, __low2half(sz1), -__high2float(hi));
          const __half2 lo = __floats2half2_rn(r0, r1);
          qb[p / 2][p % 2] = h2_as_u32(lo_part ? lo : hi);
          zf[p] = h2_as_u32(
              __hmul2(__highs2half2(sz0, sz1), __float2half2_rn(pow2f(WP::exp(j) - 24))));
        }
      }
      // every row of the accumulator is sum_d z_d (q s)_d over the column's
      // part, in the QK MMA's units: columns 2 tig (hi) and 2 tig + 1 (lo)
      // of head tig mod g, the lane's own
      float b_even[4] = {0.f, 0.f, 0.f, 0.f}, b_odd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_f16((ks & 1) ? b_odd : b_even, zf[2 * ks], zf[2 * ks], zf[2 * ks + 1], zf[2 * ks + 1],
                qb[ks][0], qb[ks][1]);
      kbias = (b_even[0] + b_odd[0]) + (b_even[1] + b_odd[1]);
    }
  };

  // ---- running state.  m_ref (per owned head) is a reference point at
  // least as large as every score seen, so p = 2^(x - m_ref) <= 1 and
  // P' = p * s_V stays within fp16 range; it moves (with a rescale) only when
  // a stage's max exceeds it, and then to that max + kLazy.
  float o_acc[C::NO][8][4];
#pragma unroll
  for (int nb = 0; nb < C::NO; ++nb)
#pragma unroll
    for (int i = 0; i < 8; ++i) o_acc[nb][i][0] = o_acc[nb][i][1] = o_acc[nb][i][2] = o_acc[nb][i][3] = 0.f;
  float corr[NP];  // sum of P' * z_V of combination (b, tig) over this lane's tokens
#pragma unroll
  for (int nb = 0; nb < NP; ++nb) corr[nb] = 0.f;
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
    kpc_rebuild(sKm);
    if constexpr (OAK) {
      // the K outlier slots' score terms, lane = token of the stage: sum
      // over its slots of d * otab[dim] for every query head, into spx
      // (a slot is the dim in its low byte, the signed shift in its high
      // byte; an empty slot is 0 and adds 0; rows past the valid length may
      // hold any bytes, their scores are masked below)
      const uint4* sl = reinterpret_cast<const uint4*>(sKm + lane * C::MB);
      const uint4 s0 = sl[0], s1 = sl[1];
      const uint32_t sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      if constexpr (GR % 2 == 0) {
        // heads in pairs: packed f32x2 products
        uint64_t acc[GR / 2];
#pragma unroll
        for (int h = 0; h < GR / 2; ++h) acc[h] = 0ull;
#pragma unroll
        for (int k = 0; k < KVQ_OAKEN_SLOTS; ++k) {
          const uint32_t u = (k & 1) ? (sw[k >> 1] >> 16) : sw[k >> 1];
          const float d = (float)(int)(int8_t)(uint8_t)(u >> 8);
          const uint64_t d2 = f2_pack(d, d);
          const uint64_t* tr = reinterpret_cast<const uint64_t*>(otab + (u & 0x7Fu) * GR);
#pragma unroll
          for (int h = 0; h < GR / 2; ++h) acc[h] = f2_fma(d2, tr[h], acc[h]);
        }
#pragma unroll
        for (int h = 0; h < GR / 2; ++h) reinterpret_cast<uint64_t*>(spx + lane * GR)[h] = acc[h];
      } else {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < KVQ_OAKEN_SLOTS; ++k) {
          const uint32_t u = (k & 1) ? (sw[k >> 1] >> 16) : sw[k >> 1];
          acc = fmaf((float)(int)(int8_t)(uint8_t)(u >> 8), otab[u & 0x7Fu], acc);
        }
        spx[lane] = acc;
      }
      __syncwarp();
    }
    auto valid = [&](int tok) { return FULL || tok < n_valid; };  // tok: 0 .. STOK-1
    // V rows past the valid length may hold any bytes.  Integer codes are
    // finite and meet a zero weight; raw fp16 and FP8 bytes can be NaN or
    // Inf, which a zero weight does not cancel in the MMA: zero those words.
    auto zero_invalid = [&](int sub, auto& wA, auto& wB, auto& wC, auto& wD) {
      if constexpr ((BITS == 16 || BITS == kE4M3 || BITS == kE5M2) && !FULL) {
        constexpr int NW = sizeof(wA) / sizeof(wA[0]);
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          wA[w] = valid(sub * kTile + tvA) ? wA[w] : 0u;
          wB[w] = valid(sub * kTile + tvB) ? wB[w] : 0u;
          wC[w] = valid(sub * kTile + tvA + 8) ? wC[w] : 0u;
          wD[w] = valid(sub * kTile + tvB + 8) ? wD[w] : 0u;
        }
      }
    };

    // ---- S^T = K * Qx^T per sub-tile: rows gid, gid + 8
    float x[NS][HS][2];
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
      // two accumulators (even and odd k-steps): two dependent MMA chains of
      // four instead of one of eight
      float s_acc[4] = {0.f, 0.f, 0.f, 0.f}, s_odd[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t k0[C::KW], k1[C::KW];
      load_chunk<C::KC, C::KW>(sK + (sub * kTile + tq0) * C::RB + tig * C::KC, k0);
      load_chunk<C::KC, C::KW>(sK + (sub * kTile + tq0 + 8) * C::RB + tig * C::KC, k1);
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
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t b0, b1;
        if constexpr (C::QB_SMEM) {
          const uint2 v = qf_sm[ks * 32 + lane];
          b0 = v.x;
          b1 = v.y;
        } else {
          b0 = qb[ks][0];
          b1 = qb[ks][1];
        }
        mma_f16((ks & 1) ? s_odd : s_acc, p0[2 * ks], p1[2 * ks], p0[2 * ks + 1],
                p1[2 * ks + 1], b0, b1);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) s_acc[c] += s_odd[c];
      // the owned heads' scores: sum over their groups of s_K * (S - z_K * qs);
      // rows past the valid length may hold any bytes: masked below by select
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int tok = sub * kTile + tq0 + 8 * r;
        float v[HS];
        if constexpr (BITS == 16) {
          v[0] = s_acc[2 * r];
          if constexpr (HS == 2) v[HS - 1] = s_acc[2 * r + 1];
        } else if constexpr (KPC) {
          v[0] = s_acc[2 * r] + s_acc[2 * r + 1] - kbias;
        } else if constexpr (OAK) {
          // the plane's (s_in, z_in), plus the token's slot terms
          const float* sp = spx + tok * GR;
          v[0] = fmaf(ks_in, fmaf(-kz_in, qsA, s_acc[2 * r]), sp[own_h[0]]);
          if constexpr (HS == 2)
            v[HS - 1] = fmaf(ks_in, fmaf(-kz_in, qsB, s_acc[2 * r + 1]), sp[own_h[HS - 1]]);
        } else if constexpr (NG == 1) {
          const float2 sz = __half22float2(*reinterpret_cast<const __half2*>(sKm + tok * C::MB));
          v[0] = sz.x * fmaf(-zero_of(sz.y), qsA, s_acc[2 * r]);
          if constexpr (HS == 2) v[HS - 1] = sz.x * fmaf(-zero_of(sz.y), qsB, s_acc[2 * r + 1]);
        } else {
          const uint2 u = *reinterpret_cast<const uint2*>(
              sKm + tok * C::MB + (NG == 4 ? 8 * (tig & 1) : 0));
          const float2 szA = __half22float2(u32_as_h2(u.x));
          const float2 szB = __half22float2(u32_as_h2(u.y));
          v[0] = fmaf(szB.x, fmaf(-zero_of(szB.y), qsB, s_acc[2 * r + 1]),
                      szA.x * fmaf(-zero_of(szA.y), qsA, s_acc[2 * r]));
          if constexpr (NG == 4) v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
        }
        const bool ok = valid(tok);
#pragma unroll
        for (int s = 0; s < HS; ++s) x[sub][s][r] = ok ? v[s] * hsc_sm[own_h[s]] : -INFINITY;
      }
    }

    // ---- online softmax per owned head: max over the stage's tokens (rows
    // gid and gid + 8 of every sub-tile, then across gid).  The reference
    // point moves rarely, so a warp vote first asks whether any lane's own
    // scores exceed it; only then are the maxima reduced across the rows.
    bool any_rescale = false;
    float alpha[HS];
    float lmax[HS];
    bool up = false;
#pragma unroll
    for (int s = 0; s < HS; ++s) {
      lmax[s] = -INFINITY;
#pragma unroll
      for (int sub = 0; sub < NS; ++sub) lmax[s] = fmaxf(lmax[s], fmaxf(x[sub][s][0], x[sub][s][1]));
      up |= lmax[s] > m_ref[s];
      alpha[s] = 1.f;
    }
    if (__any_sync(0xffffffffu, up)) {
#pragma unroll
      for (int s = 0; s < HS; ++s) {
        float tmax = lmax[s];
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 8));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        if (tmax > m_ref[s]) {
          const float m_new = tmax + kLazy;
          if (m_ref[s] != -INFINITY) {
            alpha[s] = fast_exp2(m_ref[s] - m_new);
            any_rescale = true;
          }
          m_ref[s] = m_new;
        }
      }
    }
    if (__any_sync(0xffffffffu, any_rescale)) {
      // every factor is this lane's own: the accumulator columns of PV block
      // b belong to the lane position that owns their head
#pragma unroll
      for (int s = 0; s < HS; ++s) l_part[s] *= alpha[s];
#pragma unroll
      for (int nb = 0; nb < C::NO; ++nb) {
        const float al = alpha[C::GPV ? 0 : slot_of(nb)];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) o_acc[nb][i][c] *= al;
      }
#pragma unroll
      for (int nb = 0; nb < NP; ++nb) corr[nb] *= alpha[slot_of(nb)];
    }

    // ---- weights and O^T += V^T * P'^T per sub-tile
    float p_keep[OAK ? NS : 1][HS][2];  // Oaken: the weights, for the V slots below
    (void)p_keep;
#pragma unroll
    for (int sub = 0; sub < NS; ++sub) {
      float p[HS][2];
#pragma unroll
      for (int s = 0; s < HS; ++s)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          p[s][r] = fast_exp2(x[sub][s][r] - m_ref[s]);  // 0 for masked tokens
          l_part[s] += p[s][r];
          if constexpr (OAK) p_keep[sub][s][r] = p[s][r];
        }
      uint32_t bf0[NP], bf1[NP];
#pragma unroll
      for (int nb = 0; nb < NP; ++nb) {
        float pp[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if constexpr (BITS == 16 || OAK) {
            // raw fp16; or the Oaken codec, whose one V scale and zero
            // point are applied at the output (z_in times the weights' sum)
            pp[r] = p[slot_of(nb)][r];
          } else {
            const int tok = sub * kTile + tq0 + 8 * r;
            // slots past the valid length may hold any bytes (NaN scales):
            // select, never multiply by a zero weight
            const float2 sz = __half22float2(*reinterpret_cast<const __half2*>(
                sVm + tok * C::MB + gv[nb] * 4));
            const bool ok = valid(tok);
            pp[r] = ok ? p[slot_of(nb)][r] * (sz.x * C::PSCALE) : 0.f;
            // in the weights' units: PSCALE is 1 for every format with a
            // zero point (the FP8 formats, lifted, have zero points of 0)
            corr[nb] = ok ? fmaf(pp[r], zero_of_v(sz.y), corr[nb]) : corr[nb];
          }
        }
        uint32_t r0, r1;
        split_pair(pp[0], pp[1], r0, r1);
        bf0[nb] = transpose8x8(r0);  // k positions 0 .. 7 (rows 0 .. 7)
        bf1[nb] = transpose8x8(r1);  // k positions 8 .. 15
      }

      if constexpr (C::GPV) {
        // m-tiles 4 gv .. 4 gv + 3 are group gv's dims: rows gid, gid + 8 of
        // m-tile 4 gv + j are dims gv * G + gid * CH + j and + CH / 2
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
          const uint8_t* vb =
              sV + sub * kTile * C::RB + gq * (GE * code_bits(BITS) / 8) + gid * VBG;
          uint32_t wA[VWG], wB[VWG], wC[VWG], wD[VWG];
          load_chunk<VBG, VWG>(vb + tvA * C::RB, wA);
          load_chunk<VBG, VWG>(vb + tvB * C::RB, wB);
          load_chunk<VBG, VWG>(vb + (tvA + 8) * C::RB, wC);
          load_chunk<VBG, VWG>(vb + (tvB + 8) * C::RB, wD);
          zero_invalid(sub, wA, wB, wC, wD);
          uint32_t xa[VWG * XP::kOut], xc[VWG * XP::kOut];
#pragma unroll
          for (int w = 0; w < VWG; ++w) {
            uint32_t ya[XP::kOut], yc[XP::kOut];
            XP::run(wA[w], wB[w], ya);
            XP::run(wC[w], wD[w], yc);
#pragma unroll
            for (int i = 0; i < XP::kOut; ++i) {
              xa[w * XP::kOut + i] = cen(ya[i]);
              xc[w * XP::kOut + i] = cen(yc[i]);
            }
          }
#pragma unroll
          for (int j = 0; j < CH / 2; ++j)
            mma_f16(o_acc[0][gq * (CH / 2) + j], xa[j], xa[j + CH / 2], xc[j],
                    xc[j + CH / 2], bf0[gq], bf1[gq]);
        }
      } else {
        const uint8_t* vb = sV + sub * kTile * C::RB + gid * C::VB;
        uint32_t wA[C::VW], wB[C::VW], wC[C::VW], wD[C::VW];
        load_chunk<C::VB, C::VW>(vb + tvA * C::RB, wA);
        load_chunk<C::VB, C::VW>(vb + tvB * C::RB, wB);
        load_chunk<C::VB, C::VW>(vb + (tvA + 8) * C::RB, wC);
        load_chunk<C::VB, C::VW>(vb + (tvB + 8) * C::RB, wD);
        zero_invalid(sub, wA, wB, wC, wD);
        uint32_t xa[16], xc[16];
#pragma unroll
        for (int w = 0; w < C::VW; ++w) {
          uint32_t ya[XP::kOut], yc[XP::kOut];
          XP::run(wA[w], wB[w], ya);
          XP::run(wC[w], wD[w], yc);
#pragma unroll
          for (int i = 0; i < XP::kOut; ++i) {
            xa[w * XP::kOut + i] = cen(ya[i]);
            xc[w * XP::kOut + i] = cen(yc[i]);
          }
        }
#pragma unroll
        for (int nb = 0; nb < NP; ++nb)
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
            mma_f16(o_acc[nb][mt], xa[mt], xa[mt + 8], xc[mt], xc[mt + 8], bf0[nb], bf1[nb]);
      }
    }

    if constexpr (OAK) {
      // ---- the V outlier slots: O^T += Vd^T * P_sp^T per sub-tile, into the
      // same accumulators.  Vd is the sub-tile's slots scattered into a
      // dense fp16 tile [128 dims][16 tokens] (d * 2^(e - 24), the exponent
      // of the dim's code position, so the output scale of the dense codes
      // applies), built in the stage's code bytes, which both products have
      // consumed; P_sp = p * s_out / s_in in the dense weights' (hi, -lo)
      // layout, so that the output's s_in gives s_out * d.  Tile row of dim
      // j: (j % 16) * 8 + j / 16, the rows of one m-tile's 8x8 blocks being
      // consecutive; the two 16-byte halves of a row (tokens 0-7, 8-15)
      // swap when bit 2 of the row is set, which keeps the 8x8 loads free
      // of bank conflicts.
      uint8_t* vd = const_cast<uint8_t*>(sK);
      const uint32_t vd_sm = smem_u32(vd);
      const int tt = lane & 15, hf = lane >> 4;  // scatter: token tt, slots 8 hf .. 8 hf + 7
      const int kap = tok_perm(tt);              // its k position in the products
      const int mq = lane >> 3, i8 = lane & 7;   // 8x8 load: block mq, row i8
      // an empty slot (0: dim 0, shift 0) must not overwrite a real outlier
      // at dim 0 of the same token: its store goes to a spare byte pair in
      // the consumed K slots
      __half* spare = reinterpret_cast<__half*>(const_cast<uint8_t*>(sKm)) + lane;
      const uint32_t kap_bits = ((uint32_t)(kap >> 3) << 4) | ((uint32_t)(kap & 7) << 1);
#pragma unroll
      for (int sub = 0; sub < NS; ++sub) {
        uint32_t bs0[NP], bs1[NP];
#pragma unroll
        for (int nb = 0; nb < NP; ++nb) {
          uint32_t r0, r1;
          split_pair(p_keep[sub][slot_of(nb)][0] * v_ratio, p_keep[sub][slot_of(nb)][1] * v_ratio,
                     r0, r1);
          bs0[nb] = transpose8x8(r0);
          bs1[nb] = transpose8x8(r1);
        }
        __syncwarp();  // every lane is done reading the tile (codes or slots)
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<uint4*>(vd)[i * 32 + lane] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
        {
          const uint4 w = *reinterpret_cast<const uint4*>(sVm + (sub * kTile + tt) * C::MB +
                                                          hf * 16);
          const uint32_t sw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t u = (k & 1) ? (sw[k >> 1] >> 16) : sw[k >> 1];
            const int d = (int)(int8_t)(uint8_t)(u >> 8);
            const uint32_t j = u & 0x7Fu;
            // byte offset: row (j % 16) * 8 + j / 16 of 32 bytes, the row's
            // half for the token (swapped when bit 2 of the row, j's bit 6,
            // is set), the token's pair of bytes
            const uint32_t off = ((j & 15u) << 8) | ((j >> 4) << 5) | (((j >> 2) & 16u) ^ kap_bits);
            // d * 2^(e - 24): the exact fp16 integer d times a power of two
            const __half hv = __hmul(__int2half_rn(d), __ushort_as_half((j & 1u) ? 0x0010 : 0x0001));
            *(d != 0 ? reinterpret_cast<__half*>(vd + off) : spare) = hv;
          }
        }
        __syncwarp();
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const uint32_t row = (uint32_t)((mt + 8 * (mq & 1)) * 8 + i8);
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(vd_sm + row * 32u + ((uint32_t)((mq >> 1) ^ ((i8 >> 2) & 1)) << 4), a0, a1,
                      a2, a3);
#pragma unroll
          for (int nb = 0; nb < NP; ++nb) mma_f16(o_acc[nb][mt], a0, a1, a2, a3, bs0[nb], bs1[nb]);
        }
      }
      // the tile was written through the generic proxy; the ring's next bulk
      // copy into this stage comes through the async proxy
      fence_proxy_async_smem();
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
    const uint8_t* sVm = sKm + C::STOK * C::MBK;
    if constexpr (BITS != 16 && !KPC && !OAK) {
      if (i == patch_i) {
        // the new token's row, from the quantized copy in shared memory
        uint32_t* dK = reinterpret_cast<uint32_t*>(stages + st * C::STAGE + patch_row * C::RB);
        uint32_t* dV = dK + C::STOK * C::RB / 4;
        uint32_t* dKm = reinterpret_cast<uint32_t*>(stages + st * C::STAGE + 2 * C::STOK * C::RB +
                                                    patch_row * C::MB);
        uint32_t* dVm = dKm + C::STOK * C::MB / 4;
        const uint32_t* nK = reinterpret_cast<const uint32_t*>(new_sm);
        const uint32_t* nV = reinterpret_cast<const uint32_t*>(new_sm + C::NEW_STRIDE);
        for (int j = lane; j < C::RB / 4; j += 32) {
          dK[j] = nK[j];
          dV[j] = nV[j];
        }
        if (lane < C::MB / 4) {
          dKm[lane] = nK[C::RB / 4 + lane];
          dVm[lane] = nV[C::RB / 4 + lane];
        }
        fence_proxy_async_smem();  // before the ring refills this stage
        __syncwarp();
      }
    }
    const int n_stage = min(C::STOK, c1 - (w0 + i * kWarps * C::STOK));
    if (n_stage == C::STOK)
      stage_body(std::integral_constant<bool, true>(), sK, sV, sKm, sVm, C::STOK);
    else
      stage_body(std::integral_constant<bool, false>(), sK, sV, sKm, sVm, n_stage);
    __syncwarp();
    if (i + C::STAGES < n_tiles) issue(i + C::STAGES, st);
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

  // ---- warp totals: sums over the token rows (gid)
#pragma unroll
  for (int s = 0; s < HS; ++s) {
    l_part[s] += __shfl_xor_sync(0xffffffffu, l_part[s], 4);
    l_part[s] += __shfl_xor_sync(0xffffffffu, l_part[s], 8);
    l_part[s] += __shfl_xor_sync(0xffffffffu, l_part[s], 16);
  }
#pragma unroll
  for (int nb = 0; nb < NP; ++nb) {
    corr[nb] += __shfl_xor_sync(0xffffffffu, corr[nb], 4);
    corr[nb] += __shfl_xor_sync(0xffffffffu, corr[nb], 8);
    corr[nb] += __shfl_xor_sync(0xffffffffu, corr[nb], 16);
  }

  __syncthreads();
  float* ms = reinterpret_cast<float*>(smem + C::HDR_BYTES);  // [kWarps][8]
  float* ls = ms + kWarps * 8;                                 // [kWarps][8]
  float* os = ls + kWarps * 8;                                 // [kWarps][8][D]
  if (gid == 0 && distinct) {
    // lanes owning the same head hold the same values: any may write
#pragma unroll
    for (int s = 0; s < HS; ++s) {
      ms[warp * 8 + own_h[s]] = m_ref[s];
      ls[warp * 8 + own_h[s]] = l_part[s];
    }
  }
  if constexpr (C::GPV) {
    // every lane: head tig (its own), 8 dims of each group
    float* oh = os + (warp * 8 + own_h[0]) * D + gid * CH;
#pragma unroll
    for (int gq = 0; gq < NG; ++gq)
#pragma unroll
      for (int j = 0; j < CH / 2; ++j) {
        const float f0 = pow2f(24 - XP::exp(j % XP::kOut)) * C::INV_PSCALE;
        const float f1 = pow2f(24 - XP::exp((j + CH / 2) % XP::kOut)) * C::INV_PSCALE;
        const float* o = o_acc[0][gq * (CH / 2) + j];
        oh[gq * GE + j] = fmaf(o[0] - o[1], f0, -corr[gq]);
        oh[gq * GE + j + CH / 2] = fmaf(o[2] - o[3], f1, -corr[gq]);
      }
  } else if (distinct) {
#pragma unroll
    for (int nb = 0; nb < NP; ++nb) {
      if (gv[nb] == dgrp) {
        float* oh = os + (warp * 8 + own_h[slot_of(nb)]) * D + 16 * gid;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          // hi column minus the negated-remainder column, then undo the
          // subnormal code scale 2^(e - 24) of the row's dim
          // (Oaken: the plane's z_in times the weights' sum, and its s_in)
          const float f0 = pow2f(24 - XP::exp(mt % XP::kOut)) * C::INV_PSCALE;
          const float f1 = pow2f(24 - XP::exp((mt + 8) % XP::kOut)) * C::INV_PSCALE;
          const float cz = OAK ? vz_in * l_part[slot_of(nb)] : corr[nb];
          const float osc = OAK ? vs_in : 1.f;
          oh[mt] = osc * fmaf(o_acc[nb][mt][0] - o_acc[nb][mt][1], f0, -cz);
          oh[mt + 8] = osc * fmaf(o_acc[nb][mt][2] - o_acc[nb][mt][3], f1, -cz);
        }
      }
    }
  }
  __syncthreads();
  cta_merge_store<GR>(a, ms, ls, os, os + kWarps * 8 * D, b, kvh, seg.part_base + split, t);
  if (step && t == 0) advance_if_last(a, seg, b, seg.n_split * a.kv_heads, L);
  // the merge wrote the stage buffers: order that before the next unit's copies
  fence_proxy_async_smem();
  }  // unit loop

  if (t == 0) release_counters(counters);
  // after the previous segment's kernel (a no-op for a plain launch): the
  // merge after the last segment then sees every segment done
  grid_dependency_wait();
}

template <int BITS, int GE, int GR, bool KPC>
cudaError_t launch_tm(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  using C = TmCfg<BITS, GE, GR, KPC>;
  // the shared-memory opt-in is a per-device function attribute: set it once
  // per device (bit i of the mask = device i)
  static std::atomic<unsigned long long> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(decode_tm_kernel<BITS, GE, GR, KPC>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  SplitParams P{a, seg};
  const long long units = (long long)seg.n_split * a.kv_heads * a.batch;
  const long long slots = (long long)seg.sms * C::MIN_CTAS;  // one wave of persistent CTAs
  const unsigned grid = (unsigned)(units < slots ? units : slots);
  return launch_segment_kernel(decode_tm_kernel<BITS, GE, GR, KPC>, grid, kWarps * 32, C::SMEM, s,
                               seg.after_prev != 0, P);
}

// Per-channel K (G is V's group size): the (bits, G, g) whose QK columns
// give lane tig head tig % g in two columns (see TmCfg).
#define KVQ_TM_KPC_FORMATS(X) X(4, 64, 4) X(8, 128, 1) X(4, 128, 4) X(4, 128, 1)

// Every (bits, G, g) with NG * g <= 8 that the cache formats allow.
#define KVQ_TM_FORMATS(X)                                              \
  X(16, 128, 1) X(16, 128, 2) X(16, 128, 4) X(16, 128, 8)              \
  X(8, 128, 1) X(8, 128, 2) X(8, 128, 4) X(8, 128, 8)                  \
  X(4, 128, 1) X(4, 128, 2) X(4, 128, 4) X(4, 128, 8)                  \
  X(2, 128, 1) X(2, 128, 2) X(2, 128, 4) X(2, 128, 8)                  \
  X(8, 64, 1) X(8, 64, 2) X(8, 64, 4)                                  \
  X(4, 64, 1) X(4, 64, 2) X(4, 64, 4)                                  \
  X(2, 64, 1) X(2, 64, 2) X(2, 64, 4)                                  \
  X(8, 32, 1) X(8, 32, 2) X(4, 32, 1) X(4, 32, 2) X(2, 32, 1) X(2, 32, 2)                  \
  X(kE4M3, 128, 1) X(kE4M3, 128, 2) X(kE4M3, 128, 4) X(kE4M3, 128, 8)  \
  X(kE4M3, 64, 1) X(kE4M3, 64, 2) X(kE4M3, 64, 4) X(kE4M3, 32, 1) X(kE4M3, 32, 2) \
  X(kSym8, 128, 1) X(kSym8, 128, 2) X(kSym8, 128, 4) X(kSym8, 128, 8)  \
  X(kSym8, 64, 1) X(kSym8, 64, 2) X(kSym8, 64, 4) X(kSym8, 32, 1) X(kSym8, 32, 2) \
  X(kE5M2, 128, 1) X(kE5M2, 128, 2) X(kE5M2, 128, 4) X(kE5M2, 128, 8)  \
  X(kE5M2, 64, 1) X(kE5M2, 64, 2) X(kE5M2, 64, 4) X(kE5M2, 32, 1) X(kE5M2, 32, 2) \
  X(kOaken, 128, 1) X(kOaken, 128, 2) X(kOaken, 128, 4) X(kOaken, 128, 8)

}  // namespace

bool decode_tm_supported(int bits, int group, int group_ratio, bool kpc) {
#define KVQ_X(B, G_, R) \
  if (bits == B && group == G_ && group_ratio == R) return true;
  if (kpc) {
    KVQ_TM_KPC_FORMATS(KVQ_X)
    return false;
  }
  KVQ_TM_FORMATS(KVQ_X)
#undef KVQ_X
  return false;
}

int decode_tm_ctas_per_sm(int bits, int group, int group_ratio, bool kpc) {
#define KVQ_X(B, G_, R) \
  if (bits == B && group == G_ && group_ratio == R) return TmCfg<B, G_, R, false>::MIN_CTAS;
#define KVQ_XK(B, G_, R) \
  if (bits == B && group == G_ && group_ratio == R) return TmCfg<B, G_, R, true>::MIN_CTAS;
  if (kpc) {
    KVQ_TM_KPC_FORMATS(KVQ_XK)
    return 0;
  }
  KVQ_TM_FORMATS(KVQ_X)
#undef KVQ_X
#undef KVQ_XK
  return 0;
}

cudaError_t launch_decode_tm(const DecodeArgs& a, const SegView& seg, cudaStream_t s) {
  const int bits = seg.bits, group = (seg.bits == 16) ? kHeadDim : seg.group;
  const int g = a.group_ratio;
#define KVQ_X(B, G_, R) \
  if (bits == B && group == G_ && g == R) return launch_tm<B, G_, R, false>(a, seg, s);
#define KVQ_XK(B, G_, R) \
  if (bits == B && group == G_ && g == R) return launch_tm<B, G_, R, true>(a, seg, s);
  if (seg.k_channels) {
    KVQ_TM_KPC_FORMATS(KVQ_XK)
    return cudaErrorInvalidValue;
  }
  KVQ_TM_FORMATS(KVQ_X)
#undef KVQ_X
#undef KVQ_XK
  return cudaErrorInvalidValue;
}

}  // namespace kvq
