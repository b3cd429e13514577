// kvq_quant_core.cuh -- the per-thread core of group quantization, shared
// by the quantize-on-append kernels and the chunk reorder kernel.
//
// Quantization (Cocktail page, section 3.2.2: quant(x) = round(x/s) + z, one
// s and z per group; scale = (max - min) / (2^bits - 1), static-quantization
// page section 2.1; s floored at 1e-5, KV-cache page troubleshooting):
//   s32 = max((mx - mn) / qmax, 1e-5);  s = fp16 value of s32 rounded up;
//   z = rint(-mn / s) + 0 (clamped to +-65504, fp16);
//   code = clamp(rint(x / s) + z, 0, qmax).
// Every step is one IEEE fp32 operation with round-to-nearest-even (explicit
// intrinsics, so no contraction can change a result), which makes codes,
// scales and zero points reproducible bit for bit.  The per-element division
// by s is a correction step on a product with RN(1/s) that returns the IEEE
// quotient exactly (div_rn below), and the rounding and clamping of the code
// use an equivalent order that needs no conversion instruction.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

// Two fp32 values to E4M3 codes, each rounded to the nearest E4M3 value
// (ties to even) and saturated at +-448; `lo` goes to the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// The same for E5M2 codes, saturated at +-57344.
__device__ __forceinline__ uint32_t e5m2x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// x / d rounded to nearest-even fp32 (the IEEE quotient), given r = RN(1/d):
// q0 = RN(x r) approximates x / d within one ulp, the remainder x - q0 d is
// exact in one fma, and RN(q0 + (x - q0 d) r) is the correctly rounded
// quotient (Markstein's theorem: P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990).  Used with fp16-valued x and d, where no step under- or overflows;
// the identity with IEEE division holds for every pair of 11-bit
// significands, which covers every fp16 x and d up to a power of two.  A zero
// quotient comes out +0 whatever the sign of x.
__device__ __forceinline__ float div_rn(float x, float d, float r) {
  const float q0 = __fmul_rn(x, r);
  const float e = __fmaf_rn(-q0, d, x);
  return __fmaf_rn(e, r, q0);
}

// div_rn on two values at once, each with its own divisor: x2 = (x0, x1),
// nd2 = (-d0, -d1), r2 = (r0, r1) (q0 * -d + x is the same fma as -q0 * d + x).
__device__ __forceinline__ uint64_t div_rn2(uint64_t x2, uint64_t nd2, uint64_t r2) {
  const uint64_t q0 = f2_mul(x2, r2);
  const uint64_t e = f2_fma(q0, nd2, x2);
  return f2_fma(e, r2, q0);
}

// Packed code words of NV values of a BITS-bit format (at least one word).
template <int BITS, int NV>
__host__ __device__ constexpr int code_words() {
  return (NV * code_bits(BITS) + 31) / 32;
}

// Pack codes into words, element j at bit offset CB * j.  t[i] holds the
// codes of elements i (low lane) and i + NV / 2 (high lane) as fp32 integers
// in [0, 2^CB).  Adjacent registers are merged lane by lane, c_even +
// 2^(width) * c_odd, an exact fp32 fma while values stay below 2^24, until a
// lane holds 16 bits of codes (8 for 8 values of 2 bits); adding 1.5 * 2^23
// then puts them in the low mantissa bits, and byte permutes assemble the
// words.
template <int CB, int NV>
__device__ __forceinline__ void pack_codes(uint64_t (&t)[NV / 2], uint32_t* w) {
  constexpr int NH = NV / 2;
  constexpr int L = (16 / CB < NH) ? 16 / CB : NH;  // codes per lane chunk
  constexpr int LEVELS = L == 1 ? 0 : L == 2 ? 1 : L == 4 ? 2 : 3;
  constexpr int N = NH / L;                          // chunk registers
#pragma unroll
  for (int lev = 0; lev < LEVELS; ++lev) {
    const float mult = float(1u << (CB << lev));
    const uint64_t m = f2_pack(mult, mult);
#pragma unroll
    for (int j = 0; j < (NH >> (lev + 1)); ++j) t[j] = f2_fma(t[2 * j + 1], m, t[2 * j]);
  }
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint64_t m2 = f2_pack(kMagic, kMagic);
  uint32_t c[2 * N];  // chunks in element order: the low lanes, then the high lanes
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float2 f = f2_unpack(f2_add(t[j], m2));
    c[j] = __float_as_uint(f.x);
    c[N + j] = __float_as_uint(f.y);
  }
  if constexpr (CB * L == 16) {
#pragma unroll
    for (int k = 0; k < N; ++k) w[k] = __byte_perm(c[2 * k], c[2 * k + 1], 0x5410);
  } else {
    static_assert(CB * L == 8 && N == 1, "8-bit chunks only for 8 values of 2 bits");
    w[0] = __byte_perm(c[0], c[1], 0x0040) & 0xFFFFu;
  }
}

// A pair of 16-bit input values in one 32-bit word: binary16 (BF false) or
// bfloat16 (BF true).  Both widen to fp32 exactly, and their pairwise min and
// max are exact; the sign bit is bit 15 of each half in both formats.
template <bool BF>
struct InPair {
  static __device__ __forceinline__ float2 widen(uint32_t w) {
    if constexpr (BF)
      return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    else
      return __half22float2(u32_as_h2(w));
  }
  static __device__ __forceinline__ uint32_t min2(uint32_t a, uint32_t b) {
    if constexpr (BF) {
      const __nv_bfloat162 r = __hmin2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                       *reinterpret_cast<const __nv_bfloat162*>(&b));
      return *reinterpret_cast<const uint32_t*>(&r);
    } else {
      return h2_as_u32(__hmin2(u32_as_h2(a), u32_as_h2(b)));
    }
  }
  static __device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b) {
    if constexpr (BF) {
      const __nv_bfloat162 r = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                                       *reinterpret_cast<const __nv_bfloat162*>(&b));
      return *reinterpret_cast<const uint32_t*>(&r);
    } else {
      return h2_as_u32(__hmax2(u32_as_h2(a), u32_as_h2(b)));
    }
  }
  static __device__ __forceinline__ uint32_t swap(uint32_t a) { return __byte_perm(a, 0, 0x1032); }
};

// One thread holds NV (8, 16 or 32) consecutive 16-bit values of a token row
// (fp16, or bf16 with BF); the G / NV threads of a group are consecutive lanes
// (groups never straddle a row).  Produces the packed codes of the NV values
// (BITS bits each, element j at bit offset BITS * j) and the (scale, zero)
// half2 of the group.  Every value is widened to fp32 exactly, so both input
// types go through the same fp32 steps.
template <int BITS, int G, int NV, bool BF = false>
__device__ __forceinline__ void quantize_vals(const uint4 (&raw)[NV / 8],
                                              uint32_t (&codes)[code_words<BITS, NV>()],
                                              uint32_t& meta) {
  static_assert(NV == 8 || NV == 16 || NV == 32, "values per thread");
  static_assert(G % NV == 0 && G / NV <= 32 && G <= kHeadDim, "group size");
  using P = InPair<BF>;
  constexpr int NH = NV / 2;
  constexpr int GL = G / NV;  // lanes per group
  const uint32_t* w2 = reinterpret_cast<const uint32_t*>(&raw[0]);
  float x[NV];
#pragma unroll
  for (int i = 0; i < NH; ++i) {
    const float2 f = P::widen(w2[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
  if constexpr (BITS == kE4M3 || BITS == kE5M2 || BITS == kSym8) {
    // the group's |max|, taken on the 16-bit values (exact): clearing the
    // sign bits is |.| in both formats
    uint32_t am = w2[0] & 0x7FFF7FFFu;
#pragma unroll
    for (int i = 1; i < NH; ++i) am = P::max2(am, w2[i] & 0x7FFF7FFFu);
    am = P::max2(am, P::swap(am));
#pragma unroll
    for (int off = 1; off < GL; off <<= 1)
      am = P::max2(am, __shfl_xor_sync(0xffffffffu, am, off));
    const float amax = P::widen(am).x;
    if constexpr (BITS == kSym8) {
      // Symmetric INT8 (the KV-cache page's INT8 item): s = max(amax / 127,
      // 1e-5) stored in fp16 rounded up, so |x / s| <= 127 and the clamp to
      // [-128, 127] never acts; code = rint(x / s) as a two's complement
      // byte; zero point 0.  The codes go through the integer packing as
      // c + 128 in [1, 255]; flipping bit 7 of every byte then gives c.
      constexpr float kInv127 = 1.0f / 127.0f;
      constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
      const float s32 = fmaxf(div_rn(amax, 127.0f, kInv127), 1e-5f);
      const __half s16 = __float2half_ru(s32);
      const float s = __half2float(s16);
      const float r = __frcp_rn(s);
      const uint64_t r2 = f2_pack(r, r), nd2 = f2_pack(-s, -s);
      const uint64_t m2 = f2_pack(kMagic, kMagic);
      const uint64_t om2 = f2_pack(128.0f - kMagic, 128.0f - kMagic);
      uint64_t t[NH];  // pair i holds elements i and i + NH
#pragma unroll
      for (int i = 0; i < NH; ++i)
        t[i] = f2_add(f2_add(div_rn2(f2_pack(x[i], x[i + NH]), nd2, r2), m2), om2);
      pack_codes<8, NV>(t, codes);
#pragma unroll
      for (int i = 0; i < code_words<BITS, NV>(); ++i) codes[i] ^= 0x80808080u;
      meta = h2_as_u32(__halves2half2(s16, __float2half_rn(0.f)));
      return;
    }
    // FP8 (the KV-cache page's FP8 KV cache, dynamic scale): s = max(amax /
    // F, 1e-5) stored in fp16 rounded up, so |x / s| <= F, the format's
    // largest finite value (E4M3 448, E5M2 57344); code = the FP8 value of
    // the fp32 quotient x / s; zero point 0.
    constexpr float kMaxF = BITS == kE4M3 ? 448.0f : 57344.0f;
    constexpr float kInvMax = 1.0f / kMaxF;
    const float s32 = fmaxf(div_rn(amax, kMaxF, kInvMax), 1e-5f);
    const __half s16 = __float2half_ru(s32);
    const float s = __half2float(s16);
    const float r = __frcp_rn(s);
    const uint64_t r2 = f2_pack(r, r), nd2 = f2_pack(-s, -s);
    uint32_t c[NH];
#pragma unroll
    for (int i = 0; i < NH; ++i) {
      const float2 q = f2_unpack(div_rn2(f2_pack(x[2 * i], x[2 * i + 1]), nd2, r2));
      if constexpr (BITS == kE4M3)
        c[i] = e4m3x2(copysignf(q.x, x[2 * i]), copysignf(q.y, x[2 * i + 1]));
      else
        c[i] = e5m2x2(copysignf(q.x, x[2 * i]), copysignf(q.y, x[2 * i + 1]));
    }
#pragma unroll
    for (int i = 0; i < NH / 2; ++i) codes[i] = __byte_perm(c[2 * i], c[2 * i + 1], 0x5410);
    meta = h2_as_u32(__halves2half2(s16, __float2half_rn(0.f)));
  } else {
    // group (min, -max) as one 16-bit pair: one shuffle and one min per step
    uint32_t lo2 = w2[0], hi2 = w2[0];
#pragma unroll
    for (int i = 1; i < NH; ++i) {
      lo2 = P::min2(lo2, w2[i]);
      hi2 = P::max2(hi2, w2[i]);
    }
    lo2 = P::min2(lo2, P::swap(lo2));
    hi2 = P::max2(hi2, P::swap(hi2)) ^ 0x80008000u;  // -max in both halves
    uint32_t mm = __byte_perm(lo2, hi2, 0x7610);      // (min, -max)
#pragma unroll
    for (int off = 1; off < GL; off <<= 1)
      mm = P::min2(mm, __shfl_xor_sync(0xffffffffu, mm, off));
    const float2 mmf = P::widen(mm);
    const float mn = mmf.x, mx = -mmf.y;
    constexpr int qmax_i = (1 << code_bits(BITS)) - 1;
    constexpr float qmax = float(qmax_i);
    constexpr float kInvQmax = 1.0f / qmax;
    const float s32 = fmaxf(div_rn(__fsub_rn(mx, mn), qmax, kInvQmax), 1e-5f);
    const __half s16 = __float2half_ru(s32);
    const float s = __half2float(s16);
    const float r = __frcp_rn(s);
    float zf = __fadd_rn(rintf(div_rn(-mn, s, r)), 0.0f);
    zf = fminf(fmaxf(zf, -65504.0f), 65504.0f);
    const __half z16 = __float2half_rn(zf);
    const float z = __half2float(z16);  // an integer
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: adding it rounds |v| < 2^22 to an integer
    // pair i of the packed arithmetic holds elements i and i + NH
    const uint64_t r2 = f2_pack(r, r), nd2 = f2_pack(-s, -s);
    const uint64_t m2 = f2_pack(kMagic, kMagic);
    const float zm = z - kMagic;  // exact: an integer of magnitude below 2^24
    const uint64_t zm2 = f2_pack(zm, zm);
    uint64_t t[NH];  // codes as fp32 integers
    // code = clamp(rint(x / s) + z, 0, qmax); (q + 1.5 * 2^23) + (z - 1.5 *
    // 2^23) is rint(q) + z exactly for |q| < 2^22.
    const float top = __fadd_rn(__fadd_rn(div_rn(mx, s, r), kMagic), zm);
    if (__all_sync(0xffffffffu, fabsf(zf) <= 2048.0f && top <= qmax)) {
      // z is exact in fp16 and equals -rint(RN(mn / s)) (rounding and rint
      // are monotone and odd-symmetric), so every code of the group is >= 0,
      // the group's largest code (at its max) is <= qmax, and every quotient
      // lies within 2048 + qmax + 2 of zero: no clamp is needed.
#pragma unroll
      for (int i = 0; i < NH; ++i)
        t[i] = f2_add(f2_add(div_rn2(f2_pack(x[i], x[i + NH]), nd2, r2), m2), zm2);
    } else {
      // Clamping the quotient to [-z, qmax - z] first gives the same code (z
      // is an integer: a quotient below -z rounds to at most -z, one above
      // qmax - z to at least qmax - z) and bounds it well inside +-2^22.
      const float lo = -z, hi = __fadd_rn(qmax, -z);
#pragma unroll
      for (int i = 0; i < NH; ++i) {
        const float2 q = f2_unpack(div_rn2(f2_pack(x[i], x[i + NH]), nd2, r2));
        const uint64_t qc = f2_pack(fminf(fmaxf(q.x, lo), hi), fminf(fmaxf(q.y, lo), hi));
        t[i] = f2_add(f2_add(qc, m2), zm2);
      }
    }
    pack_codes<code_bits(BITS), NV>(t, codes);
    meta = h2_as_u32(__halves2half2(s16, z16));
  }
}

// quantize_vals for 8 values per thread: codes in (codes_lo, codes_hi).
template <int BITS, int G, bool BF = false>
__device__ __forceinline__ void quantize8(const uint4 raw, uint32_t& codes_lo,
                                          uint32_t& codes_hi, uint32_t& meta) {
  const uint4 r[1] = {raw};
  uint32_t w[code_words<BITS, 8>()];
  quantize_vals<BITS, G, 8, BF>(r, w, meta);
  codes_lo = w[0];
  if constexpr (code_words<BITS, 8>() > 1)
    codes_hi = w[1];
  else
    codes_hi = 0;
}

// ---- the bulk kernels' shared-memory ring (prefill quantize, chunk
// reorder): per-lane cp.async copies of 16 bytes, committed in groups

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Ring offset of 16-byte chunk k (0..15) of row ri of a unit: position
// k ^ (bit 3 of k) ^ (6 for odd rows) within the row.  16-byte shared-memory
// accesses are served eight lanes (two rows) at a time; for a copy step
// (lane (ri, li) moves chunk 4c + li) and for a read step (lane (ri, li)
// reads chunk 4li + c) the eight chunks of each such pair of rows then fall
// in eight different groups of four banks: no bank conflicts.
__device__ __forceinline__ uint32_t bulk_slot_off(int ri, int k) {
  return (uint32_t)(ri * (kHeadDim * 2) + ((k ^ ((k >> 3) & 1) ^ ((ri & 1) * 6)) * 16));
}


// Quantize one 16-byte slice of a row (fp16 values, or bf16 with BF) and
// store it.  lane16 = index of the slice within the 128-value row (0..15); all 32 lanes of the warp must call
// this together (the group reduction uses warp shuffles); `active` false
// lanes load nothing and store nothing.
template <int BITS, int G, bool BF = false>
__device__ __forceinline__ void quantize_slice(const __half* src_row, uint8_t* codes_row,
                                               uint8_t* meta_row, int lane16, bool active) {
  uint4 raw = make_uint4(0u, 0u, 0u, 0u);
  if (active) raw = __ldg(reinterpret_cast<const uint4*>(src_row) + lane16);
  uint32_t lo, hi, meta;
  quantize8<BITS, G, BF>(raw, lo, hi, meta);
  if (!active) return;
  if (code_bits(BITS) == 8) {
    reinterpret_cast<uint2*>(codes_row)[lane16] = make_uint2(lo, hi);
  } else if (BITS == 4) {
    reinterpret_cast<uint32_t*>(codes_row)[lane16] = lo;
  } else {
    reinterpret_cast<uint16_t*>(codes_row)[lane16] = static_cast<uint16_t>(lo);
  }
  if ((lane16 % (G / 8)) == 0) reinterpret_cast<uint32_t*>(meta_row)[lane16 / (G / 8)] = meta;
}

}  // namespace kvq
