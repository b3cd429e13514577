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
// scales and zero points reproducible bit for bit.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_internal.h"

namespace kvq {

// One thread holds 8 consecutive fp16 values of a token row; the G/8
// threads of a group are consecutive lanes (groups never straddle a row).
// Returns the packed codes of the 8 values (BITS bits each, element j at
// bit offset BITS*j) and the (scale, zero) half2 of the group.
// Two fp32 values to E4M3 codes, each rounded to the nearest E4M3 value
// (ties to even) and saturated at +-448; `lo` goes to the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int BITS, int G>
__device__ __forceinline__ void quantize8(const uint4 raw, uint32_t& codes_lo,
                                          uint32_t& codes_hi, uint32_t& meta) {
  static_assert(G % 8 == 0 && G >= 16 && G <= 256, "group size");
  const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
  float x[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h2[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
  if constexpr (BITS == kE4M3) {
    // FP8 E4M3 (the KV-cache page's FP8 KV cache, dynamic scale): s = max(
    // amax / 448, 1e-5) stored in fp16 rounded up, so |x / s| <= 448;
    // code = E4M3 of the fp32 quotient x / s; zero point 0.
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int off = 1; off < G / 8; off <<= 1)
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    float s32 = __fdiv_rn(amax, 448.0f);
    s32 = fmaxf(s32, 1e-5f);
    const __half s16 = __float2half_ru(s32);
    const float s = __half2float(s16);
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = e4m3x2(__fdiv_rn(x[2 * i], s), __fdiv_rn(x[2 * i + 1], s));
    codes_lo = c[0] | (c[1] << 16);
    codes_hi = c[2] | (c[3] << 16);
    const __half2 sz = __halves2half2(s16, __float2half_rn(0.f));
    meta = *reinterpret_cast<const uint32_t*>(&sz);
  } else {
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
      mn = fminf(mn, x[i]);
      mx = fmaxf(mx, x[i]);
    }
#pragma unroll
    for (int off = 1; off < G / 8; off <<= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    }
    constexpr float qmax = float((1 << code_bits(BITS)) - 1);
    float s32 = __fdiv_rn(__fsub_rn(mx, mn), qmax);
    s32 = fmaxf(s32, 1e-5f);
    const __half s16 = __float2half_ru(s32);
    const float s = __half2float(s16);
    float zf = __fadd_rn(rintf(__fdiv_rn(-mn, s)), 0.0f);
    zf = fminf(fmaxf(zf, -65504.0f), 65504.0f);
    const __half z16 = __float2half_rn(zf);
    const float z = __half2float(z16);

    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float v = __fadd_rn(rintf(__fdiv_rn(x[i], s)), z);
      v = fminf(fmaxf(v, 0.0f), qmax);
      c[i] = static_cast<uint32_t>(v);
    }
    if (code_bits(BITS) == 8) {
      codes_lo = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
      codes_hi = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
    } else {
      uint32_t w = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) w |= c[i] << (code_bits(BITS) * i);
      codes_lo = w;
      codes_hi = 0;
    }
    const __half2 sz = __halves2half2(s16, z16);
    meta = *reinterpret_cast<const uint32_t*>(&sz);
  }
}

// Quantize one 16-byte slice of a row and store it.  lane16 = index of the
// slice within the 128-value row (0..15); all 32 lanes of the warp must call
// this together (the group reduction uses warp shuffles); `active` false
// lanes load nothing and store nothing.
template <int BITS, int G>
__device__ __forceinline__ void quantize_slice(const __half* src_row, uint8_t* codes_row,
                                               uint8_t* meta_row, int lane16, bool active) {
  uint4 raw = make_uint4(0u, 0u, 0u, 0u);
  if (active) raw = __ldg(reinterpret_cast<const uint4*>(src_row) + lane16);
  uint32_t lo, hi, meta;
  quantize8<BITS, G>(raw, lo, hi, meta);
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
