// kvq_device.cuh -- device-side helpers of libkvq (sm_100a): PTX wrappers for
// the bulk-copy engine (TMA), mbarriers, warp-level tensor-core MMA, and the
// bit tricks that turn packed integer codes into exact fp16 values.
#pragma once

#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "kvq_internal.h"

namespace kvq {

constexpr int kHeadDim = 128;  // the head_dim the kernels are compiled for
constexpr int kTile = 16;      // tokens per warp step (one m16n8k16 K-extent)
constexpr int kWarps = kWarpsPerCta;  // consumer warps per decode CTA

// Device error flag bits (sticky word at the start of the decode workspace).
constexpr uint32_t kErrWaitTimeout = 1u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's generic-proxy accesses of shared memory before later
// async-proxy (bulk copy) accesses of it.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for a phase with an iteration limit: returns false if the limit ran
// out (the caller records an error and stops issuing work).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// ---------------------------------------------------------------- dependent launch
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization after this one may be scheduled once every CTA of this one
// has executed the trigger (or exited) ...
__device__ __forceinline__ void grid_dependents_may_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// ... and waits here until this one has completed and its memory operations
// are visible (a no-op for a kernel launched without that attribute).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- bulk copy
// One-dimensional bulk copy global -> shared, completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- tensor core
// D += A * B, m16n8k16, fp16 inputs, fp32 accumulate (register fragments).
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 tiles of 16-bit elements from shared memory, in the register
// layout of an m16n8k16 A operand: lane i supplies the address of row i % 8
// of tile i / 8 (16 contiguous bytes); tile t lands in r[t].
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// ---------------------------------------------------------------- bit casts
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}

// Two fp32 values in one 64-bit register pair (element 0 in the low half),
// for sm_100's packed f32x2 arithmetic: one instruction, both values, each
// rounded as the scalar fp32 operation would be.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
// ---------------------------------------------------------------- code -> fp16
// A b-bit code masked in place into mantissa bits 0..9 of a half is already
// an exact fp16 value: the subnormal code * 2^(e - 24), where e is the bit
// offset of the field (a code at bits 4..7 is code * 2^-20).  The tensor
// cores multiply fp16 subnormals exactly, so the conversion is one AND per
// pair of codes; the power-of-two factors are folded into the (exact,
// power-of-two scaled) query operand and into the output scale.
//
// Pairs of one token (K side): a 32-bit word of packed codes of consecutive
// dims yields half2 pairs (kPairs of them, covering kDims dims):
//   INT4 word (dims 0..7):  pair j (0..3) = dims (j, j + 4), e = 4 * (j & 1)
//   INT2 word (dims 0..15): pair j (0..7) = dims (j, j + 8), e = 2 * (j & 3)
//   INT8 word (dims 0..3):  pair j (0..1) = dims (j, j + 2), e = 0
//   FP16 word (dims 0..1):  the word itself, e = 24 (factor 1)
template <int BITS>
struct WordPairs;

template <>
struct WordPairs<4> {
  static constexpr int kPairs = 4, kDims = 8, kEmax = 4;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[4]) {
    const uint32_t w8 = w >> 8;
    p[0] = w & 0x000F000Fu;
    p[1] = w & 0x00F000F0u;
    p[2] = w8 & 0x000F000Fu;
    p[3] = w8 & 0x00F000F0u;
  }
  __host__ __device__ static constexpr int dim(int j, int e) { return j + 4 * e; }
  __host__ __device__ static constexpr int exp(int j) { return 4 * (j & 1); }
  // pair j alone (j a compile-time constant after unrolling)
  __device__ __forceinline__ static uint32_t one(uint32_t w, int j) {
    const uint32_t v = (j & 2) ? (w >> 8) : w;
    return v & ((j & 1) ? 0x00F000F0u : 0x000F000Fu);
  }
};

template <>
struct WordPairs<2> {
  static constexpr int kPairs = 8, kDims = 16, kEmax = 6;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[8]) {
    const uint32_t w8 = w >> 8;
    p[0] = w & 0x00030003u;
    p[1] = w & 0x000C000Cu;
    p[2] = w & 0x00300030u;
    p[3] = w & 0x00C000C0u;
    p[4] = w8 & 0x00030003u;
    p[5] = w8 & 0x000C000Cu;
    p[6] = w8 & 0x00300030u;
    p[7] = w8 & 0x00C000C0u;
  }
  __host__ __device__ static constexpr int dim(int j, int e) { return j + 8 * e; }
  __host__ __device__ static constexpr int exp(int j) { return 2 * (j & 3); }
  __device__ __forceinline__ static uint32_t one(uint32_t w, int j) {
    const uint32_t v = (j & 4) ? (w >> 8) : w;
    return v & (0x00030003u << (2 * (j & 3)));
  }
};

template <>
struct WordPairs<8> {
  static constexpr int kPairs = 2, kDims = 4, kEmax = 0;
  // bytes 1 and 3 are moved down by a byte permute with zero fill
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[2]) {
    p[0] = w & 0x00FF00FFu;
    p[1] = prmt(w, 0u, 0x4341u);
  }
  __host__ __device__ static constexpr int dim(int j, int e) { return j + 2 * e; }
  __host__ __device__ static constexpr int exp(int) { return 0; }
  __device__ __forceinline__ static uint32_t one(uint32_t w, int j) {
    return j ? prmt(w, 0u, 0x4341u) : (w & 0x00FF00FFu);
  }
};

template <>
struct WordPairs<16> {
  static constexpr int kPairs = 1, kDims = 2, kEmax = 24;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[1]) { p[0] = w; }
  __host__ __device__ static constexpr int dim(int, int e) { return e; }
  __host__ __device__ static constexpr int exp(int) { return 24; }
  __device__ __forceinline__ static uint32_t one(uint32_t w, int) { return w; }
};

// FP8 E5M2 word (dims 0..3): an E5M2 code is the high byte of the fp16 of
// the same value, so a byte permute with zero fill gives pair j = dims
// (2j, 2j + 1), the values themselves (factor 1, like raw fp16).
template <>
struct WordPairs<kE5M2> {
  static constexpr int kPairs = 2, kDims = 4, kEmax = 24;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[2]) {
    p[0] = prmt(w, 0u, 0x1404u);  // [0 w.b0 0 w.b1]
    p[1] = prmt(w, 0u, 0x3424u);  // [0 w.b2 0 w.b3]
  }
  __host__ __device__ static constexpr int dim(int j, int e) { return 2 * j + e; }
  __host__ __device__ static constexpr int exp(int) { return 24; }
  __device__ __forceinline__ static uint32_t one(uint32_t w, int j) {
    return prmt(w, 0u, j ? 0x3424u : 0x1404u);
  }
};

// Symmetric INT8 word (two's complement bytes): bit 7 of every byte flipped
// gives the offset-binary code c + 128, read like the 8-bit integer codes
// with a zero point of 128.
template <>
struct WordPairs<kSym8> {
  static constexpr int kPairs = 2, kDims = 4, kEmax = 0;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[2]) {
    p[0] = (w & 0x00FF00FFu) ^ 0x00800080u;
    p[1] = prmt(w, 0u, 0x4341u) ^ 0x00800080u;
  }
  __host__ __device__ static constexpr int dim(int j, int e) { return j + 2 * e; }
  __host__ __device__ static constexpr int exp(int) { return 0; }
  __device__ __forceinline__ static uint32_t one(uint32_t w, int j) {
    return (j ? prmt(w, 0u, 0x4341u) : (w & 0x00FF00FFu)) ^ 0x00800080u;
  }
};

// Two E4M3 codes (low byte, high byte) to an fp16 pair (low half, high
// half); exact, every E4M3 value being an fp16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t v16) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)v16));
  return r;
}

// FP8 E4M3 word (dims 0..3): pair j = dims (2j, 2j + 1), the values
// themselves (factor 1, like raw fp16).
template <>
struct WordPairs<kE4M3> {
  static constexpr int kPairs = 2, kDims = 4, kEmax = 24;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[2]) {
    p[0] = e4m3x2_to_h2(w & 0xFFFFu);
    p[1] = e4m3x2_to_h2(w >> 16);
  }
  __host__ __device__ static constexpr int dim(int j, int e) { return 2 * j + e; }
  __host__ __device__ static constexpr int exp(int) { return 24; }
  __device__ __forceinline__ static uint32_t one(uint32_t w, int j) {
    return e4m3x2_to_h2(j ? (w >> 16) : (w & 0xFFFFu));
  }
};

// The Oaken codec's dense part is 4-bit codes packed like INT4.
template <>
struct WordPairs<kOaken> : WordPairs<4> {};

// Pairs across two tokens (V side): words a (token A) and b (token B) hold
// the same dims; out[i] = half2(code_A[dim i], code_B[dim i]) for the dims of
// the word in order, with the subnormal exponent exp(i).
template <int BITS>
struct CrossPairs;

template <>
struct CrossPairs<4> {
  static constexpr int kOut = 8;  // dims per 32-bit word
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[8]) {
    const uint32_t x = prmt(a, b, 0x5410u);  // [a.b0 a.b1 b.b0 b.b1]
    const uint32_t y = prmt(a, b, 0x7632u);  // [a.b2 a.b3 b.b2 b.b3]
    const uint32_t x8 = x >> 8, y8 = y >> 8;
    o[0] = x & 0x000F000Fu;
    o[1] = x & 0x00F000F0u;
    o[2] = x8 & 0x000F000Fu;
    o[3] = x8 & 0x00F000F0u;
    o[4] = y & 0x000F000Fu;
    o[5] = y & 0x00F000F0u;
    o[6] = y8 & 0x000F000Fu;
    o[7] = y8 & 0x00F000F0u;
  }
  __host__ __device__ static constexpr int exp(int i) { return 4 * (i & 1); }
};

template <>
struct CrossPairs<kOaken> : CrossPairs<4> {};

template <>
struct CrossPairs<2> {
  static constexpr int kOut = 16;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[16]) {
    const uint32_t x = prmt(a, b, 0x5410u);
    const uint32_t y = prmt(a, b, 0x7632u);
    const uint32_t v[4] = {x, x >> 8, y, y >> 8};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[4 * i + 0] = v[i] & 0x00030003u;
      o[4 * i + 1] = v[i] & 0x000C000Cu;
      o[4 * i + 2] = v[i] & 0x00300030u;
      o[4 * i + 3] = v[i] & 0x00C000C0u;
    }
  }
  __host__ __device__ static constexpr int exp(int i) { return 2 * (i & 3); }
};

template <>
struct CrossPairs<8> {
  static constexpr int kOut = 4;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[4]) {
    const uint32_t x = prmt(a, b, 0x5410u);  // [a.b0 a.b1 b.b0 b.b1]
    const uint32_t y = prmt(a, b, 0x7632u);  // [a.b2 a.b3 b.b2 b.b3]
    o[0] = x & 0x00FF00FFu;
    o[1] = prmt(x, 0u, 0x4341u);              // [x.b1 0 x.b3 0]
    o[2] = y & 0x00FF00FFu;
    o[3] = prmt(y, 0u, 0x4341u);
  }
  __host__ __device__ static constexpr int exp(int) { return 0; }
};

template <>
struct CrossPairs<kSym8> {
  static constexpr int kOut = 4;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[4]) {
    const uint32_t x = prmt(a, b, 0x5410u);  // [a.b0 a.b1 b.b0 b.b1]
    const uint32_t y = prmt(a, b, 0x7632u);  // [a.b2 a.b3 b.b2 b.b3]
    o[0] = (x & 0x00FF00FFu) ^ 0x00800080u;  // offset binary, as in WordPairs<kSym8>
    o[1] = prmt(x, 0u, 0x4341u) ^ 0x00800080u;
    o[2] = (y & 0x00FF00FFu) ^ 0x00800080u;
    o[3] = prmt(y, 0u, 0x4341u) ^ 0x00800080u;
  }
  __host__ __device__ static constexpr int exp(int) { return 0; }
};

template <>
struct CrossPairs<kE5M2> {
  static constexpr int kOut = 4;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[4]) {
    const uint32_t x = prmt(a, b, 0x5140u);  // [a.b0 b.b0 a.b1 b.b1]
    const uint32_t y = prmt(a, b, 0x7362u);  // [a.b2 b.b2 a.b3 b.b3]
    o[0] = prmt(x, 0u, 0x1404u);              // [0 a.b0 0 b.b0]: fp16 of the codes
    o[1] = prmt(x, 0u, 0x3424u);
    o[2] = prmt(y, 0u, 0x1404u);
    o[3] = prmt(y, 0u, 0x3424u);
  }
  __host__ __device__ static constexpr int exp(int) { return 24; }
};

template <>
struct CrossPairs<kE4M3> {
  static constexpr int kOut = 4;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[4]) {
    const uint32_t x = prmt(a, b, 0x5140u);  // [a.b0 b.b0 a.b1 b.b1]
    const uint32_t y = prmt(a, b, 0x7362u);  // [a.b2 b.b2 a.b3 b.b3]
    o[0] = e4m3x2_to_h2(x & 0xFFFFu);
    o[1] = e4m3x2_to_h2(x >> 16);
    o[2] = e4m3x2_to_h2(y & 0xFFFFu);
    o[3] = e4m3x2_to_h2(y >> 16);
  }
  __host__ __device__ static constexpr int exp(int) { return 24; }
};

template <>
struct CrossPairs<16> {
  static constexpr int kOut = 2;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[2]) {
    o[0] = prmt(a, b, 0x5410u);
    o[1] = prmt(a, b, 0x7632u);
  }
  __host__ __device__ static constexpr int exp(int) { return 24; }
};

// 2^x for the softmax (hardware approximation, relative error ~2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace kvq
