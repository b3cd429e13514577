// kvq_device.cuh -- device-side helpers of libkvq (sm_100a): PTX wrappers for
// the bulk-copy engine (TMA), mbarriers, warp-level tensor-core MMA, and the
// bit tricks that turn packed integer codes into exact fp16 values.
#pragma once

#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace kvq {

constexpr int kHeadDim = 128;  // head_dim supported by this build
constexpr int kTile = 16;      // tokens per warp step (one m16n8k16 K-extent)
constexpr int kWarps = 4;      // consumer warps per decode CTA

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

// ---------------------------------------------------------------- bit casts
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) {
  return *reinterpret_cast<__half2*>(&u);
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
// (x & mask) | base in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t x, uint32_t mask, uint32_t base) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(mask), "r"(base));
  return r;
}
// Exact fp16 subtraction of the conversion offset (both halves).
__device__ __forceinline__ uint32_t hsub_u32(uint32_t x, uint32_t off) {
  return h2_as_u32(__hsub2(u32_as_h2(x), u32_as_h2(off)));
}

// ---------------------------------------------------------------- code -> fp16
// Integer codes become exact fp16 values by writing them into the mantissa
// of a power of two whose unit in the last place is 1 for that bit field
// (bits 0-1 of a half: 1024 = 0x6400; bits 2-3: 256 = 0x5C00; bits 4-5:
// 64 = 0x5400; bits 6-7: 16 = 0x4C00), then subtracting the power of two,
// which is exact.
//
// Pairs of one token (K side): a 32-bit word of packed codes of consecutive
// dims yields half2 pairs; the pair -> dim order is fixed by
//   INT4 word (dims 0..7):  pair j (0..3) = dims (j, j + 4)
//   INT2 word (dims 0..15): pair j (0..7) = dims (j, j + 8)
//   INT8 word (dims 0..3):  pair j (0..1) = dims (2j, 2j + 1)
//   FP16 word (dims 0..1):  the word itself
template <int BITS>
struct WordPairs;

template <>
struct WordPairs<4> {
  static constexpr int kPairs = 4, kDims = 8;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[4]) {
    const uint32_t w8 = w >> 8;
    p[0] = hsub_u32(and_or(w, 0x000F000Fu, 0x64006400u), 0x64006400u);
    p[1] = hsub_u32(and_or(w, 0x00F000F0u, 0x54005400u), 0x54005400u);
    p[2] = hsub_u32(and_or(w8, 0x000F000Fu, 0x64006400u), 0x64006400u);
    p[3] = hsub_u32(and_or(w8, 0x00F000F0u, 0x54005400u), 0x54005400u);
  }
  __device__ __forceinline__ static int dim(int j, int e) { return j + 4 * e; }
};

template <>
struct WordPairs<2> {
  static constexpr int kPairs = 8, kDims = 16;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[8]) {
    const uint32_t w8 = w >> 8;
    p[0] = hsub_u32(and_or(w, 0x00030003u, 0x64006400u), 0x64006400u);
    p[1] = hsub_u32(and_or(w, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u);
    p[2] = hsub_u32(and_or(w, 0x00300030u, 0x54005400u), 0x54005400u);
    p[3] = hsub_u32(and_or(w, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u);
    p[4] = hsub_u32(and_or(w8, 0x00030003u, 0x64006400u), 0x64006400u);
    p[5] = hsub_u32(and_or(w8, 0x000C000Cu, 0x5C005C00u), 0x5C005C00u);
    p[6] = hsub_u32(and_or(w8, 0x00300030u, 0x54005400u), 0x54005400u);
    p[7] = hsub_u32(and_or(w8, 0x00C000C0u, 0x4C004C00u), 0x4C004C00u);
  }
  __device__ __forceinline__ static int dim(int j, int e) { return j + 8 * e; }
};

template <>
struct WordPairs<8> {
  static constexpr int kPairs = 2, kDims = 4;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[2]) {
    p[0] = hsub_u32(prmt(w, 0x64646464u, 0x4140u), 0x64006400u);
    p[1] = hsub_u32(prmt(w, 0x64646464u, 0x4342u), 0x64006400u);
  }
  __device__ __forceinline__ static int dim(int j, int e) { return 2 * j + e; }
};

template <>
struct WordPairs<16> {
  static constexpr int kPairs = 1, kDims = 2;
  __device__ __forceinline__ static void run(uint32_t w, uint32_t (&p)[1]) { p[0] = w; }
  __device__ __forceinline__ static int dim(int j, int e) { return e; }
};

// Pairs across two tokens (V side): words a (token A) and b (token B) hold
// the same dims; out[i] = half2(code_A[dim i], code_B[dim i]) for the dims of
// the low 16 bits (INT4: 4 dims, INT2: 8 dims, INT8: 2 dims, FP16: 1 dim)
// and of the high 16 bits (the same count again), in dim order.
template <int BITS>
struct CrossPairs;

template <>
struct CrossPairs<4> {
  static constexpr int kOut = 8;  // dims per 32-bit word
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[8]) {
    uint32_t x = prmt(a, b, 0x5410u);  // [a.b0 a.b1 b.b0 b.b1]
    uint32_t y = prmt(a, b, 0x7632u);  // [a.b2 a.b3 b.b2 b.b3]
    uint32_t x8 = x >> 8, y8 = y >> 8;
    o[0] = hsub_u32(and_or(x, 0x000F000Fu, 0x64006400u), 0x64006400u);
    o[1] = hsub_u32(and_or(x, 0x00F000F0u, 0x54005400u), 0x54005400u);
    o[2] = hsub_u32(and_or(x8, 0x000F000Fu, 0x64006400u), 0x64006400u);
    o[3] = hsub_u32(and_or(x8, 0x00F000F0u, 0x54005400u), 0x54005400u);
    o[4] = hsub_u32(and_or(y, 0x000F000Fu, 0x64006400u), 0x64006400u);
    o[5] = hsub_u32(and_or(y, 0x00F000F0u, 0x54005400u), 0x54005400u);
    o[6] = hsub_u32(and_or(y8, 0x000F000Fu, 0x64006400u), 0x64006400u);
    o[7] = hsub_u32(and_or(y8, 0x00F000F0u, 0x54005400u), 0x54005400u);
  }
};

template <>
struct CrossPairs<2> {
  static constexpr int kOut = 16;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[16]) {
    uint32_t x = prmt(a, b, 0x5410u);
    uint32_t y = prmt(a, b, 0x7632u);
    uint32_t v[4] = {x, x >> 8, y, y >> 8};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[4 * i + 0] = hsub_u32(and_or(v[i], 0x00030003u, 0x64006400u), 0x64006400u);
      o[4 * i + 1] = hsub_u32(and_or(v[i], 0x000C000Cu, 0x5C005C00u), 0x5C005C00u);
      o[4 * i + 2] = hsub_u32(and_or(v[i], 0x00300030u, 0x54005400u), 0x54005400u);
      o[4 * i + 3] = hsub_u32(and_or(v[i], 0x00C000C0u, 0x4C004C00u), 0x4C004C00u);
    }
  }
};

template <>
struct CrossPairs<8> {
  static constexpr int kOut = 4;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[4]) {
    uint32_t lo = prmt(a, b, 0x5140u);  // [a.b0 b.b0 a.b1 b.b1]
    uint32_t hi = prmt(a, b, 0x7362u);  // [a.b2 b.b2 a.b3 b.b3]
    o[0] = hsub_u32(prmt(lo, 0x64646464u, 0x4140u), 0x64006400u);
    o[1] = hsub_u32(prmt(lo, 0x64646464u, 0x4342u), 0x64006400u);
    o[2] = hsub_u32(prmt(hi, 0x64646464u, 0x4140u), 0x64006400u);
    o[3] = hsub_u32(prmt(hi, 0x64646464u, 0x4342u), 0x64006400u);
  }
};

template <>
struct CrossPairs<16> {
  static constexpr int kOut = 2;
  __device__ __forceinline__ static void run(uint32_t a, uint32_t b, uint32_t (&o)[2]) {
    o[0] = prmt(a, b, 0x5410u);
    o[1] = prmt(a, b, 0x7632u);
  }
};

}  // namespace kvq
