// kvq_decode_common.cuh -- pieces shared by the two decode-attention kernels
// (the tokens-on-M kernel in kvq_decode_tm.cu and the 16-row kernel in
// kvq_decode.cu): operand packing, the persistent work-unit loop's
// bookkeeping, the in-CTA log-sum-exp merge of the four warps' partial
// results with its store to the output or to a split partial, and the
// sequence-length advance of a decode step.
#pragma once

#include <cuda_runtime.h>
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

struct SplitParams {
  DecodeArgs a;
  SegView seg;
};

// 2^n as an exact float constant (|n| <= 60).
__host__ __device__ constexpr float pow2f(int n) {
  return n >= 0 ? float(1ull << (n > 60 ? 60 : n)) : 1.0f / float(1ull << (-n > 60 ? 60 : -n));
}

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

// The query rows of KV head `kvh` of sequence `b` (g rows of head_dim) into
// shared memory as fp16, row h times 2^sh[h]: the kernels lift a query
// element by up to 2^QUP before it becomes an fp16 tensor-core operand, so
// sh[h] <= 0 is the largest value that keeps 2^QUP times the row's largest
// |q| below 2^15.  A row with max |q| < 2^(15 - QUP) has sh = 0 and is stored
// as it is (fp16 queries exactly; bf16 queries exactly for magnitudes in
// [2^-14, 65504]); a larger row loses only the bits of its elements that
// fall below 2^-24 after the shift.  The caller multiplies the row's scores
// by 2^-sh[h].  All threads of the CTA call this (rows are half-warps of
// threads 0 .. g * 16 - 1); qexp[h] receives sh[h].
template <int G, int QUP>
__device__ __forceinline__ void stage_queries(const DecodeArgs& a, int b, int kvh, __half* q_sm,
                                              int* qexp, int t) {
  static_assert(G * (kHeadDim / 8) <= kWarps * 32, "one thread per 8 query elements");
  const long long qbase = ((long long)b * a.q_heads + (long long)kvh * G) * kHeadDim;
  const bool mine = t < G * (kHeadDim / 8);
  uint4 raw = make_uint4(0u, 0u, 0u, 0u);
  if (mine) raw = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.q) + qbase)[t];
  // the row's largest magnitude as a bit pattern with the sign cleared (for
  // fp16 and bf16 alike, the order of these patterns is the order of the
  // magnitudes), over the thread's 8 elements, then its half-warp
  constexpr uint32_t kAbs = 0x7FFF7FFFu;
  uint32_t m = __vmaxu2(__vmaxu2(raw.x & kAbs, raw.y & kAbs), __vmaxu2(raw.z & kAbs, raw.w & kAbs));
  m = max(m & 0xFFFFu, m >> 16);
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 8));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 4));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  if (mine) {
    // floor(log2) of the largest magnitude (its biased exponent field; a
    // subnormal gives the smallest normal exponent, which is small enough)
    const int e = a.q_is_bf16 ? (int)(m >> 7) - 127 : (int)(m >> 10) - 15;
    const int sh = e >= 15 - QUP ? max(14 - QUP - e, -120) : 0;
    if (sh == 0 && !a.q_is_bf16) {
      reinterpret_cast<uint4*>(q_sm)[t] = raw;
    } else {
      const float sc = __int_as_float((127 + sh) << 23);  // 2^sh, exact
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      uint4 h16;
      uint32_t* hw = reinterpret_cast<uint32_t*>(&h16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 x;
        if (a.q_is_bf16)
          x = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
        else
          x = __half22float2(u32_as_h2(w[i]));
        hw[i] = h2_as_u32(__floats2half2_rn(x.x * sc, x.y * sc));
      }
      reinterpret_cast<uint4*>(q_sm)[t] = h16;
    }
    if ((t & 15) == 0) qexp[t >> 4] = sh;
  }
}

// 2^-sh for a row exponent of stage_queries (exact).
__device__ __forceinline__ float unshift(int sh) { return __int_as_float((127 - sh) << 23); }

// Token range [c0, c1) of split `split` of a sequence of length L: the splits
// are whole 32-token stages, so a stage's copy never runs past
// round_up(L, 32) <= max_tokens.
__device__ __forceinline__ void split_range(int L, int n_split, int split, int& c0, int& c1) {
  const int per_split = (L + n_split - 1) / n_split;
  const int chunk = ((per_split + 31) / 32) * 32;
  c0 = split * chunk;
  c1 = min(c0 + chunk, L);
}

// Log-sum-exp merge of the kWarps warps' partial results for the G heads of
// one (sequence, KV head, split) unit, then the store.  On entry (after a
// barrier) shared memory holds, per warp w and head h:
//   ms[w * 8 + h]  running max (log2 units), ls[w * 8 + h]  sum of weights,
//   os[(w * 8 + h) * D + d]  unnormalised output;
// a warp with ls == 0 saw no token.  `scratch` holds 8 * (kWarps + 2) floats.
// All 128 threads call this; thread t owns output dim t.
template <int G>
__device__ __forceinline__ void cta_merge_store(const DecodeArgs& a, const float* ms,
                                                const float* ls, const float* os, float* scratch,
                                                int b, int kvh, int part, int t) {
  constexpr int D = kHeadDim;
  float* wt = scratch;            // [8][kWarps] weights 2^(m_w - M)
  float* Mh = wt + 8 * kWarps;    // [8]
  float* Lh = Mh + 8;             // [8]
  if (t < G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      if (ls[w * 8 + t] > 0.f) M = fmaxf(M, ms[w * 8 + t]);
    float Ls = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float x = (ls[w * 8 + t] > 0.f) ? exp2f(ms[w * 8 + t] - M) : 0.f;
      wt[t * kWarps + w] = x;
      Ls += x * ls[w * 8 + t];
    }
    Mh[t] = M;
    Lh[t] = Ls;
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) O = fmaf(wt[h * kWarps + w], os[(w * 8 + h) * D + t], O);
    const float M = Mh[h], Ls = Lh[h];
    const long long bh = (long long)b * a.q_heads + (long long)kvh * G + h;
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

// Decode step: after a unit of sequence b finished (thread 0 calls this),
// the last of the sequence's `units_per_seq` units advances seq_lens[b] to
// `new_len`; every unit of b read the old length at its start.
__device__ __forceinline__ void advance_if_last(const DecodeArgs& a, const SegView& seg, int b,
                                                int units_per_seq, int new_len) {
  const unsigned prev = atomicAdd(&a.seq_cnt[b], 1u);
  if (prev == (unsigned)units_per_seq - 1) {
    const_cast<int32_t*>(seg.seq_lens)[b] = new_len;
    a.seq_cnt[b] = 0u;
  }
}

// Called once per CTA by thread 0 after its last unit: the last CTA to finish
// resets the work counters for the next launch on this workspace (nothing
// waits on them).
__device__ __forceinline__ void release_counters(uint32_t* counters) {
  __threadfence();
  const unsigned done = atomicAdd(&counters[1], 1u);
  if (done == gridDim.x - 1) {
    atomicExch(&counters[0], 0u);
    atomicExch(&counters[1], 0u);
    __threadfence();
  }
}

}  // namespace kvq
