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
// shared memory as fp16.  bf16 queries are used through fp16, which is exact
// for |q| in [2^-14, 65504].  Threads 0 .. g * 16 - 1 take part.
template <int G>
__device__ __forceinline__ void stage_queries(const DecodeArgs& a, int b, int kvh, __half* q_sm,
                                              int t) {
  const long long qbase = ((long long)b * a.q_heads + (long long)kvh * G) * kHeadDim;
  if (t < G * (kHeadDim / 8)) {
    const uint4 raw = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.q) + qbase)[t];
    uint4 h16 = raw;
    if (a.q_is_bf16) {
      const __nv_bfloat162* bb = reinterpret_cast<const __nv_bfloat162*>(&raw);
      __half2* hh = reinterpret_cast<__half2*>(&h16);
#pragma unroll
      for (int i = 0; i < 4; ++i) hh[i] = __float22half2_rn(__bfloat1622float2(bb[i]));
    }
    reinterpret_cast<uint4*>(q_sm)[t] = h16;
  }
}

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
