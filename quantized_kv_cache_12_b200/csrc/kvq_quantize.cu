// kvq_quantize.cu -- quantize-on-write of new K/V tokens into the packed
// cache (Cocktail page 3.2.2 formula; Oaken page 3.2.3 pipeline, where the
// quantizer sits inside the memory write).
//
// Layout of a thread's work: a token row of 128 16-bit values (fp16, or bf16
// through the BF template flag) is 16 lanes x 16 bytes; a warp quantizes two
// rows per step.  The row's groups are reduced
// with warp shuffles, codes are packed in registers and written with one
// 2/4/8-byte store per lane, and the group leader writes (scale, zero).
#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_bulk.cuh"
#include "kvq_quant_core.cuh"

namespace kvq {

namespace {

struct RowRef {
  const __half* src;
  uint8_t* codes;
  uint8_t* meta;
  bool active;
};

// Row r of the 2 * batch * kv_heads * n_new input rows (K rows first).
template <int BITS, int G>
__device__ __forceinline__ RowRef locate_row(const QuantArgs& a, long long r, int base_pos) {
  const long long per = (long long)a.batch * a.kv_heads * a.n_new;
  const bool is_v = r >= per;
  const long long rr = is_v ? r - per : r;
  const int t = (int)(rr % a.n_new);
  const long long bh = rr / a.n_new;  // b * kv_heads + h
  constexpr int RB = kHeadDim * code_bits(BITS) / 8;
  constexpr int MB = (kHeadDim / G) * 4;
  const int pos = base_pos + t;
  RowRef ref;
  ref.src = (is_v ? a.v_new : a.k_new) + rr * kHeadDim;
  ref.active = pos < a.max_tokens;
  const long long dst = bh * a.max_tokens + pos;
  ref.codes = (is_v ? a.v_codes : a.k_codes) + dst * RB;
  ref.meta = (is_v ? a.v_meta : a.k_meta) + dst * MB;
  return ref;
}

// Decode-step append: one CTA per sequence handles all of its rows, then
// advances seq_lens[b] itself (every thread has read the old value before
// the barrier, so the update cannot race with the writes).
template <int BITS, int G, bool BF>
__global__ void __launch_bounds__(1024) quantize_append_kernel(const QuantArgs a) {
  const int b = blockIdx.x;
  const int base = a.seq_lens[b];
  if (a.k_channels && base % kChannelBlock != 0) return;  // not written, not advanced
  const int rows_per_side = a.kv_heads * a.n_new;
  const int rows = 2 * rows_per_side;
  const int lane16 = threadIdx.x & 15;
  const long long per = (long long)a.batch * rows_per_side;
  for (int r0 = a.side0 * rows_per_side; r0 < rows; r0 += blockDim.x / 16) {
    const int r = r0 + (int)(threadIdx.x >> 4);
    const bool in = r < rows;
    const int rs = in ? r : 0;
    const long long global_row =
        (rs < rows_per_side) ? (long long)b * rows_per_side + rs
                             : per + (long long)b * rows_per_side + (rs - rows_per_side);
    RowRef ref = locate_row<BITS, G>(a, global_row, base);
    quantize_slice<BITS, G, BF>(ref.src, ref.codes, ref.meta, lane16, in && ref.active);
  }
  if (a.advance) {
    __syncthreads();
    if (threadIdx.x == 0) a.seq_lens[b] = min(base + a.n_new, a.max_tokens);
  }
}

template <int BITS, int G, bool BF>
__device__ __forceinline__ void bulk_work(const QuantArgs& a, int li,
                                          const BulkDst<kHeadDim * code_bits(BITS) / 8,
                                                        (kHeadDim / G) * 4>& c,
                                          const uint32_t (&roff)[kBulkNV / 8],
                                          const uint8_t* slot) {
  constexpr int NW = code_words<BITS, kBulkNV>();
  const bool in = c.p.t < a.n_new;
  uint4 raw[kBulkNV / 8];
#pragma unroll
  for (int k = 0; k < kBulkNV / 8; ++k)
    raw[k] = in ? *reinterpret_cast<const uint4*>(slot + roff[k]) : make_uint4(0u, 0u, 0u, 0u);
  uint32_t cw[NW], m;
  quantize_vals<BITS, G, kBulkNV, BF>(raw, cw, m);
  if (in && c.pos < a.max_tokens && !c.skip) {
    if constexpr (NW == 8) {
      reinterpret_cast<uint4*>(c.codes)[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      reinterpret_cast<uint4*>(c.codes)[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
    } else if constexpr (NW == 4) {
      *reinterpret_cast<uint4*>(c.codes) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    } else {
      *reinterpret_cast<uint2*>(c.codes) = make_uint2(cw[0], cw[1]);
    }
    constexpr int GL = G / kBulkNV;  // lanes per group
    if ((li % GL) == 0) reinterpret_cast<uint32_t*>(c.meta)[li / GL] = m;
  }
}

template <int BITS, int G, bool BF>
__global__ void __launch_bounds__(kBulkWarps * 32) quantize_bulk_kernel(const QuantArgs a,
                                                                        int units_per_row,
                                                                        int n_units,
                                                                        int units_per_warp) {
  __shared__ __align__(16) uint8_t ring[kBulkWarps][kBulkDepth][kUnitBytes];
  const int li = (threadIdx.x & 31) % kBulkLanes;
  using Dst = BulkDst<kHeadDim * code_bits(BITS) / 8, (kHeadDim / G) * 4>;
  bulk_loop<Dst>(a, units_per_row, n_units, units_per_warp, &ring[threadIdx.x >> 5][0][0],
                 [&](const Dst& c, const uint32_t (&roff)[kBulkNV / 8], const uint8_t* slot) {
                   bulk_work<BITS, G, BF>(a, li, c, roff, slot);
                 });
}

__global__ void advance_seq_lens_kernel(int32_t* seq_lens, int batch, int n_new,
                                        int max_tokens, int k_channels) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch && !(k_channels && seq_lens[b] % kChannelBlock != 0))
    seq_lens[b] = min(seq_lens[b] + n_new, max_tokens);
}

// Per-channel K (the KV-cache page's INT8 item: the Key quantized per
// channel).  Work item: a block of kChannelBlock new tokens of one (sequence,
// KV head), whose fp16 rows are one contiguous 8 KB run of the input.  Each
// CTA (thread d owning channel d) takes every gridDim.x-th block and keeps
// the next kChanDepth - 1 blocks in flight as cp.async copies into its ring.
// Each channel's min, max, scale, zero point and codes follow the same fp32
// steps as the per-token groups (the IEEE quotient, round half to even), then
// the codes are packed along the token rows.  A sequence whose length is not
// a multiple of the block is skipped; blocks at or past max_tokens (a
// multiple of 64) are dropped whole.
constexpr int kChanDepth = 3;

template <int BITS>
__global__ void __launch_bounds__(kHeadDim) quantize_k_channels_kernel(const QuantArgs a) {
  constexpr int D = kHeadDim, TB = kChannelBlock, RB = D * BITS / 8;
  constexpr int CHUNKS = TB * D / 8 / kHeadDim;  // 16-byte copies per thread and block
  __shared__ __align__(16) __half ring[kChanDepth][TB][D];
  __shared__ __align__(16) uint8_t cs[TB][D];
  const int nblk = a.n_new / TB;
  const long long total = (long long)a.batch * a.kv_heads * nblk;
  const int d = threadIdx.x;
  const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(&ring[0][0][0]);
  // block k of this CTA (global index blockIdx.x + k * gridDim.x) into slot k % depth
  auto issue = [&](long long k) {
    const long long q = blockIdx.x + k * gridDim.x;
    if (q < total) {
      const uint4* src = reinterpret_cast<const uint4*>(a.k_new) + q * (TB * D / 8);
      const uint32_t slot = ring0 + (uint32_t)((k % kChanDepth) * (TB * D * 2));
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c)
        cp_async16(slot + (c * kHeadDim + d) * 16, src + c * kHeadDim + d);
    }
    cp_async_commit();  // possibly empty: the wait count stays uniform
  };
#pragma unroll
  for (int k = 0; k < kChanDepth - 1; ++k) issue(k);
  for (long long k = 0;; ++k) {
    const long long q = blockIdx.x + k * gridDim.x;
    if (q >= total) break;
    // the slot of block k - 1 was read before the previous barrier
    issue(k + kChanDepth - 1);
    cp_async_wait<kChanDepth - 1>();  // this thread's copies of block k have landed
    __syncthreads();                  // ... and every thread's; cs is free
    const int bh = (int)(q / nblk);
    const int j = (int)(q - (long long)bh * nblk);
    const int b = bh / a.kv_heads;
    const int base = a.seq_lens[b];
    const int pos0 = base + j * TB;
    const bool skip = base % TB != 0 || pos0 >= a.max_tokens;  // uniform over the CTA
    const __half (*xs)[D] = ring[k % kChanDepth];
    if (!skip) {
      float x[TB];
#pragma unroll
      for (int t = 0; t < TB; ++t) x[t] = __half2float(xs[t][d]);
      // the channel's extremes (-0 and +0 give the same scale and zero point)
      float mn = x[0], mx = x[0];
#pragma unroll
      for (int t = 1; t < TB; ++t) {
        mn = fminf(mn, x[t]);
        mx = fmaxf(mx, x[t]);
      }
      constexpr int qmax_i = (1 << BITS) - 1;
      constexpr float qmax = float(qmax_i), kInvQmax = 1.0f / qmax;
      constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
      // x / d below: the correction step on RN(1/d), the IEEE quotient
      const float s32 = fmaxf(div_rn(__fsub_rn(mx, mn), qmax, kInvQmax), 1e-5f);
      const __half s16 = __float2half_ru(s32);
      const float s = __half2float(s16);
      const float r = __frcp_rn(s);
      float zf = __fadd_rn(rintf(div_rn(-mn, s, r)), 0.0f);
      zf = fminf(fmaxf(zf, -65504.0f), 65504.0f);
      const __half z16 = __float2half_rn(zf);
      const float z = __half2float(z16);
      const float zm = z - kMagic;
      // code = clamp(rint(x / s) + z, 0, qmax): (q + M) + z is M + the code, whose
      // low mantissa bits are the code, when the channel needs no clamp (|z| <=
      // 2048 and its top code, (q_max + M) + (z - M), <= qmax; see the per-token
      // quantizer), else with the quotient clamped first.  Tokens t and t + 16
      // share one packed f32x2 operation.
      const float top = __fadd_rn(__fadd_rn(div_rn(mx, s, r), kMagic), zm);
      const uint64_t r2 = f2_pack(r, r), nd2 = f2_pack(-s, -s);
      const uint64_t m2 = f2_pack(kMagic, kMagic), z2 = f2_pack(z, z);
      constexpr int HT = TB / 2;
      if (fabsf(zf) <= 2048.0f && top <= qmax) {
#pragma unroll
        for (int t = 0; t < HT; ++t) {
          const float2 c =
              f2_unpack(f2_add(f2_add(div_rn2(f2_pack(x[t], x[t + HT]), nd2, r2), m2), z2));
          cs[t][d] = (uint8_t)__float_as_uint(c.x);
          cs[t + HT][d] = (uint8_t)__float_as_uint(c.y);
        }
      } else {
        const float lo = -z, hi = __fadd_rn(qmax, -z);
#pragma unroll
        for (int t = 0; t < HT; ++t) {
          const float2 qv = f2_unpack(div_rn2(f2_pack(x[t], x[t + HT]), nd2, r2));
          const uint64_t qc = f2_pack(fminf(fmaxf(qv.x, lo), hi), fminf(fmaxf(qv.y, lo), hi));
          const float2 c = f2_unpack(f2_add(f2_add(qc, m2), z2));
          cs[t][d] = (uint8_t)__float_as_uint(c.x);
          cs[t + HT][d] = (uint8_t)__float_as_uint(c.y);
        }
      }
      const long long blk = (long long)bh * (a.max_tokens / TB) + pos0 / TB;
      reinterpret_cast<__half2*>(a.k_meta)[blk * D + d] = __halves2half2(s16, z16);
    }
    __syncthreads();  // the block's codes are in cs
    if (!skip) {
      // rows of codes: whole words read from the byte codes
      for (int i = threadIdx.x; i < TB * RB / 4; i += blockDim.x) {
        const int t = i / (RB / 4), w = i % (RB / 4);
        uint32_t word;
        if constexpr (BITS == 8) {
          word = *reinterpret_cast<const uint32_t*>(&cs[t][4 * w]);
        } else if constexpr (BITS == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(&cs[t][8 * w]);
          const uint32_t a0 = v.x | (v.x >> 4), a1 = v.y | (v.y >> 4);  // bytes 0, 2: code pairs
          word = __byte_perm(a0, a1, 0x6420);
        } else {
          const uint4 v = *reinterpret_cast<const uint4*>(&cs[t][16 * w]);
          const uint32_t q4[4] = {v.x, v.y, v.z, v.w};
          uint32_t c4[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t c1 = q4[m] | (q4[m] >> 6);  // bytes 0, 2: code pairs
            c4[m] = c1 | (c1 >> 12);                   // byte 0: four codes
          }
          word = __byte_perm(__byte_perm(c4[0], c4[1], 0x0040), __byte_perm(c4[2], c4[3], 0x0040),
                             0x5410);
        }
        reinterpret_cast<uint32_t*>(a.k_codes + ((long long)bh * a.max_tokens + pos0 + t) * RB)[w] =
            word;
      }
    }
  }
  cp_async_wait<0>();
}

template <int BITS, int G, bool BF>
cudaError_t launch_q(const QuantArgs& a_in, cudaStream_t s) {
  QuantArgs a = a_in;
  if (a.k_channels) {
    // K: whole blocks, per channel; then the per-token kernels write V only
    if constexpr ((BITS == 2 || BITS == 4 || BITS == 8) && !BF) {
      if (a.n_new % kChannelBlock != 0) return cudaErrorInvalidValue;
      static int ch_per_sm = 0;  // resident CTAs per SM of the channel kernel
      if (ch_per_sm == 0) {
        int r = 0;
        const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &r, quantize_k_channels_kernel<BITS>, kHeadDim, 0);
        if (e != cudaSuccess) return e;
        ch_per_sm = r > 0 ? r : 1;
      }
      const long long blocks = (long long)a.batch * a.kv_heads * (a.n_new / kChannelBlock);
      const long long slots = (long long)device_sm_count() * ch_per_sm;
      const unsigned grid = (unsigned)(blocks < slots ? blocks : slots);
      if (grid > 0) quantize_k_channels_kernel<BITS><<<grid, kHeadDim, 0, s>>>(a);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      a.side0 = 1;
    } else {
      return cudaErrorInvalidValue;
    }
  }
  const int rows_per_seq = (2 - a.side0) * a.kv_heads * a.n_new;
  if (a.n_new < kUnitRows || rows_per_seq <= 64) {
    // a few tokens per sequence (the decode-step append): one CTA per
    // sequence, one pass when its rows fit
    int threads = ((rows_per_seq * 16 + 63) / 64) * 64;
    if (threads > 1024) threads = 1024;
    quantize_append_kernel<BITS, G, BF><<<a.batch, threads, 0, s>>>(a);
    return cudaGetLastError();
  }
  static int per_sm = 0;  // resident CTAs per SM of this kernel
  if (per_sm == 0) {
    int r = 0;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &r, quantize_bulk_kernel<BITS, G, BF>, kBulkWarps * 32, 0);
    if (e != cudaSuccess) return e;
    per_sm = r > 0 ? r : 1;
  }
  BulkShape sh;
  if (!bulk_shape(a, per_sm, &sh)) return cudaErrorInvalidValue;
  quantize_bulk_kernel<BITS, G, BF><<<sh.blocks, kBulkWarps * 32, 0, s>>>(
      a, sh.units_per_row, sh.n_units, sh.per_warp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.advance) return e;
  advance_seq_lens_kernel<<<(a.batch + 127) / 128, 128, 0, s>>>(a.seq_lens, a.batch, a.n_new,
                                                               a.max_tokens, a.k_channels);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const QuantArgs& a, int bits, int group, cudaStream_t s) {
#define KVQ_Q(B, G_)                                              \
  if (bits == B && group == G_)                                   \
    return a.in_bf16 ? launch_q<B, G_, true>(a, s) : launch_q<B, G_, false>(a, s);
  KVQ_Q(8, 32) KVQ_Q(8, 64) KVQ_Q(8, 128)
  KVQ_Q(4, 32) KVQ_Q(4, 64) KVQ_Q(4, 128)
  KVQ_Q(2, 32) KVQ_Q(2, 64) KVQ_Q(2, 128)
  KVQ_Q(kE4M3, 32) KVQ_Q(kE4M3, 64) KVQ_Q(kE4M3, 128)
  KVQ_Q(kSym8, 32) KVQ_Q(kSym8, 64) KVQ_Q(kSym8, 128)
  KVQ_Q(kE5M2, 32) KVQ_Q(kE5M2, 64) KVQ_Q(kE5M2, 128)
#undef KVQ_Q
  return cudaErrorInvalidValue;
}

}  // namespace kvq
