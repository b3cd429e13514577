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
  grid_dependents_may_launch();  // the seq_lens update may be scheduled
  const int li = (threadIdx.x & 31) % kBulkLanes;
  using Dst = BulkDst<kHeadDim * code_bits(BITS) / 8, (kHeadDim / G) * 4>;
  bulk_loop<Dst>(a, units_per_row, n_units, units_per_warp, &ring[threadIdx.x >> 5][0][0],
                 [&](const Dst& c, const uint32_t (&roff)[kBulkNV / 8], const uint8_t* slot) {
                   bulk_work<BITS, G, BF>(a, li, c, roff, slot);
                 });
  // launched as the per-channel K kernel's dependent (V rows only), this one
  // starts on the SMs that kernel leaves and must not finish before it: the
  // seq_lens update after it assumes both are done (a no-op otherwise)
  grid_dependency_wait();
}

__global__ void advance_seq_lens_kernel(int32_t* seq_lens, int batch, int n_new,
                                        int max_tokens, int k_channels) {
  grid_dependency_wait();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch && !(k_channels && seq_lens[b] % kChannelBlock != 0))
    seq_lens[b] = min(seq_lens[b] + n_new, max_tokens);
}

// Per-channel K (the KV-cache page's INT8 item: the Key quantized per
// channel).  Work item: a block of kChannelBlock new tokens of one (sequence,
// KV head), whose fp16 (or, with BF, bf16) rows are one contiguous 8 KB run
// of the input and
// whose code rows are one contiguous run of the cache.  Each CTA takes every
// gridDim.x-th block and keeps the next kChanDepth - 1 blocks in flight as
// cp.async copies into its ring; thread p owns channels 2p and 2p + 1, read
// as 16-bit pairs (widened to fp32 exactly).  Each channel's min, max, scale,
// zero point and codes follow
// the same fp32 steps as the per-token groups (the IEEE quotient, round half
// to even), the two channels sharing packed f32x2 operations; the codes are
// packed into the block's rows in shared memory and copied out whole.  A
// sequence whose length is not a multiple of the block is skipped; blocks at
// or past max_tokens (a multiple of 64) are dropped whole.
constexpr int kChanDepth = 3;
constexpr int kChanThreads = kHeadDim / 2;

// Scale and zero point of one channel of a block from its extremes, and
// whether its codes need no clamp (see the per-token quantizer): |z| <= 2048
// and the top code (q_max + M) + (z - M) <= q_max.
template <int BITS>
__device__ __forceinline__ bool channel_params(float mn, float mx, __half& s16, __half& z16,
                                               float& s, float& r, float& z) {
  constexpr float qmax = float((1 << BITS) - 1), kInvQmax = 1.0f / qmax;
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const float s32 = fmaxf(div_rn(__fsub_rn(mx, mn), qmax, kInvQmax), 1e-5f);
  s16 = __float2half_ru(s32);
  s = __half2float(s16);
  r = __frcp_rn(s);
  float zf = __fadd_rn(rintf(div_rn(-mn, s, r)), 0.0f);
  zf = fminf(fmaxf(zf, -65504.0f), 65504.0f);
  z16 = __float2half_rn(zf);
  z = __half2float(z16);
  const float top = __fadd_rn(__fadd_rn(div_rn(mx, s, r), kMagic), z - kMagic);
  return fabsf(zf) <= 2048.0f && top <= qmax;
}

template <int BITS, bool BF>
__global__ void __launch_bounds__(kChanThreads) quantize_k_channels_kernel(const QuantArgs a) {
  using IP = InPair<BF>;
  constexpr int D = kHeadDim, TB = kChannelBlock, RB = D * BITS / 8;
  constexpr int CHUNKS = TB * D * 2 / 16 / kChanThreads;  // 16-byte copies per thread and block
  constexpr int OUT = TB * RB / 16 / kChanThreads;        // 16-byte code stores per thread
  static_assert(OUT >= 1 && TB * RB == OUT * 16 * kChanThreads, "whole 16-byte code stores");
  __shared__ __align__(16) __half ring[kChanDepth][TB][D];
  __shared__ __align__(16) uint8_t cs[TB][RB];  // the block's packed code rows
  grid_dependents_may_launch();  // the V kernel may fill the SMs this one leaves
  const int nblk = a.n_new / TB;
  const int planes = a.batch * a.kv_heads;
  const int p = threadIdx.x;
  const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(&ring[0][0][0]);
  // the copy cursor: block (bh, j) = blockIdx.x + k * gridDim.x, k = 0, 1, ...
  // (stepped without dividing), and its ring slot
  const int step_bh = (int)(gridDim.x / nblk), step_j = (int)(gridDim.x % nblk);
  auto advance = [&](int& bh, int& j) {
    j += step_j;
    bh += step_bh;
    if (j >= nblk) {
      j -= nblk;
      ++bh;
    }
  };
  int ibh = (int)(blockIdx.x / nblk), ij = (int)(blockIdx.x % nblk), islot = 0;
  auto issue = [&]() {
    if (ibh < planes) {
      const uint4* src =
          reinterpret_cast<const uint4*>(a.k_new + ((long long)ibh * a.n_new + ij * TB) * D);
      const uint32_t slot = ring0 + (uint32_t)(islot * (TB * D * 2));
#pragma unroll
      for (int c = 0; c < CHUNKS; ++c)
        cp_async16(slot + (c * kChanThreads + p) * 16, src + c * kChanThreads + p);
    }
    cp_async_commit();  // possibly empty: the wait count stays uniform
    advance(ibh, ij);
    islot = islot + 1 == kChanDepth ? 0 : islot + 1;
  };
#pragma unroll
  for (int k = 0; k < kChanDepth - 1; ++k) issue();
  // the work cursor
  int bh = (int)(blockIdx.x / nblk), j = (int)(blockIdx.x % nblk), slot = 0;
  for (; bh < planes; advance(bh, j)) {
    issue();  // into the slot read before the previous barrier
    cp_async_wait<kChanDepth - 1>();  // this thread's copies of the block have landed
    __syncthreads();                  // ... and every thread's; cs is free
    const uint32_t* xs = reinterpret_cast<const uint32_t*>(&ring[slot][0][0]);  // [TB][D / 2]
    slot = slot + 1 == kChanDepth ? 0 : slot + 1;
    const int b = bh / a.kv_heads;
    const int base = a.seq_lens[b];
    const int pos0 = base + j * TB;
    const bool skip = base % TB != 0 || pos0 >= a.max_tokens;  // uniform over the CTA
    if (!skip) {
      uint32_t xv[TB];  // token t: the pair (channel 2p, channel 2p + 1)
#pragma unroll
      for (int t = 0; t < TB; ++t) xv[t] = xs[t * (D / 2) + p];
      // the channels' extremes, a pairwise tree (exact; -0 and +0 give the
      // same scale and zero point)
      uint32_t lo2[TB / 2], hi2[TB / 2];
#pragma unroll
      for (int t = 0; t < TB / 2; ++t) {
        lo2[t] = IP::min2(xv[2 * t], xv[2 * t + 1]);
        hi2[t] = IP::max2(xv[2 * t], xv[2 * t + 1]);
      }
#pragma unroll
      for (int w = TB / 4; w >= 1; w /= 2)
#pragma unroll
        for (int t = 0; t < w; ++t) {
          lo2[t] = IP::min2(lo2[t], lo2[t + w]);
          hi2[t] = IP::max2(hi2[t], hi2[t + w]);
        }
      const float2 mn = IP::widen(lo2[0]), mx = IP::widen(hi2[0]);
      __half s0h, z0h, s1h, z1h;
      float s0, r0, z0, s1, r1, z1;
      const bool ok0 = channel_params<BITS>(mn.x, mx.x, s0h, z0h, s0, r0, z0);
      const bool ok1 = channel_params<BITS>(mn.y, mx.y, s1h, z1h, s1, r1, z1);
      const long long blk = (long long)bh * (a.max_tokens / TB) + pos0 / TB;
      reinterpret_cast<uint2*>(a.k_meta)[blk * (D / 2) + p] =
          make_uint2(h2_as_u32(__halves2half2(s0h, z0h)), h2_as_u32(__halves2half2(s1h, z1h)));
      // code = clamp(rint(x / s) + z, 0, qmax): (q + M) + z is M + the code,
      // whose low mantissa bits are the code, when neither channel needs a
      // clamp, else with the quotients clamped first
      constexpr float qmax = float((1 << BITS) - 1), kMagic = 12582912.0f;
      const uint64_t r2 = f2_pack(r0, r1), nd2 = f2_pack(-s0, -s1);
      const uint64_t m2 = f2_pack(kMagic, kMagic), z2 = f2_pack(z0, z1);
      const float lo0 = -z0, hi0 = __fadd_rn(qmax, -z0), lo1 = -z1, hi1 = __fadd_rn(qmax, -z1);
      // the token's two codes into its code row
      auto put = [&](int t, uint64_t qv) {
        const float2 c = f2_unpack(f2_add(f2_add(qv, m2), z2));
        const uint32_t c0 = __float_as_uint(c.x) & 0xFFu, c1 = __float_as_uint(c.y) & 0xFFu;
        if constexpr (BITS == 8) {
          *reinterpret_cast<uint16_t*>(&cs[t][2 * p]) = (uint16_t)(c0 | (c1 << 8));
        } else if constexpr (BITS == 4) {
          cs[t][p] = (uint8_t)(c0 | (c1 << 4));
        } else {
          // four 2-bit codes a byte: the odd thread's pair joins the even one's
          const uint32_t nib = c0 | (c1 << 2);
          const uint32_t other = __shfl_down_sync(0xffffffffu, nib, 1);
          if ((p & 1) == 0) cs[t][p >> 1] = (uint8_t)(nib | (other << 4));
        }
      };
      // two loops, so that the common case carries no clamp; the choice is
      // the warp's (the clamp leaves in-range quotients as they are), which
      // keeps the 2-bit path's shuffle convergent
      if (__all_sync(0xffffffffu, ok0 && ok1)) {
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          const float2 xf = IP::widen(xv[t]);
          put(t, div_rn2(f2_pack(xf.x, xf.y), nd2, r2));
        }
      } else {
#pragma unroll
        for (int t = 0; t < TB; ++t) {
          const float2 xf = IP::widen(xv[t]);
          const float2 u = f2_unpack(div_rn2(f2_pack(xf.x, xf.y), nd2, r2));
          put(t, f2_pack(fminf(fmaxf(u.x, lo0), hi0), fminf(fmaxf(u.y, lo1), hi1)));
        }
      }
    }
    __syncthreads();  // the block's code rows are in cs
    if (!skip) {
      uint4* dst = reinterpret_cast<uint4*>(a.k_codes + ((long long)bh * a.max_tokens + pos0) * RB);
#pragma unroll
      for (int c = 0; c < OUT; ++c)
        dst[c * kChanThreads + p] =
            reinterpret_cast<const uint4*>(&cs[0][0])[c * kChanThreads + p];
    }
  }
  cp_async_wait<0>();
}

template <int BITS, int G, bool BF>
cudaError_t launch_q(const QuantArgs& a_in, cudaStream_t s) {
  QuantArgs a = a_in;
  bool after_k = false;  // the per-channel K kernel was launched just before
  if (a.k_channels) {
    // K: whole blocks, per channel; then the per-token kernels write V only
    if constexpr (BITS == 2 || BITS == 4 || BITS == 8) {
      if (a.n_new % kChannelBlock != 0) return cudaErrorInvalidValue;
      static int ch_per_sm = 0;  // resident CTAs per SM of the channel kernel
      if (ch_per_sm == 0) {
        int r = 0;
        const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &r, quantize_k_channels_kernel<BITS, BF>, kChanThreads, 0);
        if (e != cudaSuccess) return e;
        ch_per_sm = r > 0 ? r : 1;
      }
      const long long blocks = (long long)a.batch * a.kv_heads * (a.n_new / kChannelBlock);
      const long long slots = (long long)device_sm_count() * ch_per_sm;
      const unsigned grid = (unsigned)(blocks < slots ? blocks : slots);
      if (grid > 0) {
        quantize_k_channels_kernel<BITS, BF><<<grid, kChanThreads, 0, s>>>(a);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        after_k = true;
      }
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
  cudaError_t e;
  if (after_k) {
    // V only, after the per-channel K kernel: a programmatic dependent, so
    // its CTAs take the SMs that kernel's CTAs leave
    e = launch_dependent(quantize_bulk_kernel<BITS, G, BF>, dim3(sh.blocks),
                         dim3(kBulkWarps * 32), s, a, sh.units_per_row, sh.n_units, sh.per_warp);
  } else {
    quantize_bulk_kernel<BITS, G, BF><<<sh.blocks, kBulkWarps * 32, 0, s>>>(
        a, sh.units_per_row, sh.n_units, sh.per_warp);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess || !a.advance) return e;
  // a programmatic dependent: scheduled while the quantizer runs, it waits
  // for it before moving seq_lens (which the quantizer reads)
  return launch_dependent(advance_seq_lens_kernel, dim3((a.batch + 127) / 128), dim3(128), s,
                          a.seq_lens, a.batch, a.n_new, a.max_tokens, a.k_channels);
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
