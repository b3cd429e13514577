// kvq_quantize.cu -- quantize-on-write of new K/V tokens into the packed
// cache (Cocktail page 3.2.2 formula; Oaken page 3.2.3 pipeline, where the
// quantizer sits inside the memory write).
//
// Layout of a thread's work: a token row of 128 fp16 values is 16 lanes x 16
// bytes; a warp quantizes two rows per step.  The row's groups are reduced
// with warp shuffles, codes are packed in registers and written with one
// 2/4/8-byte store per lane, and the group leader writes (scale, zero).
#include <cuda_runtime.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"
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
template <int BITS, int G>
__global__ void __launch_bounds__(1024) quantize_append_kernel(const QuantArgs a) {
  const int b = blockIdx.x;
  const int base = a.seq_lens[b];
  const int rows_per_side = a.kv_heads * a.n_new;
  const int rows = 2 * rows_per_side;
  const int lane16 = threadIdx.x & 15;
  const long long per = (long long)a.batch * rows_per_side;
  for (int r0 = 0; r0 < rows; r0 += blockDim.x / 16) {
    const int r = r0 + (int)(threadIdx.x >> 4);
    const bool in = r < rows;
    const int rs = in ? r : 0;
    const long long global_row =
        (rs < rows_per_side) ? (long long)b * rows_per_side + rs
                             : per + (long long)b * rows_per_side + (rs - rows_per_side);
    RowRef ref = locate_row<BITS, G>(a, global_row, base);
    quantize_slice<BITS, G>(ref.src, ref.codes, ref.meta, lane16, in && ref.active);
  }
  if (a.advance) {
    __syncthreads();
    if (threadIdx.x == 0) a.seq_lens[b] = min(base + a.n_new, a.max_tokens);
  }
}

// Bulk quantize (prefill): grid-stride over all rows.  Reads each thread's
// sequence length once per row; lengths are advanced by a separate kernel.
template <int BITS, int G>
__global__ void __launch_bounds__(256) quantize_bulk_kernel(const QuantArgs a) {
  const long long rows = 2LL * a.batch * a.kv_heads * a.n_new;
  const int lane16 = threadIdx.x & 15;
  const long long rows_per_step = (long long)gridDim.x * (blockDim.x / 16);
  const long long first = (long long)blockIdx.x * (blockDim.x / 16) + (threadIdx.x >> 4);
  // trip count is uniform across the warp (both half-warps take the same steps)
  const long long warp_first = first & ~1LL;
  for (long long r = first; warp_first + (r - first) < rows; r += rows_per_step) {
    const bool in = r < rows;
    const long long rs = in ? r : 0;
    const long long per = (long long)a.batch * a.kv_heads * a.n_new;
    const long long rr = rs >= per ? rs - per : rs;
    const int b = (int)(rr / ((long long)a.kv_heads * a.n_new));
    RowRef ref = locate_row<BITS, G>(a, rs, a.seq_lens[b]);
    quantize_slice<BITS, G>(ref.src, ref.codes, ref.meta, lane16, in && ref.active);
  }
}

__global__ void advance_seq_lens_kernel(int32_t* seq_lens, int batch, int n_new,
                                        int max_tokens) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch) seq_lens[b] = min(seq_lens[b] + n_new, max_tokens);
}

template <int BITS, int G>
cudaError_t launch_q(const QuantArgs& a, cudaStream_t s) {
  const int rows_per_seq = 2 * a.kv_heads * a.n_new;
  if (rows_per_seq <= 512) {
    // one pass over the sequence's rows when they fit in one CTA
    int threads = ((rows_per_seq * 16 + 63) / 64) * 64;
    if (threads > 1024) threads = 1024;
    quantize_append_kernel<BITS, G><<<a.batch, threads, 0, s>>>(a);
    return cudaGetLastError();
  }
  const long long rows = (long long)a.batch * rows_per_seq;
  long long blocks = (rows + 15) / 16;
  const long long cap = 148LL * 8;  // 8 resident 256-thread CTAs per SM
  if (blocks > cap) blocks = cap;
  quantize_bulk_kernel<BITS, G><<<(unsigned)blocks, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.advance) return e;
  advance_seq_lens_kernel<<<(a.batch + 127) / 128, 128, 0, s>>>(a.seq_lens, a.batch, a.n_new,
                                                               a.max_tokens);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const QuantArgs& a, int bits, int group, cudaStream_t s) {
#define KVQ_Q(B, G_) \
  if (bits == B && group == G_) return launch_q<B, G_>(a, s);
  KVQ_Q(8, 32) KVQ_Q(8, 64) KVQ_Q(8, 128)
  KVQ_Q(4, 32) KVQ_Q(4, 64) KVQ_Q(4, 128)
  KVQ_Q(2, 32) KVQ_Q(2, 64) KVQ_Q(2, 128)
  KVQ_Q(kE4M3, 32) KVQ_Q(kE4M3, 64) KVQ_Q(kE4M3, 128)
#undef KVQ_Q
  return cudaErrorInvalidValue;
}

}  // namespace kvq
