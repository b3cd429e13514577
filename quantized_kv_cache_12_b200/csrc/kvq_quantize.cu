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

// Bulk quantize (prefill).  Work unit: kUnitRows consecutive tokens of one
// (side, sequence, KV head) plane row, whose fp16 rows are contiguous in the
// input and whose codes and (s, z) are contiguous in the cache.  A warp takes
// units round-robin, four rows per step (8 lanes x 32 bytes per row, 16
// values per lane), and loads the next unit's rows before it quantizes the
// current one, so every lane keeps 64 bytes of reads in flight.
constexpr int kUnitRows = 8;
constexpr int kBulkNV = 16;                           // values per lane
constexpr int kBulkLanes = kHeadDim / kBulkNV;        // lanes per row
constexpr int kBulkRowsPerStep = 32 / kBulkLanes;     // rows per warp step
constexpr int kBulkSteps = kUnitRows / kBulkRowsPerStep;

struct BulkUnit {
  uint4 raw[kBulkSteps][kBulkNV / 8];
  long long dst_row;  // cache row of position 0 of the unit's plane row
  int t0, base, is_v;
};

__device__ __forceinline__ void bulk_fetch(const QuantArgs& a, int u, int units_per_row, int li,
                                           int ri, BulkUnit& w) {
  const int planes = a.batch * a.kv_heads;
  const int p = u / units_per_row;
  const int j = u - p * units_per_row;
  const bool is_v = p >= planes;
  const int bh = is_v ? p - planes : p;
  w.t0 = j * kUnitRows;
  w.base = a.seq_lens[bh / a.kv_heads];
  w.dst_row = (long long)bh * a.max_tokens;
  w.is_v = is_v;
  const uint4* src = reinterpret_cast<const uint4*>(
      (is_v ? a.v_new : a.k_new) + ((long long)bh * a.n_new + w.t0) * kHeadDim);
#pragma unroll
  for (int k = 0; k < kBulkSteps; ++k) {
    const int row = kBulkRowsPerStep * k + ri;
    const bool in = w.t0 + row < a.n_new;
#pragma unroll
    for (int c = 0; c < kBulkNV / 8; ++c)
      w.raw[k][c] = in ? __ldcs(src + row * (kHeadDim / 8) + li * (kBulkNV / 8) + c)
                       : make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int BITS, int G>
__device__ __forceinline__ void bulk_work(const QuantArgs& a, int li, int ri, const BulkUnit& w) {
  constexpr int RB = kHeadDim * code_bits(BITS) / 8;
  constexpr int MB = (kHeadDim / G) * 4;
  constexpr int NW = code_words<BITS, kBulkNV>();
  uint8_t* codes = w.is_v ? a.v_codes : a.k_codes;
  uint8_t* meta = w.is_v ? a.v_meta : a.k_meta;
#pragma unroll
  for (int k = 0; k < kBulkSteps; ++k) {
    const int t = w.t0 + kBulkRowsPerStep * k + ri;
    const int pos = w.base + t;
    uint32_t cw[NW], m;
    quantize_vals<BITS, G, kBulkNV>(w.raw[k], cw, m);
    if (t < a.n_new && pos < a.max_tokens) {
      const long long row = w.dst_row + pos;
      uint8_t* cr = codes + row * RB;
      if constexpr (NW == 4) {
        reinterpret_cast<uint4*>(cr)[li] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      } else if constexpr (NW == 2) {
        reinterpret_cast<uint2*>(cr)[li] = make_uint2(cw[0], cw[1]);
      } else {
        reinterpret_cast<uint32_t*>(cr)[li] = cw[0];
      }
      constexpr int GL = G / kBulkNV;  // lanes per group
      if ((li % GL) == 0) reinterpret_cast<uint32_t*>(meta + row * MB)[li / GL] = m;
    }
  }
}

template <int BITS, int G>
__global__ void __launch_bounds__(256) quantize_bulk_kernel(const QuantArgs a, int units_per_row,
                                                            int n_units) {
  const int lane = threadIdx.x & 31;
  const int li = lane % kBulkLanes, ri = lane / kBulkLanes;
  const int nw = gridDim.x * (blockDim.x >> 5);
  int u = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // uniform across the warp
  BulkUnit A, B;
  if (u < n_units) bulk_fetch(a, u, units_per_row, li, ri, A);
  while (u < n_units) {
    const int u1 = u + nw;
    if (u1 < n_units) bulk_fetch(a, u1, units_per_row, li, ri, B);
    bulk_work<BITS, G>(a, li, ri, A);
    if (u1 >= n_units) break;
    const int u2 = u1 + nw;
    if (u2 < n_units) bulk_fetch(a, u2, units_per_row, li, ri, A);
    bulk_work<BITS, G>(a, li, ri, B);
    u = u2;
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
  const int units_per_row = (a.n_new + kUnitRows - 1) / kUnitRows;
  const long long n_units = 2LL * a.batch * a.kv_heads * units_per_row;
  if (n_units > 0x7fffffffLL) return cudaErrorInvalidValue;
  static int slots = 0;  // resident 256-thread CTAs on the device
  if (slots == 0) {
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_bulk_kernel<BITS, G>,
                                                        256, 0);
    if (e != cudaSuccess) return e;
    slots = sms * (per_sm > 0 ? per_sm : 1);
  }
  long long blocks = (n_units + 7) / 8;
  if (blocks > slots) blocks = slots;
  quantize_bulk_kernel<BITS, G><<<(unsigned)blocks, 256, 0, s>>>(a, units_per_row, (int)n_units);
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
