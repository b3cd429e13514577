// kvq_chunk.cu -- Cocktail's chunk-level mixed precision (peacm.com news
// 1099647): the per-chunk bit-width search of section 3.1.1 and the reorder
// of section 3.1.2 (equal bit-widths made contiguous, then quantized).
#include <cuda_runtime.h>
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant_core.cuh"

namespace kvq {

namespace {

constexpr int kAssignThreads = 256;

// One CTA per sequence.  Similarities are fp64 with every sum taken in index
// order and multiply/add kept separate (explicit _rn intrinsics), so each
// class decision is reproducible bit for bit.
__global__ void __launch_bounds__(kAssignThreads)
chunk_assign_kernel(const float* __restrict__ emb, const float* __restrict__ qemb, int n_chunks,
                    int dim, double alpha, double beta, double* __restrict__ sim_out,
                    uint8_t* __restrict__ bits_out) {
  extern __shared__ double sims[];  // [n_chunks]
  __shared__ double s_nq, s_min_w[kAssignThreads / 32], s_max_w[kAssignThreads / 32];
  const int b = blockIdx.x;
  const float* q = qemb + (long long)b * dim;
  if (threadIdx.x == 0) {
    double qq = 0.0;
    for (int d = 0; d < dim; ++d) qq = __dadd_rn(qq, __dmul_rn((double)q[d], (double)q[d]));
    s_nq = __dsqrt_rn(qq);
  }
  __syncthreads();
  const double nq = s_nq;
  double lo = INFINITY, hi = -INFINITY;
  for (int i = threadIdx.x; i < n_chunks; i += blockDim.x) {
    const float* c = emb + ((long long)b * n_chunks + i) * dim;
    double dot = 0.0, cc = 0.0;
    for (int d = 0; d < dim; ++d) {
      const double cd = (double)c[d];
      dot = __dadd_rn(dot, __dmul_rn((double)q[d], cd));
      cc = __dadd_rn(cc, __dmul_rn(cd, cd));
    }
    const double s = __ddiv_rn(dot, __dmul_rn(nq, __dsqrt_rn(cc)));
    sims[i] = s;
    lo = fmin(lo, s);
    hi = fmax(hi, s);
  }
  for (int off = 16; off > 0; off >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if ((threadIdx.x & 31) == 0) {
    s_min_w[threadIdx.x >> 5] = lo;
    s_max_w[threadIdx.x >> 5] = hi;
  }
  __syncthreads();
  double s_min = s_min_w[0], s_max = s_max_w[0];
  for (int w = 1; w < kAssignThreads / 32; ++w) {
    s_min = fmin(s_min, s_min_w[w]);
    s_max = fmax(s_max, s_max_w[w]);
  }
  const double span = __dsub_rn(s_max, s_min);
  const double t_low = __dadd_rn(s_min, __dmul_rn(span, alpha));
  const double t_high = __dsub_rn(s_max, __dmul_rn(span, beta));
  for (int i = threadIdx.x; i < n_chunks; i += blockDim.x) {
    const double s = sims[i];
    bits_out[(long long)b * n_chunks + i] = (s > t_high) ? 16 : ((s > t_low) ? 4 : 2);
    if (sim_out != nullptr) sim_out[(long long)b * n_chunks + i] = s;
  }
}

// One warp per sequence: stable partition of chunk indices, FP16 class
// first, then INT4, then INT2 (ascending original index within a class);
// writes perm and the three segments' token counts.
__global__ void chunk_partition_kernel(const uint8_t* __restrict__ bits, int n_chunks,
                                       int chunk_tokens, int32_t* __restrict__ perm,
                                       int32_t* len16, int32_t* len4, int32_t* len2) {
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  const uint8_t* cb = bits + (long long)b * n_chunks;
  int32_t* pb = perm + (long long)b * n_chunks;
  const uint8_t classes[3] = {16, 4, 2};
  int32_t* lens[3] = {len16, len4, len2};
  int base = 0;
  for (int c = 0; c < 3; ++c) {
    int count = 0;
    for (int i0 = 0; i0 < n_chunks; i0 += 32) {
      const int i = i0 + lane;
      // any value other than 16 or 4 counts as INT2, so every chunk lands in
      // exactly one class and every perm entry is written
      const int v = (i < n_chunks) ? cb[i] : -1;
      const int cls = (v == 16 || v == 4) ? v : 2;
      const bool hit = (i < n_chunks) && cls == classes[c];
      const unsigned m = __ballot_sync(0xffffffffu, hit);
      if (hit) pb[base + count + __popc(m & ((1u << lane) - 1u))] = i;
      count += __popc(m);
    }
    if (lane == 0) lens[c][b] = count * chunk_tokens;
    base += count;
  }
}

struct ReorderDev {
  const __half* k_src;
  const __half* v_src;
  const int32_t* perm;
  uint8_t* codes[3][2];  // [segment][K/V]
  uint8_t* meta[3][2];
  const int32_t* lens[3];
  int32_t max_tokens[3];
  int32_t batch, kv_heads, context_len, chunk_tokens, n_chunks;
};

// Rows in reordered order: r = ((b * H + h) * n_chunks + k) * T + j for the
// K side, then the same count for V.  Two consecutive rows of a warp share a
// chunk (T even), so the class -- and the code path -- is warp-uniform.
template <int G>
__global__ void __launch_bounds__(256) chunk_gather_quantize_kernel(const ReorderDev a) {
  const long long per = (long long)a.batch * a.kv_heads * a.context_len;
  const long long rows = 2 * per;
  const int lane16 = threadIdx.x & 15;
  const long long step = (long long)gridDim.x * (blockDim.x / 16);
  const long long first = (long long)blockIdx.x * (blockDim.x / 16) + (threadIdx.x >> 4);
  const long long warp_first = first & ~1LL;
  for (long long r = first; warp_first + (r - first) < rows; r += step) {
    const bool in = r < rows;
    const long long rr0 = in ? r : (r - 1);  // partner row: same chunk, same class
    const int side = rr0 >= per ? 1 : 0;
    const long long rr = side ? rr0 - per : rr0;
    const int j = (int)(rr % a.chunk_tokens);
    const long long kk = rr / a.chunk_tokens;  // (b * H + h) * n_chunks + k
    const int k = (int)(kk % a.n_chunks);
    const long long bh = kk / a.n_chunks;
    const int b = (int)(bh / a.kv_heads);
    const int n16 = a.lens[0][b] / a.chunk_tokens;
    const int n4 = a.lens[1][b] / a.chunk_tokens;
    int seg, pos;
    if (k < n16) {
      seg = 0;
      pos = k;
    } else if (k < n16 + n4) {
      seg = 1;
      pos = k - n16;
    } else {
      seg = 2;
      pos = k - n16 - n4;
    }
    const int src_chunk = a.perm[(long long)b * a.n_chunks + k];
    const __half* src = (side ? a.v_src : a.k_src) +
                        (bh * a.context_len + (long long)src_chunk * a.chunk_tokens + j) * kHeadDim;
    const long long drow = bh * a.max_tokens[seg] + (long long)pos * a.chunk_tokens + j;
    const bool ok = in && ((long long)pos * a.chunk_tokens + j) < a.max_tokens[seg];
    if (seg == 0) {
      if (ok) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + lane16);
        reinterpret_cast<uint4*>(a.codes[0][side] + drow * (kHeadDim * 2))[lane16] = v;
      }
    } else if (seg == 1) {
      quantize_slice<4, G>(src, a.codes[1][side] + drow * (kHeadDim / 2),
                           a.meta[1][side] + drow * ((kHeadDim / G) * 4), lane16, ok);
    } else {
      quantize_slice<2, G>(src, a.codes[2][side] + drow * (kHeadDim / 4),
                           a.meta[2][side] + drow * ((kHeadDim / G) * 4), lane16, ok);
    }
  }
}

}  // namespace

cudaError_t launch_chunk_assign(const float* emb, const float* qemb, int batch, int n_chunks,
                                int emb_dim, double alpha, double beta, double* sim,
                                uint8_t* bits, cudaStream_t s) {
  const size_t smem = (size_t)n_chunks * sizeof(double);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(chunk_assign_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  chunk_assign_kernel<<<batch, kAssignThreads, smem, s>>>(emb, qemb, n_chunks, emb_dim, alpha,
                                                          beta, sim, bits);
  return cudaGetLastError();
}

cudaError_t launch_chunk_reorder(const ReorderArgs& r, cudaStream_t s) {
  chunk_partition_kernel<<<r.batch, 32, 0, s>>>(r.chunk_bits, r.n_chunks, r.chunk_tokens, r.perm,
                                                r.seg[0].seq_lens, r.seg[1].seq_lens,
                                                r.seg[2].seq_lens);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ReorderDev a;
  a.k_src = r.k_src;
  a.v_src = r.v_src;
  a.perm = r.perm;
  for (int i = 0; i < 3; ++i) {
    a.codes[i][0] = static_cast<uint8_t*>(r.seg[i].k.codes);
    a.codes[i][1] = static_cast<uint8_t*>(r.seg[i].v.codes);
    a.meta[i][0] = static_cast<uint8_t*>(r.seg[i].k.meta);
    a.meta[i][1] = static_cast<uint8_t*>(r.seg[i].v.meta);
    a.lens[i] = r.seg[i].seq_lens;
    a.max_tokens[i] = r.seg[i].max_tokens;
  }
  a.batch = r.batch;
  a.kv_heads = r.kv_heads;
  a.context_len = r.context_len;
  a.chunk_tokens = r.chunk_tokens;
  a.n_chunks = r.n_chunks;
  const long long rows = 2LL * r.batch * r.kv_heads * r.context_len;
  long long blocks = (rows + 15) / 16;
  if (blocks > 148LL * 8) blocks = 148LL * 8;
  const int G = r.seg[1].k.group_size;
  if (G == 32)
    chunk_gather_quantize_kernel<32><<<(unsigned)blocks, 256, 0, s>>>(a);
  else if (G == 64)
    chunk_gather_quantize_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(a);
  else
    chunk_gather_quantize_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace kvq
