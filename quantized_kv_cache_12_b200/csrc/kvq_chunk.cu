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

constexpr int kAssignThreads = 1024;  // one chunk per thread per round
constexpr int kAssignTile = 16;       // embedding dims per staged tile
constexpr int kAssignStride = 20;     // floats per staged row (16-B aligned, conflict-free reads)

// One CTA per sequence.  Similarities are fp64 with every sum taken in index
// order and multiply/add kept separate (explicit _rn intrinsics), so each
// class decision is reproducible bit for bit.  The chunk embeddings reach
// shared memory in coalesced, double-buffered cp.async tiles of kAssignTile
// dims for kAssignThreads chunks (four threads copy one row's 64 bytes);
// each thread then runs its own chunk's sums over the tile.
__global__ void __launch_bounds__(kAssignThreads)
chunk_assign_kernel(const float* __restrict__ emb, const float* __restrict__ qemb, int n_chunks,
                    int dim, double alpha, double beta, double* __restrict__ sim_out,
                    uint8_t* __restrict__ bits_out) {
  extern __shared__ __align__(16) uint8_t assign_smem[];
  double* sims = reinterpret_cast<double*>(assign_smem);              // [n_chunks]
  double* qd = sims + n_chunks;                                        // [dim]
  float* tiles = reinterpret_cast<float*>(qd + dim);                   // [2][threads][stride]
  __shared__ double s_nq, s_min_w[kAssignThreads / 32], s_max_w[kAssignThreads / 32];
  const int b = blockIdx.x, t = threadIdx.x;
  const float* q = qemb + (long long)b * dim;
  for (int d = t; d < dim; d += blockDim.x) qd[d] = (double)q[d];
  const uint32_t tiles0 = (uint32_t)__cvta_generic_to_shared(tiles);
  constexpr uint32_t kTileBytes = kAssignThreads * kAssignStride * 4;
  const int n_tiles = (dim + kAssignTile - 1) / kAssignTile;
  double lo = INFINITY, hi = -INFINITY;
  for (int c0 = 0; c0 < n_chunks; c0 += kAssignThreads) {
    // rows c0 .. c0 + kAssignThreads - 1, dims [d0, d0 + kAssignTile) into buffer buf
    auto load_tile = [&](int tile, int buf) {
      const int d0 = tile * kAssignTile;
#pragma unroll
      for (int r = 0; r < kAssignTile / 4; ++r) {
        const int idx = r * kAssignThreads + t;
        const int row = idx / (kAssignTile / 4), part = idx % (kAssignTile / 4);
        const int chunk = c0 + row, d = d0 + 4 * part;
        const uint32_t dst = tiles0 + buf * kTileBytes + (uint32_t)(row * kAssignStride + 4 * part) * 4;
        if (chunk < n_chunks && d + 4 <= dim)
          cp_async16(dst, emb + ((long long)b * n_chunks + chunk) * dim + d);
      }
      cp_async_commit();
    };
    load_tile(0, 0);
    if (c0 == 0 && t == 0) {
      double qq = 0.0;
      for (int d = 0; d < dim; ++d) qq = __dadd_rn(qq, __dmul_rn((double)q[d], (double)q[d]));
      s_nq = __dsqrt_rn(qq);
    }
    const int i = c0 + t;
    double dot = 0.0, cc = 0.0;
    for (int tile = 0; tile < n_tiles; ++tile) {
      if (tile + 1 < n_tiles) {
        load_tile(tile + 1, (tile + 1) & 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // every thread's copies of this tile have landed
      if (i < n_chunks) {
        const float* row = tiles + (tile & 1) * (kTileBytes / 4) + t * kAssignStride;
        const int d0 = tile * kAssignTile;
#pragma unroll
        for (int j4 = 0; j4 < kAssignTile; j4 += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(row + j4);
          const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (d0 + j4 + j < dim) {
              const double cd = (double)vv[j];
              dot = __dadd_rn(dot, __dmul_rn(qd[d0 + j4 + j], cd));
              cc = __dadd_rn(cc, __dmul_rn(cd, cd));
            }
          }
        }
      }
      __syncthreads();  // the buffer is read before it is refilled
    }
    if (i < n_chunks) {
      const double sv = __ddiv_rn(dot, __dmul_rn(s_nq, __dsqrt_rn(cc)));
      sims[i] = sv;
      lo = fmin(lo, sv);
      hi = fmax(hi, sv);
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if ((t & 31) == 0) {
    s_min_w[t >> 5] = lo;
    s_max_w[t >> 5] = hi;
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
  for (int k = t; k < n_chunks; k += blockDim.x) {
    const double sv = sims[k];
    bits_out[(long long)b * n_chunks + k] = (sv > t_high) ? 16 : ((sv > t_low) ? 4 : 2);
    if (sim_out != nullptr) sim_out[(long long)b * n_chunks + k] = sv;
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

// The reorder's gather and quantize in the layout of the bulk quantize
// kernel.  A unit is kRoRows consecutive token rows of one chunk of one
// (side, sequence, KV head); units are ordered (side, b, h, chunk k, sub) with
// chunk k of the reordered order.  A warp takes a contiguous range of units,
// copies the rows of the next units into its shared-memory ring with
// cp.async (4 lanes x 64 bytes per row), and writes each unit to its class's
// segment: FP16 rows copied, INT4 / INT2 rows quantized, 32 values per lane.
// The class is the same for a whole unit, so every code path is
// warp-uniform.
constexpr int kRoRows = 8, kRoLanes = 4, kRoNV = 32, kRoDepth = 4, kRoWarps = 4;
constexpr int kRoUnitBytes = kRoRows * kHeadDim * 2;

// A position in a warp's unit sequence, advanced one unit at a time.
struct RoPos {
  int side, b, h, k, sub;
  __device__ __forceinline__ void start(const ReorderDev& a, long long u, int upc) {
    sub = (int)(u % upc);
    u /= upc;
    k = (int)(u % a.n_chunks);
    u /= a.n_chunks;
    h = (int)(u % a.kv_heads);
    u /= a.kv_heads;
    b = (int)(u % a.batch);
    side = (int)(u / a.batch);
  }
  // true when the next unit starts another chunk
  __device__ __forceinline__ bool step(const ReorderDev& a, int upc) {
    if (++sub < upc) return false;
    sub = 0;
    if (++k == a.n_chunks) {
      k = 0;
      if (++h == a.kv_heads) {
        h = 0;
        if (++b == a.batch) {
          b = 0;
          ++side;
        }
      }
    }
    return true;
  }
  __device__ __forceinline__ long long bh(const ReorderDev& a) const {
    return (long long)b * a.kv_heads + h;
  }
};

// Copy side: the first source row of the unit, read from the chunk's
// original position (perm).
struct RoSrc {
  RoPos p;
  const uint4* src;
  __device__ __forceinline__ void locate(const ReorderDev& a) {
    const int src_chunk = a.perm[(long long)p.b * a.n_chunks + p.k];
    src = reinterpret_cast<const uint4*>(
        (p.side ? a.v_src : a.k_src) +
        (p.bh(a) * a.context_len + (long long)src_chunk * a.chunk_tokens + p.sub * kRoRows) *
            kHeadDim);
  }
  __device__ __forceinline__ void advance(const ReorderDev& a, int upc) {
    if (p.step(a, upc))
      locate(a);
    else
      src += kRoRows * (kHeadDim / 8);
  }
};

// Write side: the unit's segment (class) and its first destination row.
struct RoDst {
  RoPos p;
  int seg;
  long long row;  // destination row of the unit's first token in segment seg
  __device__ __forceinline__ void locate(const ReorderDev& a) {
    const int n16 = a.lens[0][p.b] / a.chunk_tokens;
    const int n4 = a.lens[1][p.b] / a.chunk_tokens;
    seg = p.k < n16 ? 0 : (p.k < n16 + n4 ? 1 : 2);
    const int pos = p.k - (seg == 0 ? 0 : (seg == 1 ? n16 : n16 + n4));
    row = p.bh(a) * a.max_tokens[seg] + (long long)pos * a.chunk_tokens + p.sub * kRoRows;
  }
  __device__ __forceinline__ void advance(const ReorderDev& a, int upc) {
    if (p.step(a, upc))
      locate(a);
    else
      row += kRoRows;
  }
};

template <int G>
__device__ __forceinline__ void ro_work(const ReorderDev& a, int li, int ri, const RoDst& c,
                                        const uint32_t (&roff)[kRoNV / 8], const uint8_t* slot) {
  uint4 raw[kRoNV / 8];
#pragma unroll
  for (int k = 0; k < kRoNV / 8; ++k) raw[k] = *reinterpret_cast<const uint4*>(slot + roff[k]);
  const long long row = c.row + ri;
  const bool ok = (row - c.p.bh(a) * a.max_tokens[c.seg]) < a.max_tokens[c.seg];
  constexpr int GL = G / kRoNV;  // lanes per group
  constexpr int MB = (kHeadDim / G) * 4;
  if (c.seg == 0) {
    if (ok) {
      uint4* d = reinterpret_cast<uint4*>(a.codes[0][c.p.side] + row * (kHeadDim * 2)) +
                 li * (kRoNV / 8);
#pragma unroll
      for (int k = 0; k < kRoNV / 8; ++k) d[k] = raw[k];
    }
  } else if (c.seg == 1) {
    uint32_t cw[code_words<4, kRoNV>()], m;
    quantize_vals<4, G, kRoNV>(raw, cw, m);
    if (ok) {
      *reinterpret_cast<uint4*>(a.codes[1][c.p.side] + row * (kHeadDim / 2) + li * 16) =
          make_uint4(cw[0], cw[1], cw[2], cw[3]);
      if (li % GL == 0)
        reinterpret_cast<uint32_t*>(a.meta[1][c.p.side] + row * MB)[li / GL] = m;
    }
  } else {
    uint32_t cw[code_words<2, kRoNV>()], m;
    quantize_vals<2, G, kRoNV>(raw, cw, m);
    if (ok) {
      *reinterpret_cast<uint2*>(a.codes[2][c.p.side] + row * (kHeadDim / 4) + li * 8) =
          make_uint2(cw[0], cw[1]);
      if (li % GL == 0)
        reinterpret_cast<uint32_t*>(a.meta[2][c.p.side] + row * MB)[li / GL] = m;
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kRoWarps * 32) chunk_bulk_kernel(const ReorderDev a,
                                                                   long long n_units,
                                                                   long long units_per_warp) {
  __shared__ __align__(16) uint8_t ring[kRoWarps][kRoDepth][kRoUnitBytes];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int li = lane % kRoLanes, ri = lane / kRoLanes;
  const long long first = ((long long)blockIdx.x * kRoWarps + warp) * units_per_warp;
  if (first >= n_units) return;  // the whole warp
  const long long rem = n_units - first;
  const int n = (int)(units_per_warp < rem ? units_per_warp : rem);
  const int upc = a.chunk_tokens / kRoRows;
  const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(&ring[warp][0][0]);
  uint32_t soff[kRoNV / 8], roff[kRoNV / 8];
#pragma unroll
  for (int k = 0; k < kRoNV / 8; ++k) {
    soff[k] = bulk_slot_off(ri, k * kRoLanes + li);
    roff[k] = bulk_slot_off(ri, li * (kRoNV / 8) + k);
  }
  RoSrc ic;  // next unit to copy
  ic.p.start(a, first, upc);
  ic.locate(a);
  RoDst wc;  // next unit to write
  wc.p = ic.p;
  wc.locate(a);
  auto issue = [&](uint32_t slot) {
#pragma unroll
    for (int k = 0; k < kRoNV / 8; ++k)
      cp_async16(slot + soff[k], ic.src + ri * (kHeadDim / 8) + k * kRoLanes + li);
    cp_async_commit();
  };
#pragma unroll
  for (int k = 0; k < kRoDepth - 1; ++k) {
    if (k < n) {
      issue(ring0 + k * kRoUnitBytes);
      ic.advance(a, upc);
    } else {
      cp_async_commit();  // empty group: the wait count stays uniform
    }
  }
  for (int i = 0; i < n; ++i) {
    cp_async_wait<kRoDepth - 2>();  // this lane's copies of unit i have landed
    __syncwarp();                   // ... and every lane's; unit i - 1 is read
    if (i + kRoDepth - 1 < n) {
      issue(ring0 + ((i + kRoDepth - 1) % kRoDepth) * kRoUnitBytes);
      ic.advance(a, upc);
    } else {
      cp_async_commit();
    }
    ro_work<G>(a, li, ri, wc, roff, &ring[warp][i % kRoDepth][0]);
    wc.advance(a, upc);
  }
  cp_async_wait<0>();
}

}  // namespace

cudaError_t launch_chunk_assign(const float* emb, const float* qemb, int batch, int n_chunks,
                                int emb_dim, double alpha, double beta, double* sim,
                                uint8_t* bits, cudaStream_t s) {
  if (emb_dim % 4 != 0) return cudaErrorInvalidValue;  // 16-byte rows for the staged copies
  const size_t smem = (size_t)(n_chunks + emb_dim) * sizeof(double) +
                      2 * (size_t)kAssignThreads * kAssignStride * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(chunk_assign_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
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
  const int G = r.seg[1].k.group_size;
  // chunk_tokens is a multiple of 16 (checked by the caller): whole units.
  // One wave, an equal contiguous range of units per warp.
  const long long n_units = 2LL * r.batch * r.kv_heads * r.n_chunks * (r.chunk_tokens / kRoRows);
  int dev = 0, sms = 0, per_sm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, G == 32 ? chunk_bulk_kernel<32> : (G == 64 ? chunk_bulk_kernel<64>
                                                            : chunk_bulk_kernel<128>),
        kRoWarps * 32, 0);
  if (e != cudaSuccess) return e;
  const long long warps = (long long)sms * (per_sm > 0 ? per_sm : 1) * kRoWarps;
  const long long per_warp = (n_units + warps - 1) / warps;
  const long long blocks = (n_units + per_warp * kRoWarps - 1) / (per_warp * kRoWarps);
  if (G == 32)
    chunk_bulk_kernel<32><<<(unsigned)blocks, kRoWarps * 32, 0, s>>>(a, n_units, per_warp);
  else if (G == 64)
    chunk_bulk_kernel<64><<<(unsigned)blocks, kRoWarps * 32, 0, s>>>(a, n_units, per_warp);
  else
    chunk_bulk_kernel<128><<<(unsigned)blocks, kRoWarps * 32, 0, s>>>(a, n_units, per_warp);
  return cudaGetLastError();
}

}  // namespace kvq
