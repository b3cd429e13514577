// kvq_oaken.cu -- the Oaken group-shift codec ("大模型KV缓存量化技术：原理、
// 优化与实践" page: section 3.1, thresholds fixed offline and applied online
// with group-shift quantization and a dense-sparse encoding; 3.2.1, the
// outer zone at 5-7 bits, the inner and middle zones at 4 bits; 3.2.2, the
// outer values shifted by the threshold they crossed, Delta = value - T_hi
// or value - T_lo, and dequantized as T + Delta * scale).
//
// Encoding of one token row of head_dim values with the plane's offline
// (s_in, z_in, s_out, b): T_lo = -z_in s_in, T_hi = (15 - z_in) s_in.
//   T_lo <= v <= T_hi: code c = clamp(rne(v / s_in) + z_in, 0, 15);
//   v > T_hi: c = 15, outlier +min(rne((v - T_hi) / s_out), 2^b - 1);
//   v < T_lo: c = 0,  outlier -min(rne((T_lo - v) / s_out), 2^b - 1).
// Dense part: the 4-bit codes, packed two per byte (low nibble first).
// Sparse part: KVQ_OAKEN_SLOTS 16-bit slots per row, the outliers in
// ascending dim order (dim in the low byte, signed magnitude in the high
// byte), zeros after them; outliers past the last slot are dropped.
// x_hat = (c - z_in) s_in + d s_out, d = the element's slot value: for an
// outlier the dense part is its threshold and the slot adds the shift.
//
// Kernels:
//   oaken_quantize_kernel: quantize-on-write of a few rows per sequence
//     (the decode-step append), half a warp per row (8 dims a lane), the
//     outliers' slots placed by a shuffle scan of the lanes' counts.
//   oaken_bulk_kernel: the prefill, on the bulk quantizer's load ring (four
//     lanes per row, 32 dims a lane), dense codes branch-free, outliers in
//     a compact per-lane loop.  HBM-bound: 256 B read and 96 B written per
//     row.
//   Both take fp16 or bf16 rows (BF), widened to fp32 exactly.
//   The decode attention over these planes is the tokens-on-M kernel's
//     (kvq_decode_tm.cu): the dense codes through the tensor cores like
//     INT4 with the plane's one (s, z), the K slots as per-token score
//     terms, the V slots scattered into a dense tile that the tensor cores
//     add to the output.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "kvq_bulk.cuh"
#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant_core.cuh"

namespace kvq {

namespace {

constexpr int D = kHeadDim;
constexpr int kSlots = KVQ_OAKEN_SLOTS;
constexpr int kRowBytes = D / 2;         // 4-bit codes of one row
constexpr int kSlotBytes = kSlots * 2;   // outlier slots of one row

// A 16-bit input element (fp16, or bf16 with BF) widened to fp32, exactly.
template <bool BF>
__device__ __forceinline__ float in_f32(uint16_t h) {
  if constexpr (BF)
    return __uint_as_float((uint32_t)h << 16);
  else
    return __half2float(__ushort_as_half(h));
}

// One element: its 4-bit code, and its signed outlier magnitude (0 inside).
__device__ __forceinline__ uint32_t oaken_code(float v, const OakenParams& p, int& d,
                                               bool& outlier) {
  if (v > p.t_hi) {
    const float m = fminf(rintf(__fdiv_rn(v - p.t_hi, p.s_out)), p.m_max);
    d = (int)m;
    outlier = true;
    return 15u;
  }
  if (v < p.t_lo) {
    const float m = fminf(rintf(__fdiv_rn(-(v - p.t_lo), p.s_out)), p.m_max);
    d = -(int)m;
    outlier = true;
    return 0u;
  }
  // the IEEE quotient by the fp16 scale (div_rn with its reciprocal), then
  // round half to even and the integer zero point
  const float c = fminf(fmaxf(rintf(div_rn(v, p.s_in, p.r_in)) + p.z, 0.0f), 15.0f);
  d = 0;
  outlier = false;
  return (uint32_t)c;
}

// Half a warp per row: lane li of the half owns dims 8 li .. 8 li + 7.
template <bool BF>
__global__ void __launch_bounds__(256) oaken_quantize_kernel(const QuantArgs a) {
  const int lane = threadIdx.x & 31;
  const int li = lane & 15;
  const unsigned half_mask = (lane < 16) ? 0x0000FFFFu : 0xFFFF0000u;
  const long long per_plane = (long long)a.batch * a.kv_heads * a.n_new;
  const long long rows = 2 * per_plane;
  const long long stride = (long long)gridDim.x * (blockDim.x / 16);
  for (long long r = (long long)blockIdx.x * (blockDim.x / 16) + (threadIdx.x >> 4); r < rows;
       r += stride) {
    const int plane = r >= per_plane;
    const long long rr = plane ? r - per_plane : r;
    const int i = (int)(rr % a.n_new);
    const long long bh = rr / a.n_new;
    const int b = (int)(bh / a.kv_heads);
    const int pos = a.seq_lens[b] + i;
    if (pos >= a.max_tokens) continue;  // the whole half-warp skips together
    const OakenParams& p = plane ? a.v_oaken : a.k_oaken;
    const __half* src = (plane ? a.v_new : a.k_new) + rr * D;
    const long long dst_row = bh * a.max_tokens + pos;
    uint8_t* codes = (plane ? a.v_codes : a.k_codes) + dst_row * kRowBytes;
    uint16_t* slots =
        reinterpret_cast<uint16_t*>((plane ? a.v_meta : a.k_meta) + dst_row * kSlotBytes);

    const uint4 raw = reinterpret_cast<const uint4*>(src)[li];
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw);
    uint32_t word = 0, flags = 0;
    int dv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      bool o;
      word |= oaken_code(in_f32<BF>(hv[e]), p, dv[e], o) << (4 * e);
      flags |= (uint32_t)o << e;
    }
    reinterpret_cast<uint32_t*>(codes)[li] = word;
    // slot positions: exclusive prefix of the lanes' outlier counts
    const int cnt = __popc(flags);
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) {
      const int t = __shfl_up_sync(half_mask, incl, off, 16);
      if (li >= off) incl += t;
    }
    const int total = __shfl_sync(half_mask, incl, 15, 16);
    int k = incl - cnt;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if ((flags >> e) & 1u) {
        if (k < kSlots)
          slots[k] = (uint16_t)((uint32_t)(8 * li + e) | ((uint32_t)(uint8_t)(int8_t)dv[e] << 8));
        ++k;
      }
    if (li >= total) slots[li] = 0;  // kSlots == 16 lanes: one empty slot each
  }
}

// Bulk (prefill) encoder: the bulk ring's units (kUnitRows consecutive rows
// of one (side, sequence, KV head) plane row, 4 lanes per row, 32
// consecutive dims a lane).  Per pair of fp16 values: clamped to the
// thresholds in fp16 (th = the largest fp16 <= T_hi, tl = the smallest >=
// T_lo: an fp16 value lies outside [T_lo, T_hi] exactly when it lies outside
// [tl, th]), the clamp also flagging the outliers; then the dense code
// rint(clamped / s_in) + z_in in packed f32x2 arithmetic -- an inner value
// keeps its own code, and th and tl divide to within 15/1024 of 15 - z_in
// and -z_in, so an outlier gets its threshold's code.  The outliers of the
// warp's 8 rows are then listed in shared memory (each with its row, its
// place among the row's outliers in dim order -- a scan of the row's lanes
// -- and its dim) and settled 32 at a time across the whole warp; the slot
// rows are assembled in shared memory, whose zeros stand for the empty
// slots, and go out as 8-byte stores.
using OakDst = BulkDst<kRowBytes, kSlotBytes>;
constexpr int kOakList = kUnitRows * kSlots;  // outliers a unit can keep

struct OakUnitParams {
  float s_in, r_in, z, t_lo, t_hi, s_out, m_max;
  uint32_t tl2, th2;  // pairs (tl, tl) and (th, th) in the input's 16-bit type
};

template <bool BF>
__device__ __forceinline__ OakUnitParams oaken_unit_params(const OakenParams& p) {
  OakUnitParams u;
  u.s_in = p.s_in;
  u.r_in = p.r_in;
  u.z = p.z;
  u.t_lo = p.t_lo;
  u.t_hi = p.t_hi;
  u.s_out = p.s_out;
  u.m_max = p.m_max;
  if constexpr (BF) {
    const uint32_t tl = __bfloat16_as_ushort(__float2bfloat16_ru(p.t_lo));
    const uint32_t th = __bfloat16_as_ushort(__float2bfloat16_rd(p.t_hi));
    u.tl2 = tl | (tl << 16);
    u.th2 = th | (th << 16);
  } else {
    const __half tl = __float2half_ru(p.t_lo), th = __float2half_rd(p.t_hi);
    u.tl2 = h2_as_u32(__halves2half2(tl, tl));
    u.th2 = h2_as_u32(__halves2half2(th, th));
  }
  return u;
}

template <bool BF>
__device__ __forceinline__ void oaken_work(const QuantArgs& a, int lane, const OakDst& c,
                                           const uint32_t (&roff)[kBulkNV / 8],
                                           const uint8_t* slot, uint16_t* sbuf,
                                           uint16_t* olist) {
  static_assert(kBulkNV == 32 && kBulkLanes == 4 && kSlots == 16, "lane and slot layout");
  const int li = lane % kBulkLanes, ri = lane / kBulkLanes;
  const bool in = c.p.t < a.n_new;
  // the unit's plane parameters in registers (one side per unit)
  const OakUnitParams p = oaken_unit_params<BF>(c.p.side ? a.v_oaken : a.k_oaken);
  using IP = InPair<BF>;
  uint4 raw[kBulkNV / 8];
#pragma unroll
  for (int k = 0; k < kBulkNV / 8; ++k)
    raw[k] = in ? *reinterpret_cast<const uint4*>(slot + roff[k]) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw[0]);  // pair i: elements 2i, 2i + 1
  // clamp in fp16; bit i / 16 + i of omask: element 2i / 2i + 1 is an outlier
  // (reordered to dim order below)
  float x[kBulkNV];
  uint32_t omask = 0;
#pragma unroll
  for (int i = 0; i < kBulkNV / 2; ++i) {
    const uint32_t cl = IP::min2(IP::max2(w[i], p.tl2), p.th2);
    uint32_t ne;
    if constexpr (BF)
      ne = __hne2_mask(*reinterpret_cast<const __nv_bfloat162*>(&cl),
                       *reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    else
      ne = __hne2_mask(u32_as_h2(cl), u32_as_h2(w[i]));
    omask |= ne & (0x00010001u << i);
    const float2 f = IP::widen(cl);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint64_t r2 = f2_pack(p.r_in, p.r_in), nd2 = f2_pack(-p.s_in, -p.s_in);
  const uint64_t m2 = f2_pack(kMagic, kMagic);
  const float zm = p.z - kMagic;
  const uint64_t zm2 = f2_pack(zm, zm);
  uint64_t t[kBulkNV / 2];  // pair i: elements i and i + 16 (the packing's order)
#pragma unroll
  for (int i = 0; i < kBulkNV / 2; ++i)
    // quotients within [-z_in, 15 - z_in]: (q + M) + (z_in - M) is rint(q) + z_in
    t[i] = f2_add(f2_add(div_rn2(f2_pack(x[i], x[i + kBulkNV / 2]), nd2, r2), m2), zm2);
  uint32_t cw[code_words<4, kBulkNV>()];
  pack_codes<4, kBulkNV>(t, cw);
  if (!in) omask = 0;
  // bit j: element j (dim 32 li + j) is an outlier -- the even elements'
  // bits spread to the even positions, the odd ones' to the odd
  auto spread = [](uint32_t v) {  // bit i of a 16-bit value to bit 2i
    v = (v | (v << 8)) & 0x00FF00FFu;
    v = (v | (v << 4)) & 0x0F0F0F0Fu;
    v = (v | (v << 2)) & 0x33333333u;
    return (v | (v << 1)) & 0x55555555u;
  };
  omask = spread(omask & 0xFFFFu) | (spread(omask >> 16) << 1);
  // places among the row's outliers (dim order: lanes in order); the first
  // kSlots are kept, and the kept ones get places in the warp's list
  const int cnt = __popc(omask);
  int incl = cnt;
  {
    const int u1 = __shfl_up_sync(0xffffffffu, incl, 1, kBulkLanes);
    if (li >= 1) incl += u1;
    const int u2 = __shfl_up_sync(0xffffffffu, incl, 2, kBulkLanes);
    if (li >= 2) incl += u2;
  }
  const int kept = max(0, min(cnt, kSlots - (incl - cnt)));
  int wincl = kept;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, wincl, off);
    if (lane >= off) wincl += u;
  }
  const int total = __shfl_sync(0xffffffffu, wincl, 31);
  uint16_t* srow = sbuf + ri * kSlots;
  reinterpret_cast<uint2*>(srow)[li] = make_uint2(0u, 0u);  // slots 4 li .. 4 li + 3
  // list entry: row (bits 0-2), place in the row (bits 3-7), dim (bits 8-14);
  // outliers past the row's kSlots-th are dropped (their dense code is
  // their threshold's)
  {
    int k = incl - cnt, e = wincl - kept;
    uint32_t m = omask;
    for (int n = 0; n < kept; ++n) {
      const int j = __ffs(m) - 1;
      m &= m - 1u;
      olist[e++] = (uint16_t)(ri | (k++ << 3) | ((kBulkNV * li + j) << 8));
    }
  }
  __syncwarp();
  for (int e = lane; e < total; e += 32) {
    const uint32_t en = olist[e];
    const int r = en & 7, k = (en >> 3) & 31, dim = (int)(en >> 8);
    const float v = in_f32<BF>(
        *reinterpret_cast<const uint16_t*>(slot + bulk_slot_off(r, dim >> 3) + (dim & 7) * 2));
    const bool hi = v > p.t_hi;
    const float mq = fminf(rintf(__fdiv_rn(hi ? v - p.t_hi : -(v - p.t_lo), p.s_out)), p.m_max);
    const int d = hi ? (int)mq : -(int)mq;
    sbuf[r * kSlots + k] = (uint16_t)((uint32_t)dim | ((uint32_t)(uint8_t)(int8_t)d << 8));
  }
  __syncwarp();
  if (in && c.pos < a.max_tokens) {
    *reinterpret_cast<uint4*>(c.codes) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    reinterpret_cast<uint2*>(c.meta)[li] = reinterpret_cast<const uint2*>(srow)[li];
  }
  __syncwarp();  // the slot rows and the list are rewritten by the next unit
}

template <bool BF>
__global__ void __launch_bounds__(kBulkWarps * 32) oaken_bulk_kernel(const QuantArgs a,
                                                                     int units_per_row,
                                                                     int n_units,
                                                                     int units_per_warp) {
  __shared__ __align__(16) uint8_t ring[kBulkWarps][kBulkDepth][kUnitBytes];
  __shared__ __align__(16) uint16_t sbuf[kBulkWarps][kUnitRows][kSlots];
  __shared__ __align__(16) uint16_t olist[kBulkWarps][kOakList];
  grid_dependents_may_launch();  // the seq_lens update may be scheduled
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  bulk_loop<OakDst>(a, units_per_row, n_units, units_per_warp, &ring[warp][0][0],
                    [&](const OakDst& c, const uint32_t (&roff)[kBulkNV / 8],
                        const uint8_t* slot) {
                      oaken_work<BF>(a, lane, c, roff, slot, &sbuf[warp][0][0], &olist[warp][0]);
                    });
}

__global__ void oaken_advance_kernel(int32_t* seq_lens, int batch, int n_new, int max_tokens) {
  grid_dependency_wait();  // the quantizer before it reads seq_lens
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch) seq_lens[b] = min(seq_lens[b] + n_new, max_tokens);
}

}  // namespace

OakenParams make_oaken_params(float s_in, int z_in, float s_out, int outer_bits) {
  OakenParams p;
  p.s_in = s_in;
  p.r_in = 1.0f / s_in;  // host IEEE division: the correctly rounded reciprocal
  p.z = (float)z_in;
  p.t_lo = -p.z * s_in;
  p.t_hi = (15.0f - p.z) * s_in;
  p.s_out = s_out;
  p.m_max = (float)((1 << outer_bits) - 1);
  return p;
}

namespace {

template <bool BF>
cudaError_t launch_oaken(const QuantArgs& a, cudaStream_t s) {
  cudaError_t e;
  if (a.n_new < kUnitRows) {
    // a few rows per sequence (the decode-step append): half a warp per row
    const long long rows = 2LL * a.batch * a.kv_heads * a.n_new;
    const long long blocks = (rows + 15) / 16;
    const long long cap = (long long)device_sm_count() * 8;
    const unsigned grid = (unsigned)(blocks < cap ? blocks : cap);
    oaken_quantize_kernel<BF><<<grid, 256, 0, s>>>(a);
  } else {
    static int per_sm = 0;  // resident CTAs per SM of the bulk kernel
    if (per_sm == 0) {
      int r = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&r, oaken_bulk_kernel<BF>,
                                                        kBulkWarps * 32, 0);
      if (e != cudaSuccess) return e;
      per_sm = r > 0 ? r : 1;
    }
    BulkShape sh;
    if (!bulk_shape(a, per_sm, &sh)) return cudaErrorInvalidValue;
    oaken_bulk_kernel<BF><<<sh.blocks, kBulkWarps * 32, 0, s>>>(a, sh.units_per_row, sh.n_units,
                                                                sh.per_warp);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || !a.advance) return e;
  // a programmatic dependent: scheduled while the quantizer runs
  return launch_dependent(oaken_advance_kernel, dim3((a.batch + 127) / 128), dim3(128), s,
                          a.seq_lens, a.batch, a.n_new, a.max_tokens);
}

}  // namespace

cudaError_t launch_oaken_quantize(const QuantArgs& a, cudaStream_t s) {
  return a.in_bf16 ? launch_oaken<true>(a, s) : launch_oaken<false>(a, s);
}

}  // namespace kvq
