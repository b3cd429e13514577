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
//   oaken_quantize_kernel: quantize-on-write, half a warp per row (8 dims a
//     lane), the outliers' slots placed by a shuffle scan of the lanes'
//     counts.  HBM-bound: 256 B read and 96 B written per row.
//   The decode attention over these planes is the tokens-on-M kernel's
//     (kvq_decode_tm.cu): the dense codes through the tensor cores like
//     INT4 with the plane's one (s, z), the K slots as per-token score
//     terms, the V slots scattered into a dense tile that the tensor cores
//     add to the output.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant_core.cuh"

namespace kvq {

namespace {

constexpr int D = kHeadDim;
constexpr int kSlots = KVQ_OAKEN_SLOTS;
constexpr int kRowBytes = D / 2;         // 4-bit codes of one row
constexpr int kSlotBytes = kSlots * 2;   // outlier slots of one row

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
    const __half* hv = reinterpret_cast<const __half*>(&raw);
    uint32_t word = 0, flags = 0;
    int dv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      bool o;
      word |= oaken_code(__half2float(hv[e]), p, dv[e], o) << (4 * e);
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

__global__ void oaken_advance_kernel(int32_t* seq_lens, int batch, int n_new, int max_tokens) {
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

cudaError_t launch_oaken_quantize(const QuantArgs& a, cudaStream_t s) {
  const long long rows = 2LL * a.batch * a.kv_heads * a.n_new;
  const long long blocks = (rows + 15) / 16;
  const long long cap = (long long)device_sm_count() * 8;
  const unsigned grid = (unsigned)(blocks < cap ? blocks : cap);
  oaken_quantize_kernel<<<grid, 256, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !a.advance) return e;
  oaken_advance_kernel<<<(a.batch + 127) / 128, 128, 0, s>>>(a.seq_lens, a.batch, a.n_new,
                                                             a.max_tokens);
  return cudaGetLastError();
}

}  // namespace kvq
