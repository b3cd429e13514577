// kvq_bulk.cuh -- the prefill (bulk) quantize kernels' load ring and row
// cursors, shared by the group quantizer and the Oaken codec.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"
#include "kvq_quant_core.cuh"

namespace kvq {

// Bulk quantize (prefill).  Work unit: kUnitRows consecutive tokens of one
// (side, sequence, KV head) plane row, whose fp16 rows are contiguous in the
// input and whose codes and (s, z) are contiguous in the cache.  Each warp
// takes a contiguous range of units, one unit per step (4 lanes x 64 bytes
// per row, 32 values per lane), and keeps the next kBulkDepth - 1 units in
// flight as cp.async copies into its own shared-memory ring: each copy
// instruction moves 64 contiguous bytes of every row of the unit, and after
// its own copy group has landed and a warp barrier, each lane reads its 64
// bytes of a row.
constexpr int kBulkNV = 32;                       // values per lane
constexpr int kBulkLanes = kHeadDim / kBulkNV;    // lanes per row
constexpr int kUnitRows = 32 / kBulkLanes;        // rows per unit = per warp step
constexpr int kBulkDepth = 4;                     // ring slots per warp
constexpr int kBulkWarps = 4;                     // warps per CTA
constexpr int kUnitBytes = kUnitRows * kHeadDim * 2;

// A position in a warp's unit sequence: plane row (side, b, h) and unit j
// within it, plus this lane's token t.  Moving one unit steps the addresses
// derived from it by a constant; they are rebuilt from (side, b, h, j) only
// when the position enters the next plane row.
struct BulkPos {
  int side, b, h, j, t;
  __device__ __forceinline__ void start(const QuantArgs& a, int u, int units_per_row, int ri) {
    const int p = u / units_per_row;
    j = u - p * units_per_row;
    const int planes = a.batch * a.kv_heads;
    side = p >= planes;
    const int bh = side ? p - planes : p;
    b = bh / a.kv_heads;
    h = bh - b * a.kv_heads;
    t = j * kUnitRows + ri;
  }
  // true when the next unit is in the same plane row (t advanced), false
  // when the position moved to the next plane row (t reset)
  __device__ __forceinline__ bool step(const QuantArgs& a, int units_per_row, int ri) {
    if (++j < units_per_row) {
      t += kUnitRows;
      return true;
    }
    j = 0;
    t = ri;
    if (++h == a.kv_heads) {
      h = 0;
      if (++b == a.batch) {
        b = 0;
        ++side;
      }
    }
    return false;
  }
  __device__ __forceinline__ long long bh(const QuantArgs& a) const {
    return (long long)b * a.kv_heads + h;
  }
};

// The copy side: chunk 0 of this lane's input row.
struct BulkSrc {
  BulkPos p;
  const uint4* src;
  __device__ __forceinline__ void locate(const QuantArgs& a) {
    src = reinterpret_cast<const uint4*>((p.side ? a.v_new : a.k_new) +
                                         (p.bh(a) * a.n_new + p.t) * kHeadDim);
  }
  __device__ __forceinline__ void advance(const QuantArgs& a, int units_per_row, int ri) {
    if (p.step(a, units_per_row, ri))
      src += kUnitRows * (kHeadDim / 8);
    else
      locate(a);
  }
};

// The write side: this lane's code bytes and its row's (s, z) words.  Rows
// at or past max_tokens are never written, so their addresses may run past
// the cache.
template <int RB_, int MB_>
struct BulkDst {
  static constexpr int RB = RB_;  // code bytes per row
  static constexpr int MB = MB_;  // metadata bytes per row
  static constexpr int LB = RB / kBulkLanes;  // code bytes per lane
  BulkPos p;
  int pos;
  bool skip;  // a per-channel-K cache's sequence off a block boundary
  uint8_t* codes;
  uint8_t* meta;
  __device__ __forceinline__ void locate(const QuantArgs& a, int li) {
    const int base = a.seq_lens[p.b];
    skip = a.k_channels && base % kChannelBlock != 0;
    pos = base + p.t;
    const long long row = p.bh(a) * a.max_tokens + pos;
    codes = (p.side ? a.v_codes : a.k_codes) + row * RB + li * LB;
    meta = (p.side ? a.v_meta : a.k_meta) + row * MB;
  }
  __device__ __forceinline__ void advance(const QuantArgs& a, int units_per_row, int ri,
                                          int li) {
    if (p.step(a, units_per_row, ri)) {
      pos += kUnitRows;
      codes += kUnitRows * RB;
      meta += kUnitRows * MB;
    } else {
      locate(a, li);
    }
  }
};

__device__ __forceinline__ void bulk_issue(const QuantArgs& a, const BulkSrc& c,
                                           const uint32_t (&soff)[kBulkNV / 8], int li,
                                           uint32_t slot) {
  if (c.p.t < a.n_new) {
#pragma unroll
    for (int k = 0; k < kBulkNV / 8; ++k) cp_async16(slot + soff[k], c.src + k * kBulkLanes + li);
  }
  cp_async_commit();
}


// The ring loop of a bulk kernel: each warp takes units [first, first + n)
// of the 2 * batch * kv_heads * units_per_row units (side 0 first, from
// a.side0), keeps kBulkDepth - 1 units in flight as cp.async copies into its
// ring slots, and calls work(dst, slot) for each unit once its copies have
// landed; `ring` is the warp's kBulkDepth slots of kUnitBytes.
template <class Dst, class Work>
__device__ __forceinline__ void bulk_loop(const QuantArgs& a, int units_per_row, int n_units,
                                          int units_per_warp, uint8_t* ring, Work&& work) {
  const int lane = threadIdx.x & 31;
  const int li = lane % kBulkLanes, ri = lane / kBulkLanes;
  const long long gw = (long long)blockIdx.x * kBulkWarps + (threadIdx.x >> 5);
  const long long first_ll = gw * units_per_warp;
  if (first_ll >= n_units) return;  // the whole warp
  const int first = (int)first_ll;
  const int n = min(units_per_warp, n_units - first);
  const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(ring);
  // this lane's chunk offsets in a ring slot: the chunks it copies, the
  // chunks it reads
  uint32_t soff[kBulkNV / 8], roff[kBulkNV / 8];
#pragma unroll
  for (int k = 0; k < kBulkNV / 8; ++k) {
    soff[k] = bulk_slot_off(ri, k * kBulkLanes + li);
    roff[k] = bulk_slot_off(ri, li * (kBulkNV / 8) + k);
  }
  BulkSrc ic;  // next unit to copy (units of side 0 precede those of side 1)
  ic.p.start(a, first + a.side0 * a.batch * a.kv_heads * units_per_row, units_per_row, ri);
  ic.locate(a);
  Dst wc;  // next unit to quantize
  wc.p = ic.p;
  wc.locate(a, li);
#pragma unroll
  for (int k = 0; k < kBulkDepth - 1; ++k) {
    if (k < n) {
      bulk_issue(a, ic, soff, li, ring0 + k * kUnitBytes);
      ic.advance(a, units_per_row, ri);
    } else {
      cp_async_commit();  // empty group: the wait count stays uniform
    }
  }
  for (int i = 0; i < n; ++i) {
    cp_async_wait<kBulkDepth - 2>();  // this lane's copies of unit i have landed
    __syncwarp();                     // ... and every lane's; unit i - 1 is read
    // refill the slot of unit i - 1 (read in the previous step) with unit
    // i + kBulkDepth - 1
    if (i + kBulkDepth - 1 < n) {
      bulk_issue(a, ic, soff, li, ring0 + ((i + kBulkDepth - 1) % kBulkDepth) * kUnitBytes);
      ic.advance(a, units_per_row, ri);
    } else {
      cp_async_commit();
    }
    work(wc, roff, ring + (i % kBulkDepth) * kUnitBytes);
    wc.advance(a, units_per_row, ri, li);
  }
  cp_async_wait<0>();
}

// Launch shape of a bulk kernel: every resident warp takes an equal
// contiguous range of units (one wave).
struct BulkShape {
  int units_per_row, n_units, per_warp;
  unsigned blocks;
};
inline bool bulk_shape(const QuantArgs& a, int ctas_per_sm, BulkShape* sh) {
  sh->units_per_row = (a.n_new + kUnitRows - 1) / kUnitRows;
  const long long n_units = (2LL - a.side0) * a.batch * a.kv_heads * sh->units_per_row;
  if (n_units > 0x3fffffffLL) return false;
  sh->n_units = (int)n_units;
  const long long warps = (long long)device_sm_count() * (ctas_per_sm > 0 ? ctas_per_sm : 1) *
                          kBulkWarps;
  const long long per_warp = (n_units + warps - 1) / warps;
  sh->per_warp = (int)(per_warp > 0 ? per_warp : 1);
  sh->blocks = (unsigned)((n_units + (long long)sh->per_warp * kBulkWarps - 1) /
                          ((long long)sh->per_warp * kBulkWarps));
  return true;
}

// Host side: launch `kernel` as a programmatic dependent of the kernel before
// it on the stream.  It may be scheduled once that kernel's CTAs have all
// signalled (grid_dependents_may_launch) or exited, so it must call
// grid_dependency_wait() before it touches memory that kernel writes.
template <class... KArgs, class... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                    cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace kvq
