// kvq_static.cu -- decode attention for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc: a plugin loaded into a host program
// that owns and budgets every byte of device memory, a language binding with
// no device allocator of its own, or a latency-critical serving loop where
// cudaMalloc's implicit device-wide synchronization is not acceptable.  For
// them, kvq_decode_attention_noalloc keeps its scratch (the per-split partial
// results and the error word) in a fixed-size array that lives in this
// library's own device memory, so the caller passes only inputs and outputs.
#include <cuda_runtime.h>

#include <mutex>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

// The scratch array itself.  Every GPU that loads the library holds these
// KVQ_STATIC_SCRATCH_BYTES until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[KVQ_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mutex;

// In host code the array's name is only a host-side stand-in, not a device
// address, so the device address is looked up with the caller's device
// current.  It is looked up on every call (a host-side table read once the
// module is loaded), so a call after a device reset sees the reloaded
// module's array.
kvq_status scratch_address(void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
    return KVQ_ERR_CUDA;
  *out = p;
  return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_cache* segs, int32_t n_segs,
                                                   const void* q, kvq_dtype q_dtype,
                                                   int32_t q_heads, float softmax_scale,
                                                   float* out, float* lse,
                                                   int32_t max_len_hint, void* stream) {
  size_t need = 0;
  kvq_status st = kvq_decode_workspace_bytes(segs, n_segs, q_heads, max_len_hint, &need);
  if (st != KVQ_OK) return st;
  if (need > KVQ_STATIC_SCRATCH_BYTES) return KVQ_ERR_WORKSPACE;  // request beyond the limit
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != KVQ_OK) return st;
  // every argument is checked before anything touches the shared array
  st = kvq::decode_check_args(segs, n_segs, q, q_dtype, q_heads, softmax_scale, out, lse,
                              max_len_hint, scratch, KVQ_STATIC_SCRATCH_BYTES);
  if (st != KVQ_OK) return st;
  // The array keeps the previous call's contents, which may have had another
  // layout.  The decode kernels rewrite every partial slot they hand to a
  // merge; the error word and the counters (at the front) start at zero.
  if (cudaMemsetAsync(scratch, 0, kvq::decode_zeroed_prefix_bytes(segs),
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return kvq_decode_attention(segs, n_segs, q, q_dtype, q_heads, softmax_scale, out, lse,
                              max_len_hint, scratch, KVQ_STATIC_SCRATCH_BYTES, stream);
}
