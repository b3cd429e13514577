// kvq_internal.h -- launch interfaces between the C ABI (kvq_abi.cu) and the
// kernels.  Host-visible structs only; no device code here.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

// Kernel template tag of the FP8 E4M3 code format (8-bit codes); the integer
// formats use their bit width (2, 4, 8) and raw fp16 rows use 16.
constexpr int kE4M3 = 0x108;
// symmetric INT8 codes (two's complement bytes, zero point 0); code_bits 8
constexpr int kSym8 = 0x208;
// FP8 E5M2 codes (bias 15, two mantissa bits); code_bits 8
constexpr int kE5M2 = 0x308;
// the Oaken group-shift codec (4-bit dense codes plus outlier slots)
constexpr int kOaken = 0x404;
__host__ __device__ constexpr int code_bits(int tag) { return tag & 0xFF; }

// A KVQ_FMT_OAKEN plane's offline parameters as the kernels use them:
// T_lo = -z s_in, T_hi = (15 - z) s_in, r_in = 1 / s_in (rounded to
// nearest), outlier magnitudes up to m_max = 2^b - 1.
struct OakenParams {
  float s_in, r_in, z, t_lo, t_hi, s_out, m_max;
};
OakenParams make_oaken_params(float s_in, int z_in, float s_out, int outer_bits);

// One K/V plane pair of one cache segment, as the kernels see it.
struct SegView {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const uint8_t* k_meta;  // (scale, zero) fp16 pairs; null for bits 16
  const uint8_t* v_meta;
  const int32_t* seq_lens;
  int32_t bits;
  int32_t group;
  int32_t max_tokens;
  int32_t n_split;       // units (splits) per (sequence, KV head)
  int32_t part_base;     // index of this segment's first partial slot
  int32_t k_channels;    // K grouped per channel over kChannelBlock-token blocks
  int32_t sms;           // streaming multiprocessors of the device
  OakenParams k_oaken, v_oaken;  // bits == kOaken: the planes' parameters
  // this segment's pair of work counters (next unit, CTAs done) in the
  // workspace header: words ctr, ctr + 1 after the error word at word 0
  int32_t ctr;
  // launched as a programmatic dependent of the previous segment's kernel
  // (several segments in one call): its CTAs may run beside that kernel's,
  // and it waits for that kernel before it exits
  int32_t after_prev;
};

// Launch a split-K decode kernel: a plain launch, or (after_prev) a
// programmatic dependent of the kernel before it on the stream.
template <class Kernel, class Params>
inline cudaError_t launch_segment_kernel(Kernel kernel, unsigned grid, unsigned block, size_t smem,
                                         cudaStream_t s, bool after_prev, const Params& p) {
  if (!after_prev) {
    kernel<<<grid, block, smem, s>>>(p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// warps of a decode CTA
constexpr int kWarpsPerCta = 4;
// SM count assumed when no device can be queried (a B200 has 148)
constexpr int kDefaultSms = 148;

struct DecodeArgs {
  int32_t batch, kv_heads, q_heads, group_ratio;
  const void* q;
  int32_t q_is_bf16;
  float scale_log2;      // softmax_scale * log2(e)
  int32_t parts;         // partial results per (sequence, query head)
  float* part_ml;        // [batch][q_heads][parts][2] (max in log2 units, sum)
  float* part_o;         // [batch][q_heads][parts][head_dim], unnormalised
  float* out;            // [batch][q_heads][head_dim]
  float* lse;            // [batch][q_heads] or null
  uint32_t* err;         // sticky device error word
  // decode step: one new token per (sequence, KV head), quantized into the
  // cache by the unit whose token range covers its position; seq_cnt[b]
  // counts finished units of sequence b, and the last one advances
  // seq_lens[b] (null k_new: no append)
  const __half* k_new;   // [batch][kv_heads][head_dim] fp16
  const __half* v_new;
  uint32_t* seq_cnt;
};

struct QuantArgs {
  const __half* k_new;
  const __half* v_new;
  uint8_t* k_codes;
  uint8_t* v_codes;
  uint8_t* k_meta;
  uint8_t* v_meta;
  int32_t* seq_lens;
  int32_t batch, kv_heads, max_tokens, n_new;
  int32_t advance;
  // per-channel K (K plane grouped per channel over blocks of
  // kChannelBlock tokens): the per-token kernels then write V only (side0 =
  // 1), and a sequence whose length is not a multiple of the block is not
  // written and not advanced
  int32_t side0;
  int32_t k_channels;
  // k_new and v_new hold bf16 values (else fp16); token-grouped formats only
  int32_t in_bf16;
  OakenParams k_oaken, v_oaken;  // Oaken planes (launch_oaken_quantize)
};
// tokens per block of a per-channel K plane
constexpr int kChannelBlock = 32;

// Per-bit-width launchers (kvq_quantize.cu, kvq_decode.cu, kvq_chunk.cu).
cudaError_t launch_quantize(const QuantArgs& a, int bits, int group, cudaStream_t s);
// kpc: the K plane is grouped per channel (group is then V's group size)
bool decode_supported(int bits, int group, int group_ratio, bool kpc = false);
// resident decode CTAs per SM for a segment format and query-group ratio
int decode_ctas_per_sm(int bits, int group, int group_ratio, bool kpc = false);
// the tokens-on-M kernel (kvq_decode_tm.cu): formats with NG * g <= 8
bool decode_tm_supported(int bits, int group, int group_ratio, bool kpc = false);
int decode_tm_ctas_per_sm(int bits, int group, int group_ratio, bool kpc = false);
cudaError_t launch_decode_segment(const DecodeArgs& a, const SegView& seg, cudaStream_t s);
cudaError_t launch_decode_tm(const DecodeArgs& a, const SegView& seg, cudaStream_t s);
cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t s);
// the Oaken codec (kvq_oaken.cu): quantize-on-write of both planes (and the
// seq_lens advance), and its decode-attention kernel (g = 1, 2, 4, 8)
cudaError_t launch_oaken_quantize(const QuantArgs& a, cudaStream_t s);
// kvq_decode_attention's argument checks only: KVQ_OK means a call with the
// same arguments enqueues its kernels (kvq_abi.cu)
kvq_status decode_check_args(const kvq_cache* segs, int32_t n_segs, const void* q,
                             kvq_dtype q_dtype, int32_t q_heads, float softmax_scale, float* out,
                             float* lse, int32_t max_len_hint, void* workspace,
                             size_t workspace_bytes);
// streaming multiprocessors of the current device (kvq_abi.cu)
int device_sm_count();
// leading workspace bytes that hold the header and the counters (they must
// be zero before a call whose cache shape differs from the previous call's)
size_t decode_zeroed_prefix_bytes(const kvq_cache* segs);
cudaError_t launch_chunk_assign(const float* emb, const float* qemb, int batch, int n_chunks,
                                int emb_dim, double alpha, double beta, double* sim,
                                uint8_t* bits, cudaStream_t s);
struct ReorderArgs {
  const __half* k_src;
  const __half* v_src;
  const uint8_t* chunk_bits;
  int32_t* perm;
  kvq_cache seg[3];
  int32_t batch, kv_heads, context_len, chunk_tokens, n_chunks;
};
cudaError_t launch_chunk_reorder(const ReorderArgs& a, cudaStream_t s);

}  // namespace kvq
