/*
 * kvq.h -- C ABI of libkvq: a group-quantized KV cache and decode attention
 * that reads it, for NVIDIA B200 (sm_100a).
 *
 * What the library computes (pages cited by title and section):
 *  - Group-wise asymmetric quantization of K and V as they are written:
 *    quant(x) = round(x/s) + z with one scale s and zero point z per group
 *    (Cocktail page, peacm.com news 1099647, section 3.2.2; the TurboQuant
 *    page, bhfrc.com news 57821, section 2.3, "one scale per group";
 *    s = (max - min) / (2^bits - 1), "大模型KV缓存量化技术" page section 2.1;
 *    s floored at 1e-5, "大模型推理加速之KV Cache量化压缩原理与工程实现" page,
 *    troubleshooting).
 *  - Single-query decode attention straight over the packed codes, the
 *    dequantization folded into the QK^T and PV products instead of a
 *    separate pass (TurboQuant page 2.3, last paragraph), split over the
 *    token axis and merged by log-sum-exp (Cocktail page 3.2.3: block-wise
 *    attention merged is equal to the unchunked computation).
 *  - Cocktail's chunk-level mixed precision: per-chunk FP16/INT4/INT2 class
 *    from the cosine similarity of chunk and query embeddings with
 *    T_low = s_min + (s_max - s_min) * alpha and
 *    T_high = s_max - (s_max - s_min) * beta (Cocktail page 3.1.1), and the
 *    reorder that makes equal bit-widths contiguous (3.1.2).
 *
 * Numerics (fixed so that codes, scales and zero points are reproducible
 * bit for bit): per group of G fp16 values, in fp32 with IEEE operations:
 *   mn, mx = min, max;  s32 = max((mx - mn) / qmax, 1e-5), qmax = 2^bits - 1;
 *   s = fp16 value of s32 rounded toward +infinity (stored);
 *   z = rint(-mn / s) (+0 for a zero result), clamped to +-65504, stored fp16;
 *   code = clamp(rint(x / s) + z, 0, qmax), rint = round half to even.
 * Dequantized value: (code - z) * s.
 *
 * Conventions for every entry point:
 *  - Ownership: the caller owns every buffer.  The library never allocates,
 *    frees or synchronizes; work is enqueued on the given stream and the
 *    call returns as soon as it is enqueued.  Pointers marked "device" must
 *    be device (or managed) memory of the current device.
 *  - Errors: arguments are validated on the host before anything is
 *    enqueued; a non-OK status means nothing was enqueued (except
 *    KVQ_ERR_CUDA, returned when a launch failed).  No entry point reads
 *    device memory on the host, so values held only on the device (the
 *    sequence lengths) are bounds-checked by the kernels themselves: they
 *    never read or write outside the buffers described here.
 *  - Thread safety: calls on different streams may run concurrently; calls
 *    that share a cache or workspace must be ordered by the caller.
 *  - Streams: `stream` is a cudaStream_t passed as void*; NULL is the
 *    legacy default stream.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned buffer   */
    KVQ_ERR_UNSUPPORTED = 2, /* valid but not built: (bits, G, head_dim, g) */
    KVQ_ERR_CAPACITY = 3,    /* a host-known size exceeds the cache         */
    KVQ_ERR_WORKSPACE = 4,   /* workspace missing or too small              */
    KVQ_ERR_CUDA = 5         /* a CUDA launch or runtime call failed        */
} kvq_status;

typedef enum kvq_dtype { KVQ_F16 = 0, KVQ_BF16 = 1 } kvq_dtype;

/* Code format of a plane. */
typedef enum kvq_format {
    KVQ_FMT_INT = 0,      /* asymmetric integer codes: x_hat = (c - z) * s    */
    KVQ_FMT_FP8_E4M3 = 1, /* FP8 E4M3 codes, bits 8: x_hat = e4m3(c) * s      */
    KVQ_FMT_INT8_SYM = 2, /* symmetric INT8 codes, bits 8: x_hat = c * s      */
    KVQ_FMT_FP8_E5M2 = 3, /* FP8 E5M2 codes, bits 8: x_hat = e5m2(c) * s      */
    KVQ_FMT_OAKEN = 4     /* Oaken group-shift codes, bits 4 (see below)     */
} kvq_format;

/* Grouping axis of a plane's (scale, zero point) pairs. */
typedef enum kvq_axis {
    KVQ_AXIS_TOKEN = 0,   /* groups of G along head_dim within a token row    */
    KVQ_AXIS_CHANNEL = 1  /* K only: one group per channel over each block of */
                          /* KVQ_CHANNEL_BLOCK consecutive tokens             */
} kvq_axis;

#define KVQ_CHANNEL_BLOCK 32

/* Outlier slots per token row of a KVQ_FMT_OAKEN plane. */
#define KVQ_OAKEN_SLOTS 16

/*
 * Offline parameters of a KVQ_FMT_OAKEN plane (the "大模型KV缓存量化技术：
 * 原理、优化与实践" page, section 3.1: thresholds fixed before deployment,
 * applied online; 3.2.1: outer zone 5-7 bits, inner and middle 4 bits).
 *   inner_scale s_in: a positive fp16 value (held here as a float);
 *   inner_zero z_in: integer in [0, 15]; the thresholds are T_lo = -z_in *
 *     s_in and T_hi = (15 - z_in) * s_in, both on the inner grid;
 *   outer_scale s_out: positive and finite;
 *   outer_bits b: 5, 6 or 7 (outlier magnitudes up to 2^b - 1).
 * Ignored for the other formats.
 */
typedef struct kvq_oaken {
    float inner_scale;
    int32_t inner_zero;
    float outer_scale;
    int32_t outer_bits;
} kvq_oaken;

/*
 * One K or V plane of a cache (one bit-width).
 *   bits 2, 4, 8: codes  u8  [batch][kv_heads][max_tokens][head_dim*bits/8],
 *                 element j of a token row in byte j*bits/8 at bit offset
 *                 (j*bits) mod 8 (low bits first);
 *                 meta  f16 [batch][kv_heads][max_tokens][head_dim/G][2],
 *                 the pair (scale, zero point) of each group, groups of G
 *                 consecutive head_dim elements of one token row.
 *   bits 8 with fmt KVQ_FMT_FP8_E4M3: one E4M3 code per element (bias 7,
 *                 no infinities, largest finite 448), the same meta layout
 *                 with zero point 0 (the KV-cache page's FP8 KV cache, with
 *                 the scale of each group computed from the values written,
 *                 that page's dynamic quantization).
 *   bits 8 with fmt KVQ_FMT_FP8_E5M2: one E5M2 code per element (bias 15,
 *                 largest finite 57344), the same meta layout with zero
 *                 point 0; the scale of each group is its |max| / 57344
 *                 (floored at 1e-5, fp16 rounded up), codes saturate.
 *   bits 8 with fmt KVQ_FMT_INT8_SYM: one two's complement int8 code per
 *                 element, the same meta layout with zero point 0 (the
 *                 KV-cache page's INT8 item: s = amax / 127 of the group,
 *                 floored at 1e-5 and stored in fp16 rounded up; code =
 *                 round-half-even(x / s), clamped to [-128, 127]).
 *   axis KVQ_AXIS_CHANNEL (K plane, fmt KVQ_FMT_INT, bits 2, 4 or 8): the
 *                 KV-cache page's advice to quantize the Key per channel.
 *                 Codes as above; meta f16 [batch][kv_heads][max_tokens /
 *                 KVQ_CHANNEL_BLOCK][head_dim][2], the (scale, zero point) of
 *                 channel d over the block's tokens (same formula as the
 *                 token groups); group_size is not used for this plane.
 *                 Only whole blocks are quantized: the tokens of an
 *                 unfinished block belong in a separate bits-16 segment.
 *   bits 4 with fmt KVQ_FMT_OAKEN (group_size = head_dim): the Oaken
 *                 group-shift codec of the same page's sections 3.1, 3.2.1
 *                 and 3.2.2, with the plane's offline kvq_oaken parameters.
 *                 Per element v: T_lo <= v <= T_hi gives c = clamp(rne(v /
 *                 s_in) + z_in, 0, 15); v > T_hi gives c = 15 and an outlier
 *                 m = min(rne((v - T_hi) / s_out), 2^b - 1); v < T_lo gives
 *                 c = 0 and an outlier -min(rne((T_lo - v) / s_out), 2^b - 1)
 *                 (fp32, one subtraction and one division each).  Codes
 *                 are packed like 4-bit codes.  meta u16
 *                 [batch][kv_heads][max_tokens][KVQ_OAKEN_SLOTS] holds the
 *                 row's outliers in ascending dim order (low byte the dim,
 *                 high byte the signed magnitude as a two's complement
 *                 byte), then zeros; outliers after the KVQ_OAKEN_SLOTS-th
 *                 are dropped.  x_hat = (c - z_in) * s_in + d * s_out with d
 *                 the element's slot value (0 without one): the page's
 *                 T_hi + Delta * scale and T_lo + Delta * scale.
 *   bits 16:      codes f16 [batch][kv_heads][max_tokens][head_dim] raw
 *                 values (Cocktail's FP16 class); meta unused (may be NULL).
 * Both buffers 16-byte aligned.
 */
typedef struct kvq_plane {
    int32_t bits;       /* 2, 4, 8 or 16                                    */
    int32_t group_size; /* G: 32, 64 or 128, dividing head_dim (bits < 16)  */
    void *codes;        /* device                                           */
    void *meta;         /* device; NULL when bits == 16                     */
    int32_t fmt;        /* kvq_format; the FP8 and INT8_SYM formats: bits 8 */
    int32_t axis;       /* kvq_axis; KVQ_AXIS_CHANNEL on the K plane only   */
    kvq_oaken oaken;    /* KVQ_FMT_OAKEN only                               */
} kvq_plane;

/*
 * A cache (or one bit-width segment of a mixed-precision cache).
 * seq_lens[b] is the number of valid tokens of sequence b (tokens
 * [0, seq_lens[b]) of every KV head).  max_tokens must be a multiple of 64.
 */
typedef struct kvq_cache {
    int32_t batch;
    int32_t kv_heads;
    int32_t head_dim;   /* 128 (the kernels are compiled for it)            */
    int32_t max_tokens; /* token capacity per (sequence, KV head)           */
    kvq_plane k;
    kvq_plane v;
    int32_t *seq_lens;  /* device, [batch]                                  */
} kvq_cache;

/* Human-readable name of a status. Never NULL. */
const char *kvq_status_string(kvq_status status);

/* Library version string, e.g. "kvq 0.1 sm_100a". */
const char *kvq_version(void);

/*
 * Bytes of the codes and meta buffers of one plane (host-only, no CUDA).
 * Source: the KV-cache size formula of the "大模型推理加速之KV Cache量化压缩
 * 原理与工程实现" page (2 * layers * kv_heads * head_dim * seq_len * batch *
 * bytes per element), per plane and layer, with bits/8 bytes per element
 * plus 4 bytes of (scale, zero) per group.
 * Returns KVQ_ERR_INVALID_ARG on non-positive sizes or null outputs,
 * KVQ_ERR_UNSUPPORTED on a (bits, G, head_dim) the library does not pack.
 * (A KVQ_FMT_OAKEN plane's codes are those of bits 4; its meta holds
 * KVQ_OAKEN_SLOTS * 2 bytes per token row instead of (scale, zero) pairs.)
 */
kvq_status kvq_plane_bytes(int32_t batch, int32_t kv_heads, int32_t head_dim,
                           int32_t max_tokens, int32_t bits, int32_t group_size,
                           size_t *codes_bytes, size_t *meta_bytes);

/*
 * Number of K and V elements of a model's cache, 2 * layers * kv_heads *
 * head_dim * seq_len * batch (same page's formula; the TurboQuant page's
 * section 1.2 worked example, 32 layers x 32 heads x 128 x 131072 tokens,
 * gives 34,359,738,368).  Host-only.  Returns 0 on overflow.
 */
uint64_t kvq_kv_elements(uint64_t layers, uint64_t kv_heads, uint64_t head_dim,
                         uint64_t seq_len, uint64_t batch);

/*
 * Quantize n_new tokens per sequence and write them at positions
 * seq_lens[b] .. seq_lens[b] + n_new - 1 of each sequence's K and V planes
 * (quantize-on-write: Cocktail page 3.2.2 formula; Oaken's write pipeline,
 * jsqmd.com news 825302 section 3.2.3, quantizes inside the memory write).
 *   k_new, v_new: device [batch][kv_heads][n_new][head_dim] of kv_dtype
 *                 values, 16-byte aligned.  n_new = 1 is the decode-step
 *                 append; n_new = the prompt length is the bulk prefill
 *                 (with seq_lens = 0).
 *   kv_dtype:     KVQ_F16 or KVQ_BF16.  Values of either type are widened to
 *                 fp32 exactly and go through the same fp32 steps, so a bf16
 *                 row holding fp16-representable values gives the codes of
 *                 its fp16 form.  Every format takes either (asymmetric
 *                 integer per token or, for K, per channel; FP8 E4M3/E5M2;
 *                 symmetric INT8; the Oaken codec).  bf16 values reach
 *                 beyond fp16: a group is encodable when its scale fits fp16
 *                 ((max - min) / (2^bits - 1), or |max| / 448, / 57344,
 *                 / 127, at most 65504) and its values are below 2^64 in
 *                 magnitude; the codes of other groups are unspecified.
 *   advance_seq_lens: nonzero adds n_new to seq_lens[b] after the write
 *                 (capped at max_tokens), in stream order.
 * Tokens whose position would reach max_tokens are not written (the
 * kernel checks on the device).  Both planes must have bits 2, 4 or 8 and
 * the same group size.  KVQ_FMT_OAKEN planes (bits 4, G = head_dim) are
 * encoded with their kvq_oaken parameters by one quantize kernel (half a
 * warp per token row), then seq_lens advances.  With a per-channel K plane (KVQ_AXIS_CHANNEL)
 * n_new must be a multiple of KVQ_CHANNEL_BLOCK, and so must seq_lens[b]
 * on the device: a sequence whose length is not is neither written nor
 * advanced.  Errors: KVQ_ERR_INVALID_ARG (nulls, n_new < 1, misalignment,
 * n_new off a block boundary, an unknown kv_dtype), KVQ_ERR_CAPACITY (n_new >
 * max_tokens), KVQ_ERR_UNSUPPORTED, KVQ_ERR_CUDA.
 */
kvq_status kvq_quantize_append(const kvq_cache *cache, const void *k_new,
                               const void *v_new, kvq_dtype kv_dtype,
                               int32_t n_new, int32_t advance_seq_lens,
                               void *stream);

/*
 * Workspace bytes that kvq_decode_attention (and kvq_decode_step) need for
 * these segments and arguments (host-only).  The workspace holds a 256-byte
 * header whose first 32-bit word is a sticky device error flag (nonzero
 * after a kernel gave up a bounded wait; the library never clears it),
 * followed by the work counters of the persistent decode kernel; then one
 * counter per sequence, used by the decode step; then the per-split
 * partial results (m, l, o) merged by log-sum-exp.  Every counter is back
 * at zero when a call's kernels finish.
 */
kvq_status kvq_decode_workspace_bytes(const kvq_cache *segs, int32_t n_segs,
                                      int32_t q_heads, int32_t max_len_hint,
                                      size_t *bytes);

/*
 * Decode attention of one query token per sequence over the packed cache:
 *   out[b][h] = sum_t p_t * V_hat[b][h/g][t],  p = softmax_t(softmax_scale *
 *   q[b][h] . K_hat[b][h/g][t]),  lse[b][h] = log sum_t exp(score_t),
 * over the tokens [0, seq_lens[b]) of every segment (the union, Cocktail
 * page 3.2.3), with g = q_heads / kv_heads (GQA: query head h reads KV head
 * h / g).  K_hat, V_hat are dequantized inside the QK^T and PV products
 * (TurboQuant page 2.3); scores follow the KVO-LLM page, section 3.2
 * (q . k^T / sqrt(dim)); pass softmax_scale = 1/sqrt(head_dim) for it.
 *   segs: 1 segment, or several segments of one mixed-precision cache (same
 *         batch, kv_heads, head_dim; each its own bits, planes, seq_lens).
 *   q: device [batch][q_heads][head_dim] fp16 or bf16 (q_dtype), 16-byte
 *      aligned.  The kernels feed q to fp16 tensor-core operands, lifted by
 *      a power of two that depends on the code format (up to 2^6 for 2-bit
 *      codes); a query row whose largest element would leave the fp16 range
 *      that way is staged scaled down by a power of two and its scores are
 *      scaled back, so every finite query gives finite scores.  bf16
 *      elements are rounded to fp16 after that scaling (exact where the
 *      scaled magnitude is at least 2^-14).  A score is formed per group as
 *      s * (sum q c - z * sum q), the code sum accumulated by the tensor
 *      cores in fp32, so its absolute error grows with s * |z| * max |q_j|
 *      rather than with the score itself: with 2-bit codes, query elements
 *      beyond about 1000 in magnitude can take the attention outside a
 *      1e-3 relative error.
 *   out: device fp32 [batch][q_heads][head_dim]; lse: device fp32
 *        [batch][q_heads] natural log, or NULL.
 *   max_len_hint: an upper bound of the seq_lens used to pick the split
 *        count (<= 0: max_tokens); results are correct for any seq_lens.
 *   workspace: device, >= kvq_decode_workspace_bytes(same arguments),
 *        256-byte aligned, zero-filled before its first use and again
 *        before a call on a cache of another batch size (its front holds
 *        counters that the kernels return to zero at the end of every call,
 *        at offsets that depend on the batch size only; it stays reusable
 *        without clearing across lengths, hints and segments).
 * A sequence with no tokens gives out = 0 and lse = -inf.
 * The call is one split-K kernel launch per segment, then one merge kernel
 * when the plan has more than one partial.
 * Supported: head_dim 128; g in 1..8; bits 2/4/8 with G 32/64/128, and bits
 * 16 with fp16 q; KVQ_FMT_OAKEN segments with g = 1, 2, 4 or 8 (the dense
 * codes through the tensor cores like INT4, plus the outlier slots).
 * Errors: KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_WORKSPACE,
 * KVQ_ERR_CUDA.
 */
kvq_status kvq_decode_attention(const kvq_cache *segs, int32_t n_segs,
                                const void *q, kvq_dtype q_dtype,
                                int32_t q_heads, float softmax_scale,
                                float *out, float *lse, int32_t max_len_hint,
                                void *workspace, size_t workspace_bytes,
                                void *stream);

/*
 * One decode step of one cache: quantize-on-write of one new token per
 * (sequence, KV head) -- the Oaken page's pipeline, where the quantizer sits
 * in the write path to memory (section 3.2.3), with the quantize formula of
 * the Cocktail page, 3.2.2, exactly as kvq_quantize_append computes it --
 * then kvq_decode_attention over the cache including that token.  It is the
 * same as kvq_quantize_append(cache, k_new, v_new, KVQ_F16, 1, advance = 1) followed
 * by kvq_decode_attention, with the same results bit for bit in the cache,
 * but for the tokens-on-M formats ((head_dim / G) * g <= 8) the append runs
 * inside the split-K kernel: the unit whose token range covers the new
 * position writes it, and the last unit of each sequence advances
 * seq_lens[b].  Other formats (KVQ_FMT_OAKEN included) run the two calls
 * as two launches on the stream.
 *   cache: one segment, bits 2, 4 or 8.
 *   k_new, v_new: device fp16 [batch][kv_heads][1][head_dim], 16-byte
 *        aligned.  A sequence already at max_tokens keeps its length and
 *        the token is not written (as in kvq_quantize_append).
 *   q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint, workspace:
 *        as kvq_decode_attention; max_len_hint should bound the lengths
 *        after the append.
 * Errors (nothing enqueued): KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED
 * (bits 16), KVQ_ERR_WORKSPACE; KVQ_ERR_CUDA after a failed launch.
 */
kvq_status kvq_decode_step(const kvq_cache *cache, const void *k_new,
                           const void *v_new, const void *q, kvq_dtype q_dtype,
                           int32_t q_heads, float softmax_scale, float *out,
                           float *lse, int32_t max_len_hint, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * The first half of kvq_decode_step -- the append and the split-K partials
 * -- for callers that time or overlap the halves; follow it with
 * kvq_decode_merge(cache, 1, ...) on the same stream.  Same arguments,
 * checks and errors as kvq_decode_step.
 */
kvq_status kvq_decode_step_partials(const kvq_cache *cache, const void *k_new,
                                    const void *v_new, const void *q,
                                    kvq_dtype q_dtype, int32_t q_heads,
                                    float softmax_scale, float *out, float *lse,
                                    int32_t max_len_hint, void *workspace,
                                    size_t workspace_bytes, void *stream);

/*
 * The two halves of kvq_decode_attention, for callers that time or overlap
 * them separately (same arguments, checks and errors as
 * kvq_decode_attention; call both, in this order, on the same stream).
 * kvq_decode_partials launches the split-K kernels: each split writes its
 * partial result -- running max m (log2 units), sum l = sum 2^(x - m) and
 * the unnormalised output -- into the workspace, or, when the plan has a
 * single partial, the final out/lse directly.  kvq_decode_merge combines
 * the partials by log-sum-exp (Cocktail page 3.2.3) into out/lse; it
 * enqueues nothing when there is a single partial.
 */
kvq_status kvq_decode_partials(const kvq_cache *segs, int32_t n_segs,
                               const void *q, kvq_dtype q_dtype,
                               int32_t q_heads, float softmax_scale,
                               float *out, float *lse, int32_t max_len_hint,
                               void *workspace, size_t workspace_bytes,
                               void *stream);
kvq_status kvq_decode_merge(const kvq_cache *segs, int32_t n_segs,
                            const void *q, kvq_dtype q_dtype, int32_t q_heads,
                            float softmax_scale, float *out, float *lse,
                            int32_t max_len_hint, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * Size of the library-owned scratch array used by
 * kvq_decode_attention_noalloc (8 MiB on every device that loads the
 * library, held until the process exits).
 */
#define KVQ_STATIC_SCRATCH_BYTES (8u << 20)

/*
 * kvq_decode_attention for callers that cannot allocate device memory.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot call cudaMalloc -- a plugin inside a host program that owns and
 * budgets all device memory, a language binding with no device allocator,
 * or a latency-critical loop that cannot afford cudaMalloc's implicit
 * device synchronization.  Same arguments and results as
 * kvq_decode_attention, minus the workspace: the scratch (split partials
 * and error word) lives in a fixed array of KVQ_STATIC_SCRATCH_BYTES inside
 * the library.  The caller still owns q, out, lse and the cache.
 *  - Returns KVQ_ERR_WORKSPACE, enqueuing nothing, when the request needs
 *    more scratch than KVQ_STATIC_SCRATCH_BYTES (kvq_decode_workspace_bytes
 *    with the same arguments tells how much it needs).
 *  - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *    call.  Every call looks up the array's device address
 *    (cudaGetSymbolAddress) with the caller's device current; the first
 *    call on a device is the one that loads the library's module there, so
 *    make that first call before any stream capture.
 *  - Arguments are all checked before the array is touched: a non-OK
 *    status means nothing was enqueued.
 *  - Every call shares the one array, which keeps the last call's contents
 *    (the error word is cleared at the start of each call).  Calls whose
 *    work overlaps on the GPU -- on different streams, or from different
 *    threads -- race on it; order them.
 */
kvq_status kvq_decode_attention_noalloc(const kvq_cache *segs, int32_t n_segs,
                                        const void *q, kvq_dtype q_dtype,
                                        int32_t q_heads, float softmax_scale,
                                        float *out, float *lse,
                                        int32_t max_len_hint, void *stream);

/*
 * Cocktail chunk-level bit-width search (Cocktail page 3.1.1): for each
 * sequence b and chunk i, sim = (q . c_i) / (||q|| * ||c_i||) in fp64 (sums
 * in index order); T_low and T_high from that sequence's s_min, s_max and
 * alpha, beta; class 16 if sim > T_high, 4 if T_low < sim <= T_high, else 2.
 *   chunk_emb: device fp32 [batch][n_chunks][emb_dim]
 *   query_emb: device fp32 [batch][emb_dim]
 *   sim_out:   device fp64 [batch][n_chunks], or NULL
 *   chunk_bits_out: device u8 [batch][n_chunks] (16, 4 or 2)
 * n_chunks <= 4096; emb_dim a multiple of 4, at most 4096; chunk_emb 16-byte
 * aligned.  Errors: KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED (emb_dim),
 * KVQ_ERR_CUDA.
 */
kvq_status kvq_chunk_assign(const float *chunk_emb, const float *query_emb,
                            int32_t batch, int32_t n_chunks, int32_t emb_dim,
                            double alpha, double beta, double *sim_out,
                            uint8_t *chunk_bits_out, void *stream);

/*
 * Reorder a prompt's fp16 K/V into three segments by chunk class and
 * quantize them (Cocktail page 3.1.2: reorder so equal bit-widths are
 * contiguous, then quantize, then compute).
 *   segs[0]: the FP16 segment (bits 16), segs[1]: the INT4 segment (bits 4),
 *   segs[2]: the INT2 segment (bits 2); same batch, kv_heads, head_dim; each
 *   with max_tokens >= context_len.  Their seq_lens are overwritten with the
 *   number of tokens of each class.
 *   k_src, v_src: device fp16 [batch][kv_heads][context_len][head_dim]
 *   chunk_bits: device u8 [batch][n_chunks], n_chunks = context_len /
 *               chunk_tokens (as written by kvq_chunk_assign); a value other
 *               than 16 or 4 is treated as 2
 *   perm_out: device int32 [batch][n_chunks]: perm_out[b][k] is the original
 *             index of the k-th chunk of the reordered sequence; FP16 chunks
 *             first, then INT4, then INT2, each in ascending original index.
 * chunk_tokens must be a multiple of 16 and divide context_len; n_chunks <=
 * 4096.  Errors: KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY,
 * KVQ_ERR_CUDA.
 */
kvq_status kvq_chunk_reorder(const kvq_cache *segs, const void *k_src,
                             const void *v_src, int32_t context_len,
                             int32_t chunk_tokens, const uint8_t *chunk_bits,
                             int32_t *perm_out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
