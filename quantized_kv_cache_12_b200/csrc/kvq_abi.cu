// kvq_abi.cu -- the C ABI of libkvq (declared in include/kvq.h): argument
// validation, launch configuration and dispatch.  Every check that can be
// made on the host runs before any CUDA call, so a non-OK status means
// nothing was enqueued.  No allocation, no synchronization.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

constexpr int kD = 128;
constexpr size_t kHeaderBytes = 256;


bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_group(int g) { return g == 32 || g == 64 || g == 128; }

// The kernels' template tag of a plane's format: its bit width, or kE4M3, kE5M2,
// kSym8 or kOaken.
int kernel_bits(const kvq_plane& p) {
  return p.fmt == KVQ_FMT_FP8_E4M3   ? kvq::kE4M3
         : p.fmt == KVQ_FMT_FP8_E5M2 ? kvq::kE5M2
         : p.fmt == KVQ_FMT_INT8_SYM ? kvq::kSym8
         : p.fmt == KVQ_FMT_OAKEN    ? kvq::kOaken
                                     : p.bits;
}

// An Oaken plane's offline parameters: s_in a positive fp16 value, z_in in
// [0, 15], s_out positive and finite, b in 5..7.
bool valid_oaken(const kvq_oaken& o) {
  if (!(o.inner_scale > 0.0f) || !isfinite(o.inner_scale)) return false;
  if (__half2float(__float2half_rn(o.inner_scale)) != o.inner_scale) return false;
  if (o.inner_zero < 0 || o.inner_zero > 15) return false;
  if (!(o.outer_scale > 0.0f) || !isfinite(o.outer_scale)) return false;
  return o.outer_bits >= 5 && o.outer_bits <= 7;
}

kvq::OakenParams oaken_params(const kvq_plane& p) {
  return kvq::make_oaken_params(p.oaken.inner_scale, p.oaken.inner_zero, p.oaken.outer_scale,
                                p.oaken.outer_bits);
}

kvq_status check_plane(const kvq_plane& p, int head_dim, bool allow16, bool is_k) {
  if (p.codes == nullptr || !aligned16(p.codes)) return KVQ_ERR_INVALID_ARG;
  if (p.fmt != KVQ_FMT_INT && p.fmt != KVQ_FMT_FP8_E4M3 && p.fmt != KVQ_FMT_INT8_SYM &&
      p.fmt != KVQ_FMT_FP8_E5M2 && p.fmt != KVQ_FMT_OAKEN)
    return KVQ_ERR_INVALID_ARG;
  if (p.axis != KVQ_AXIS_TOKEN && p.axis != KVQ_AXIS_CHANNEL) return KVQ_ERR_INVALID_ARG;
  if (p.fmt == KVQ_FMT_OAKEN) {
    if (p.bits != 4 || p.axis != KVQ_AXIS_TOKEN || p.group_size != head_dim)
      return KVQ_ERR_UNSUPPORTED;
    if (!valid_oaken(p.oaken)) return KVQ_ERR_INVALID_ARG;
    if (p.meta == nullptr || !aligned16(p.meta)) return KVQ_ERR_INVALID_ARG;
    return KVQ_OK;
  }
  if (p.fmt != KVQ_FMT_INT && p.bits != 8) return KVQ_ERR_UNSUPPORTED;
  if (p.axis == KVQ_AXIS_CHANNEL &&
      (!is_k || p.fmt != KVQ_FMT_INT || !(p.bits == 2 || p.bits == 4 || p.bits == 8)))
    return KVQ_ERR_UNSUPPORTED;
  if (p.bits == 16) {
    if (!allow16) return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
  }
  if (!(p.bits == 2 || p.bits == 4 || p.bits == 8)) return KVQ_ERR_UNSUPPORTED;
  if (p.axis == KVQ_AXIS_TOKEN && (!valid_group(p.group_size) || head_dim % p.group_size != 0))
    return KVQ_ERR_UNSUPPORTED;
  if (p.meta == nullptr || !aligned16(p.meta)) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

kvq_status check_cache(const kvq_cache* c, bool allow16) {
  if (c == nullptr) return KVQ_ERR_INVALID_ARG;
  if (c->batch <= 0 || c->kv_heads <= 0 || c->max_tokens <= 0 || c->head_dim <= 0)
    return KVQ_ERR_INVALID_ARG;
  if (c->head_dim != kD) return KVQ_ERR_UNSUPPORTED;
  if (c->max_tokens % 64 != 0) return KVQ_ERR_INVALID_ARG;
  if (c->seq_lens == nullptr) return KVQ_ERR_INVALID_ARG;
  kvq_status s = check_plane(c->k, c->head_dim, allow16, true);
  if (s != KVQ_OK) return s;
  s = check_plane(c->v, c->head_dim, allow16, false);
  if (s != KVQ_OK) return s;
  if (c->k.bits != c->v.bits || c->k.fmt != c->v.fmt) return KVQ_ERR_UNSUPPORTED;
  if (c->k.bits != 16 && c->k.axis == KVQ_AXIS_TOKEN && c->k.group_size != c->v.group_size)
    return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

// Split count of one segment.  A (sequence, KV head, split) is one unit of
// work; the decode kernels run one wave of persistent CTAs (C per SM, the
// format's occupancy) that take units from a counter, so each SM works
// through about u = ceil(units / SMs) units in rounds of up to C at a time.
// An SM's throughput is shared by its resident CTAs and saturates at about
// three of them, so a round of c < 3 units runs at c/3 of the SM's rate.
// The count minimises the SM's time, sum over its rounds of c x (tokens per
// unit + a fixed per-unit cost) / min(1, c/3), tokens per unit being rounded
// up to the 32-token stage, with at least 128 tokens per unit.  The fixed
// cost -- the start of a unit waits for its query rows and first copies,
// its end merges the warps -- is about 300 tokens' worth of work; more than
// one split adds the merge kernel's launch, about 600 tokens' worth (it
// decides only for tiny caches, where one split then avoids the launch).  The
// constants were fitted to split-count sweeps on B200 (INT4, INT8, FP8,
// per-channel K; 8 to 512 (sequence, head) pairs, 4k to 131k tokens).
int choose_splits_uncached(long long pairs, long long len, int sms, int ctas) {
  constexpr long long kOverhead = 300, kMerge = 600, kGran = 32, kMinTokens = 128;
  constexpr double kSat = 3.0;
  const long long cap = (len + kMinTokens - 1) / kMinTokens;
  long long best_n = 1;
  double best_cost = -1.0;
  for (long long n = 1; n <= cap && n <= 4096; ++n) {
    const long long chunk = ((len + n - 1) / n + kGran - 1) / kGran * kGran;
    const long long u = (pairs * n + sms - 1) / sms;  // units of the busiest SM
    const long long full = u / ctas, rest = u % ctas;
    const double c_full = (double)ctas, c_rest = (double)rest;
    double rounds = (double)full * c_full / (c_full < kSat ? c_full / kSat : 1.0);
    if (rest > 0) rounds += c_rest / (c_rest < kSat ? c_rest / kSat : 1.0);
    const double cost = rounds * (double)(chunk + kOverhead) + (n > 1 ? (double)kMerge : 0.0);
    if (best_cost < 0 || cost < best_cost * (1.0 - 1e-9)) {
      best_cost = cost;
      best_n = n;
    }
  }
  return (int)best_n;
}

// The search above costs a few microseconds for long sequences, and every
// decode call plans its splits: the last few answers are kept per host
// thread (the inputs are a handful of integers, so a hit is exact).
int choose_splits(const kvq_cache& c, int max_len_hint, int ctas_per_sm, int sms) {
  const long long pairs = (long long)c.batch * c.kv_heads;
  long long len = c.max_tokens;
  if (max_len_hint > 0 && max_len_hint < len) len = max_len_hint;
  if (len <= 0 || pairs <= 0) return 1;
  const int ctas = ctas_per_sm > 0 ? ctas_per_sm : 3;
  struct Memo {
    long long pairs, len;
    int sms, ctas, n;
  };
  constexpr int kMemo = 8;
  thread_local Memo memo[kMemo] = {};
  thread_local int next = 0;
  for (int i = 0; i < kMemo; ++i)
    if (memo[i].n > 0 && memo[i].pairs == pairs && memo[i].len == len && memo[i].sms == sms &&
        memo[i].ctas == ctas)
      return memo[i].n;
  const int n = choose_splits_uncached(pairs, len, sms, ctas);
  memo[next] = Memo{pairs, len, sms, ctas, n};
  next = (next + 1) % kMemo;
  return n;
}

struct SplitPlan {
  int n_split[16];
  int parts;
};

kvq_status plan_splits(const kvq_cache* segs, int n_segs, int q_heads, int max_len_hint,
                       SplitPlan* plan) {
  plan->parts = 0;
  const int g = q_heads / segs[0].kv_heads;
  const int sms = kvq::device_sm_count();
  for (int i = 0; i < n_segs; ++i) {
    const int bits = kernel_bits(segs[i].k);
    const int group = bits == 16 ? kD : segs[i].v.group_size;
    const bool kpc = segs[i].k.axis == KVQ_AXIS_CHANNEL;
    const int ctas = kvq::decode_ctas_per_sm(bits, group, g, kpc);
    plan->n_split[i] = choose_splits(segs[i], max_len_hint, ctas, sms);
    plan->parts += plan->n_split[i];
  }
  return KVQ_OK;
}

kvq_status check_segments(const kvq_cache* segs, int n_segs, int q_heads) {
  if (segs == nullptr || n_segs < 1 || n_segs > 16) return KVQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_segs; ++i) {
    kvq_status s = check_cache(&segs[i], true);
    if (s != KVQ_OK) return s;
    if (segs[i].batch != segs[0].batch || segs[i].kv_heads != segs[0].kv_heads ||
        segs[i].head_dim != segs[0].head_dim)
      return KVQ_ERR_INVALID_ARG;
  }
  if (q_heads <= 0 || q_heads % segs[0].kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  const int g = q_heads / segs[0].kv_heads;
  for (int i = 0; i < n_segs; ++i) {
    const int bits = kernel_bits(segs[i].k);
    const bool kpc = segs[i].k.axis == KVQ_AXIS_CHANNEL;
    if (!kvq::decode_supported(bits, bits == 16 ? kD : segs[i].v.group_size, g, kpc))
      return KVQ_ERR_UNSUPPORTED;
  }
  return KVQ_OK;
}

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// Workspace layout: header (error word, work counters); the per-sequence
// unit counters of the decode step, at an offset and size that depend only
// on batch; then the partial (m, l) and o, whose sizes follow the split
// plan.  Every counter returns to zero by the end of each launch, so one
// zero fill lasts for any number of calls on caches of one batch size.
struct WsLayout {
  size_t seq_cnt, ml, o, total;
};

size_t counter_bytes(const kvq_cache* segs) {
  return round256((size_t)segs[0].batch * sizeof(uint32_t));
}

WsLayout workspace_layout(const kvq_cache* segs, int q_heads, int parts) {
  const size_t bh = (size_t)segs[0].batch * q_heads;
  WsLayout w;
  w.seq_cnt = kHeaderBytes;
  w.ml = kHeaderBytes + counter_bytes(segs);
  w.o = w.ml + round256(bh * parts * 2 * sizeof(float));
  w.total = w.o + round256(bh * parts * kD * sizeof(float));
  return w;
}

size_t workspace_for(const kvq_cache* segs, int q_heads, int parts) {
  return workspace_layout(segs, q_heads, parts).total;
}

}  // namespace

namespace kvq {
// The device's streaming multiprocessors, read once per device
// (cudaDevAttrMultiProcessorCount).  KVQ_NUM_SMS in the environment
// overrides it, for planning on a host without that device; with neither,
// kDefaultSms (B200).
int device_sm_count() {
  static int env_sms = -1;  // -1: not read yet, 0: unset
  if (env_sms < 0) {
    const char* e = getenv("KVQ_NUM_SMS");
    const long v = e != nullptr ? strtol(e, nullptr, 10) : 0;
    env_sms = (v > 0 && v <= 4096) ? (int)v : 0;
  }
  if (env_sms > 0) return env_sms;
  constexpr int kMaxDev = 64;
  static std::atomic<int> cached[kMaxDev];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    cudaGetLastError();  // no device here: clear the sticky-free error state
    return kDefaultSms;
  }
  int n = cached[dev].load();
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return kDefaultSms;
    }
    cached[dev].store(n);
  }
  return n;
}

size_t decode_zeroed_prefix_bytes(const kvq_cache* segs) {
  return kHeaderBytes + counter_bytes(segs);
}
}  // namespace kvq

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "cache capacity exceeded";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* kvq_version(void) { return "kvq 0.1 sm_100a"; }

kvq_status kvq_plane_bytes(int32_t batch, int32_t kv_heads, int32_t head_dim, int32_t max_tokens,
                           int32_t bits, int32_t group_size, size_t* codes_bytes,
                           size_t* meta_bytes) {
  if (codes_bytes == nullptr || meta_bytes == nullptr) return KVQ_ERR_INVALID_ARG;
  if (batch <= 0 || kv_heads <= 0 || head_dim <= 0 || max_tokens <= 0) return KVQ_ERR_INVALID_ARG;
  if (!(bits == 2 || bits == 4 || bits == 8 || bits == 16)) return KVQ_ERR_UNSUPPORTED;
  if (bits != 16 && (!valid_group(group_size) || head_dim % group_size != 0))
    return KVQ_ERR_UNSUPPORTED;
  if ((head_dim * bits) % 8 != 0) return KVQ_ERR_UNSUPPORTED;
  const size_t rows = (size_t)batch * kv_heads * max_tokens;
  *codes_bytes = rows * (size_t)head_dim * bits / 8;
  *meta_bytes = (bits == 16) ? 0 : rows * (size_t)(head_dim / group_size) * 4;
  return KVQ_OK;
}

uint64_t kvq_kv_elements(uint64_t layers, uint64_t kv_heads, uint64_t head_dim,
                         uint64_t seq_len, uint64_t batch) {
  uint64_t f[5] = {layers, kv_heads, head_dim, seq_len, batch};
  uint64_t n = 2;
  for (int i = 0; i < 5; ++i) {
    if (f[i] != 0 && n > UINT64_MAX / f[i]) return 0;
    n *= f[i];
  }
  return n;
}

kvq_status kvq_quantize_append(const kvq_cache* cache, const void* k_new, const void* v_new,
                               kvq_dtype kv_dtype, int32_t n_new, int32_t advance_seq_lens,
                               void* stream) {
  kvq_status st = check_cache(cache, false);
  if (st != KVQ_OK) return st;
  if (k_new == nullptr || v_new == nullptr || !aligned16(k_new) || !aligned16(v_new))
    return KVQ_ERR_INVALID_ARG;
  if (kv_dtype != KVQ_F16 && kv_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (n_new < 1) return KVQ_ERR_INVALID_ARG;
  if (n_new > cache->max_tokens) return KVQ_ERR_CAPACITY;
  kvq::QuantArgs a;
  a.in_bf16 = kv_dtype == KVQ_BF16;
  a.k_new = static_cast<const __half*>(k_new);
  a.v_new = static_cast<const __half*>(v_new);
  a.k_codes = static_cast<uint8_t*>(cache->k.codes);
  a.v_codes = static_cast<uint8_t*>(cache->v.codes);
  a.k_meta = static_cast<uint8_t*>(cache->k.meta);
  a.v_meta = static_cast<uint8_t*>(cache->v.meta);
  a.seq_lens = cache->seq_lens;
  a.batch = cache->batch;
  a.kv_heads = cache->kv_heads;
  a.max_tokens = cache->max_tokens;
  a.n_new = n_new;
  a.advance = advance_seq_lens != 0;
  a.side0 = 0;
  a.k_channels = cache->k.axis == KVQ_AXIS_CHANNEL;
  if (a.k_channels && n_new % KVQ_CHANNEL_BLOCK != 0) return KVQ_ERR_INVALID_ARG;
  if (cache->k.fmt == KVQ_FMT_OAKEN) {
    a.k_oaken = oaken_params(cache->k);
    a.v_oaken = oaken_params(cache->v);
    return kvq::launch_oaken_quantize(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KVQ_OK
               : KVQ_ERR_CUDA;
  }
  cudaError_t e = kvq::launch_quantize(a, kernel_bits(cache->k), cache->k.group_size,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_decode_workspace_bytes(const kvq_cache* segs, int32_t n_segs, int32_t q_heads,
                                      int32_t max_len_hint, size_t* bytes) {
  if (bytes == nullptr) return KVQ_ERR_INVALID_ARG;
  kvq_status st = check_segments(segs, n_segs, q_heads);
  if (st != KVQ_OK) return st;
  SplitPlan plan;
  plan_splits(segs, n_segs, q_heads, max_len_hint, &plan);
  *bytes = workspace_for(segs, q_heads, plan.parts);
  return KVQ_OK;
}

}  // extern "C"

namespace {

enum DecodeStage { kPartials = 1, kMerge = 2, kBoth = 3 };

// One decode attention (stages kBoth), or only its partials or its merge,
// or (stages 0) only the argument checks.  k_new/v_new (with a single
// segment of a tokens-on-M format) make it a decode step: the kernel also
// quantizes one new token per (sequence, KV head) into the cache and
// advances seq_lens.
kvq_status decode_stages(const kvq_cache* segs, int32_t n_segs, const void* q,
                         kvq_dtype q_dtype, int32_t q_heads, float softmax_scale, float* out,
                         float* lse, int32_t max_len_hint, void* workspace,
                         size_t workspace_bytes, void* stream, int stages,
                         const void* k_new = nullptr, const void* v_new = nullptr) {
  kvq_status st = check_segments(segs, n_segs, q_heads);
  if (st != KVQ_OK) return st;
  if (q == nullptr || out == nullptr || !aligned16(q)) return KVQ_ERR_INVALID_ARG;
  if (q_dtype != KVQ_F16 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.0f) || !isfinite(softmax_scale)) return KVQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_segs; ++i)
    if (segs[i].k.bits == 16 && q_dtype == KVQ_BF16) return KVQ_ERR_UNSUPPORTED;
  SplitPlan plan;
  plan_splits(segs, n_segs, q_heads, max_len_hint, &plan);
  const size_t need = workspace_for(segs, q_heads, plan.parts);
  if (workspace == nullptr || workspace_bytes < need) return KVQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return KVQ_ERR_INVALID_ARG;
  if (stages == 0) return KVQ_OK;  // arguments checked, nothing enqueued

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const WsLayout lay = workspace_layout(segs, q_heads, plan.parts);
  kvq::DecodeArgs a;
  a.batch = segs[0].batch;
  a.kv_heads = segs[0].kv_heads;
  a.q_heads = q_heads;
  a.group_ratio = q_heads / segs[0].kv_heads;
  a.q = q;
  a.q_is_bf16 = q_dtype == KVQ_BF16;
  a.scale_log2 = (float)((double)softmax_scale * 1.4426950408889634);
  a.parts = plan.parts;
  a.err = reinterpret_cast<uint32_t*>(ws);
  a.part_ml = reinterpret_cast<float*>(ws + lay.ml);
  a.part_o = reinterpret_cast<float*>(ws + lay.o);
  a.out = out;
  a.lse = lse;
  a.seq_cnt = reinterpret_cast<uint32_t*>(ws + lay.seq_cnt);
  a.k_new = static_cast<const __half*>(k_new);
  a.v_new = static_cast<const __half*>(v_new);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int base = 0;
  for (int i = 0; i < n_segs; ++i) {
    kvq::SegView v;
    v.k_codes = static_cast<const uint8_t*>(segs[i].k.codes);
    v.v_codes = static_cast<const uint8_t*>(segs[i].v.codes);
    v.k_meta = static_cast<const uint8_t*>(segs[i].k.meta);
    v.v_meta = static_cast<const uint8_t*>(segs[i].v.meta);
    v.seq_lens = segs[i].seq_lens;
    v.bits = kernel_bits(segs[i].k);
    v.group = segs[i].k.bits == 16 ? kD : segs[i].v.group_size;
    v.k_channels = segs[i].k.axis == KVQ_AXIS_CHANNEL;
    v.max_tokens = segs[i].max_tokens;
    v.n_split = plan.n_split[i];
    v.sms = kvq::device_sm_count();
    if (segs[i].k.fmt == KVQ_FMT_OAKEN) {
      v.k_oaken = oaken_params(segs[i].k);
      v.v_oaken = oaken_params(segs[i].v);
    }
    v.part_base = base;
    base += plan.n_split[i];
    // each segment its own work counters, so that the segments' kernels may
    // run side by side: the later ones are programmatic dependents
    v.ctr = 1 + 2 * i;
    v.after_prev = i > 0;
    if ((stages & kPartials) && kvq::launch_decode_segment(a, v, s) != cudaSuccess)
      return KVQ_ERR_CUDA;
  }
  if ((stages & kMerge) && plan.parts > 1 && kvq::launch_decode_merge(a, s) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return KVQ_OK;
}

}  // namespace

namespace kvq {
// kvq_decode_attention's argument checks alone (nothing enqueued).
kvq_status decode_check_args(const kvq_cache* segs, int32_t n_segs, const void* q,
                             kvq_dtype q_dtype, int32_t q_heads, float softmax_scale, float* out,
                             float* lse, int32_t max_len_hint, void* workspace,
                             size_t workspace_bytes) {
  return decode_stages(segs, n_segs, q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint,
                       workspace, workspace_bytes, nullptr, 0);
}
}  // namespace kvq

extern "C" {

kvq_status kvq_decode_attention(const kvq_cache* segs, int32_t n_segs, const void* q,
                                kvq_dtype q_dtype, int32_t q_heads, float softmax_scale,
                                float* out, float* lse, int32_t max_len_hint, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return decode_stages(segs, n_segs, q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint,
                       workspace, workspace_bytes, stream, kBoth);
}

kvq_status kvq_decode_partials(const kvq_cache* segs, int32_t n_segs, const void* q,
                               kvq_dtype q_dtype, int32_t q_heads, float softmax_scale,
                               float* out, float* lse, int32_t max_len_hint, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return decode_stages(segs, n_segs, q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint,
                       workspace, workspace_bytes, stream, kPartials);
}

kvq_status kvq_decode_merge(const kvq_cache* segs, int32_t n_segs, const void* q,
                            kvq_dtype q_dtype, int32_t q_heads, float softmax_scale, float* out,
                            float* lse, int32_t max_len_hint, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return decode_stages(segs, n_segs, q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint,
                       workspace, workspace_bytes, stream, kMerge);
}

}  // extern "C"

namespace {

// The decode step (stages kBoth) or its first half (kPartials).
kvq_status decode_step_stages(const kvq_cache* cache, const void* k_new, const void* v_new,
                              const void* q, kvq_dtype q_dtype, int32_t q_heads,
                              float softmax_scale, float* out, float* lse, int32_t max_len_hint,
                              void* workspace, size_t workspace_bytes, void* stream, int stages) {
  kvq_status st = check_segments(cache, 1, q_heads);
  if (st != KVQ_OK) return st;
  if (cache->k.bits == 16) return KVQ_ERR_UNSUPPORTED;
  // a per-channel K block is quantized only once it is complete: single
  // tokens go to a separate fp16 segment
  if (cache->k.axis == KVQ_AXIS_CHANNEL) return KVQ_ERR_UNSUPPORTED;
  if (k_new == nullptr || v_new == nullptr || !aligned16(k_new) || !aligned16(v_new))
    return KVQ_ERR_INVALID_ARG;
  const int g = q_heads / cache->kv_heads;
  // the tokens-on-M kernel quantizes the new token itself, except for the
  // Oaken codec, whose row encoding (the outlier slots) has its own kernel
  if (cache->k.fmt != KVQ_FMT_OAKEN &&
      kvq::decode_tm_supported(kernel_bits(cache->k), cache->k.group_size, g))
    return decode_stages(cache, 1, q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint,
                         workspace, workspace_bytes, stream, stages, k_new, v_new);
  // formats of the 16-row kernel and the Oaken codec: the append kernel,
  // then the attention
  // (every argument is checked before the first launch)
  st = decode_stages(cache, 1, q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint,
                     workspace, workspace_bytes, stream, 0);
  if (st != KVQ_OK) return st;
  st = kvq_quantize_append(cache, k_new, v_new, KVQ_F16, 1, 1, stream);
  if (st != KVQ_OK) return st;
  return decode_stages(cache, 1, q, q_dtype, q_heads, softmax_scale, out, lse, max_len_hint,
                       workspace, workspace_bytes, stream, stages);
}

}  // namespace

extern "C" {

kvq_status kvq_decode_step(const kvq_cache* cache, const void* k_new, const void* v_new,
                           const void* q, kvq_dtype q_dtype, int32_t q_heads, float softmax_scale,
                           float* out, float* lse, int32_t max_len_hint, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return decode_step_stages(cache, k_new, v_new, q, q_dtype, q_heads, softmax_scale, out, lse,
                            max_len_hint, workspace, workspace_bytes, stream, kBoth);
}

kvq_status kvq_decode_step_partials(const kvq_cache* cache, const void* k_new, const void* v_new,
                                    const void* q, kvq_dtype q_dtype, int32_t q_heads,
                                    float softmax_scale, float* out, float* lse,
                                    int32_t max_len_hint, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  return decode_step_stages(cache, k_new, v_new, q, q_dtype, q_heads, softmax_scale, out, lse,
                            max_len_hint, workspace, workspace_bytes, stream, kPartials);
}

kvq_status kvq_chunk_assign(const float* chunk_emb, const float* query_emb, int32_t batch,
                            int32_t n_chunks, int32_t emb_dim, double alpha, double beta,
                            double* sim_out, uint8_t* chunk_bits_out, void* stream) {
  if (chunk_emb == nullptr || query_emb == nullptr || chunk_bits_out == nullptr)
    return KVQ_ERR_INVALID_ARG;
  if (batch <= 0 || n_chunks <= 0 || n_chunks > 4096 || emb_dim <= 0) return KVQ_ERR_INVALID_ARG;
  if (!isfinite(alpha) || !isfinite(beta)) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(chunk_emb)) return KVQ_ERR_INVALID_ARG;
  if (emb_dim % 4 != 0 || emb_dim > 4096) return KVQ_ERR_UNSUPPORTED;
  cudaError_t e = kvq::launch_chunk_assign(chunk_emb, query_emb, batch, n_chunks, emb_dim, alpha,
                                           beta, sim_out, chunk_bits_out,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

kvq_status kvq_chunk_reorder(const kvq_cache* segs, const void* k_src, const void* v_src,
                             int32_t context_len, int32_t chunk_tokens, const uint8_t* chunk_bits,
                             int32_t* perm_out, void* stream) {
  if (segs == nullptr || k_src == nullptr || v_src == nullptr || chunk_bits == nullptr ||
      perm_out == nullptr)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_src) || !aligned16(v_src)) return KVQ_ERR_INVALID_ARG;
  const int want_bits[3] = {16, 4, 2};
  for (int i = 0; i < 3; ++i) {
    kvq_status st = check_cache(&segs[i], true);
    if (st != KVQ_OK) return st;
    if (segs[i].k.bits != want_bits[i] || segs[i].k.fmt != KVQ_FMT_INT ||
        segs[i].k.axis != KVQ_AXIS_TOKEN)
      return KVQ_ERR_INVALID_ARG;
    if (segs[i].batch != segs[0].batch || segs[i].kv_heads != segs[0].kv_heads)
      return KVQ_ERR_INVALID_ARG;
  }
  if (segs[1].k.group_size != segs[2].k.group_size) return KVQ_ERR_UNSUPPORTED;
  if (chunk_tokens <= 0 || chunk_tokens % 16 != 0 || context_len <= 0 ||
      context_len % chunk_tokens != 0)
    return KVQ_ERR_INVALID_ARG;
  const int n_chunks = context_len / chunk_tokens;
  if (n_chunks > 4096) return KVQ_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (segs[i].max_tokens < context_len) return KVQ_ERR_CAPACITY;
  kvq::ReorderArgs r;
  r.k_src = static_cast<const __half*>(k_src);
  r.v_src = static_cast<const __half*>(v_src);
  r.chunk_bits = chunk_bits;
  r.perm = perm_out;
  for (int i = 0; i < 3; ++i) r.seg[i] = segs[i];
  r.batch = segs[0].batch;
  r.kv_heads = segs[0].kv_heads;
  r.context_len = context_len;
  r.chunk_tokens = chunk_tokens;
  r.n_chunks = n_chunks;
  cudaError_t e = kvq::launch_chunk_reorder(r, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}

}  // extern "C"
