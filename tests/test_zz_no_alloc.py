"""kvq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (a plugin inside a host program that owns all device
memory, a binding without a device allocator, or a loop that cannot afford
cudaMalloc's implicit synchronization).  Its scratch is the library's own
fixed-size device array, so the caller passes only inputs and outputs.

The test calls the entry point through the C ABI three times in a row (the
array keeps the previous call's contents): twice on one cache with different
lengths, then on a cache of another batch size, KV-head count and query-group
ratio whose long sequences spread over many CTAs, so the array holds the
previous call's data in another layout.  Each result is checked against
kvq_decode_attention with a caller-owned workspace and against the CPU oracle
on the same seeded inputs, within the attention tolerance used everywhere
else (2e-3 max-abs, 1e-3 relative L2).  This file is collected last so that
a stop-at-first-failure run has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_close, oracle_segment, q_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def _noalloc_call(kvq, cache, q, out, lse, hint):
    """Direct C-ABI call (ctypes), no workspace argument."""
    arr = (kvq.kvq_cache * 1)(cache.struct())
    dt = kvq.KVQ_BF16 if q.dtype == torch.bfloat16 else kvq.KVQ_F16
    return kvq.lib.kvq_decode_attention_noalloc(
        arr, 1, ctypes.c_void_p(q.data_ptr()), dt, q.shape[1], ctypes.c_float(128 ** -0.5),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), hint,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check_call(kvq, wl, cache, k, v, q, lens, hint):
    B, Hq = cache.batch, q.shape[1]
    out_ref = torch.empty((B, Hq, 128), device=DEV)
    lse_ref = torch.empty((B, Hq), device=DEV)
    ws = kvq.alloc_workspace(cache, Hq, hint, device=DEV)
    kvq.kvq_decode_attention(cache, q, out_ref, lse_ref, ws, max_len_hint=hint)
    out = torch.full((B, Hq, 128), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    st = _noalloc_call(kvq, cache, q, out, lse, hint)
    assert st == kvq.KVQ_OK, kvq.kvq_status_string(st)
    torch.cuda.synchronize()
    # against the workspace entry point
    assert_close(out, out_ref.cpu().numpy().astype(np.float64), lse, lse_ref.cpu().numpy(),
                 what="noalloc vs workspace")
    # against the oracle (it quantizes the same fp16 inputs itself)
    seg = oracle_segment(k, v, wl.bits, wl.group)
    o_ref, l_ref = oracle.decode_attention(q_bits(q), q.dtype == torch.bfloat16, [seg],
                                           [np.asarray(lens)], 128 ** -0.5)
    assert_close(out, o_ref, lse, l_ref, what="noalloc vs oracle")


@pytest.mark.parametrize("name", ["llama3_8b_gqa_int4", "llama2_7b_mha_int8"])
def test_noalloc_matches_workspace_entry_point_and_oracle(kvq, name):
    from gpu_util import fill_cache
    base = workloads.WORKLOADS[name]
    # calls 1 and 2: one cache, two length sets
    wl = base.scaled(batch=4, kv_heads=4, q_heads=4 * base.group_ratio)
    L = 1500
    k, v = workloads.kv_tokens(wl, L, DEV)
    cache = kvq.QuantizedKVCache.allocate(4, 4, 128, 1536, wl.bits, wl.group, DEV)
    for call, lens in enumerate([[L] * 4, [L, 3, 700, 1]]):
        fill_cache(kvq, cache, k, v, lens)
        q = workloads.queries(wl, DEV, step=call)
        _check_call(kvq, wl, cache, k, v, q, lens, L)
    # call 3: another batch size, KV-head count and group ratio; 6000-token
    # sequences over many CTAs (the in-kernel merge takes two levels)
    g3 = 2
    wl3 = base.scaled(batch=2, kv_heads=2, q_heads=2 * g3)
    L3 = 6000
    k3, v3 = workloads.kv_tokens(wl3, L3, DEV)
    cache3 = kvq.QuantizedKVCache.allocate(2, 2, 128, 6016, wl3.bits, wl3.group, DEV)
    lens3 = [L3, 4321]
    fill_cache(kvq, cache3, k3, v3, lens3)
    q3 = workloads.queries(wl3, DEV, step=2)
    _check_call(kvq, wl3, cache3, k3, v3, q3, lens3, L3)


def test_noalloc_rejects_requests_beyond_its_scratch(kvq):
    """A plan whose partials need more than KVQ_STATIC_SCRATCH_BYTES is
    refused before anything is enqueued."""
    c = kvq.kvq_cache()
    c.batch, c.kv_heads, c.head_dim, c.max_tokens = 64, 8, 128, 131072
    c.k = kvq.kvq_plane(4, 64, 0x10000, 0x20000)  # never dereferenced
    c.v = kvq.kvq_plane(4, 64, 0x30000, 0x40000)
    c.seq_lens = 0x50000
    need = kvq.kvq_decode_workspace_bytes(c, 64)
    assert need > (8 << 20)
    fake = ctypes.c_void_p(0x60000)
    st = kvq.lib.kvq_decode_attention_noalloc((kvq.kvq_cache * 1)(c), 1, fake, 0, 64,
                                              ctypes.c_float(0.088), fake, None, 0, None)
    assert st == kvq.KVQ_ERR_WORKSPACE


def test_noalloc_rejects_bad_arguments_before_touching_its_scratch(kvq):
    """An argument error (here a null query) returns its status with nothing
    enqueued on the stream -- in particular no clearing of the shared array."""
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=1, kv_heads=1, q_heads=4)
    cache = kvq.QuantizedKVCache.allocate(1, 1, 128, 64, wl.bits, wl.group, DEV)
    out = torch.empty((1, 4, 128), device=DEV)
    lse = torch.empty((1, 4), device=DEV)
    arr = (kvq.kvq_cache * 1)(cache.struct())
    s = torch.cuda.Stream()
    st = kvq.lib.kvq_decode_attention_noalloc(
        arr, 1, None, kvq.KVQ_F16, 4, ctypes.c_float(128 ** -0.5),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), 64,
        ctypes.c_void_p(s.cuda_stream))
    assert st == kvq.KVQ_ERR_INVALID_ARG
    assert s.query()  # nothing was enqueued
