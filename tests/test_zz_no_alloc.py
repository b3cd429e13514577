"""kvq_decode_attention_noalloc: decode attention for callers that cannot
allocate device memory (a plugin inside a host program that owns all device
memory, a binding without a device allocator, or a loop that cannot afford
cudaMalloc's implicit synchronization).  Its scratch is the library's own
fixed-size device array, so the caller passes only inputs and outputs.

The test calls the entry point through the C ABI twice in a row (the array
keeps the previous call's contents) and checks each result against
kvq_decode_attention with a caller-owned workspace, within the attention
tolerance used everywhere else (2e-3 max-abs, 1e-3 relative L2).  This file
is collected last so that a stop-at-first-failure run has already run every
other test."""
import ctypes

import numpy as np
import pytest
import torch

import workloads

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


def _close(a, b):
    a = a.cpu().numpy().astype(np.float64)
    b = b.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(a))
    assert np.abs(a - b).max() <= 2e-3
    assert np.linalg.norm(a - b) <= 1e-3 * np.linalg.norm(b)


@pytest.mark.parametrize("name", ["llama3_8b_gqa_int4", "llama2_7b_mha_int8"])
def test_noalloc_matches_workspace_entry_point_twice(kvq, name):
    base = workloads.WORKLOADS[name]
    wl = base.scaled(batch=4, kv_heads=4, q_heads=4 * base.group_ratio)
    L = 1500
    k, v = workloads.kv_tokens(wl, L, DEV)
    cache = kvq.QuantizedKVCache.allocate(4, 4, 128, 1536, wl.bits, wl.group, DEV)
    cache.seq_lens.zero_()
    kvq.kvq_quantize_append(cache, k, v, L, advance_seq_lens=True)
    B, Hq = 4, wl.q_heads
    for call in range(2):
        q = workloads.queries(wl, DEV, step=call)
        if call == 1:  # a different length on the second call
            cache.seq_lens.copy_(torch.tensor([L, 3, 700, 1], dtype=torch.int32))
        out_ref = torch.empty((B, Hq, 128), device=DEV)
        lse_ref = torch.empty((B, Hq), device=DEV)
        ws = kvq.alloc_workspace(cache, Hq, L, device=DEV)
        kvq.kvq_decode_attention(cache, q, out_ref, lse_ref, ws, max_len_hint=L)
        out = torch.full((B, Hq, 128), float("nan"), device=DEV)
        lse = torch.full((B, Hq), float("nan"), device=DEV)
        st = _noalloc_call(kvq, cache, q, out, lse, L)
        assert st == kvq.KVQ_OK, kvq.kvq_status_string(st)
        torch.cuda.synchronize()
        _close(out, out_ref)
        _close(lse, lse_ref)


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
