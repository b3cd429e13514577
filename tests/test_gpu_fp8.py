"""GPU parity of the FP8 KV formats, E4M3 and E5M2 (KV-cache page, FP8 KV
cache with a dynamic per-group scale; the oracle's readings R14 and R17):
codes and scales written by kvq_quantize_append byte for byte equal to the
oracle's, and decode attention over them within the attention tolerance of
the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_close, f16_bits, fill_cache, oracle_segment, q_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


@pytest.fixture(params=["fp8", "e5m2"])
def fmt(request):
    """The oracle's format name; the library code is looked up from it."""
    return request.param


def _code(kvq, fmt):
    return kvq.KVQ_FMT_FP8_E4M3 if fmt == "fp8" else kvq.KVQ_FMT_FP8_E5M2


def _alloc(kvq, B, H, max_tokens, G, fmt="fp8"):
    c = kvq.QuantizedKVCache.allocate(B, H, 128, max_tokens, 8, G, DEV, fmt=_code(kvq, fmt))
    c.k_codes.fill_(0x7F)  # NaN codes and NaN scales in unused slots
    c.v_codes.fill_(0xFF)
    c.k_meta.view(torch.int16).fill_(-1)
    c.v_meta.view(torch.int16).fill_(-1)
    return c


@pytest.mark.parametrize("G", [32, 64, 128])
def test_quantize_bit_exact(kvq, G, fmt):
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(batch=3, kv_heads=2, q_heads=2)
    T = 41
    k, v = workloads.kv_tokens(wl, T, DEV)
    # adversarial rows: zeros, a constant, tiny values, values near the fp16
    # maximum, exact E4M3 ties at s = 1 (amax 448), negative zeros
    k[0, 0, 0] = 0.0
    k[0, 0, 1] = 3.0
    k[0, 0, 2] = (torch.randn(128, device=DEV) * 1e-6).half()
    k[0, 0, 3] = (torch.randn(128, device=DEV) * 20000).clamp(-60000, 60000).half()
    row = torch.tensor([448.0, 1.0625, 1.1875, -2.0, 0.0999755859375, -0.0, 240.0, 232.0],
                       device=DEV).repeat(16).half()
    k[0, 1, 4] = row
    v[1, 0, 5] = -0.0
    c = _alloc(kvq, 3, 2, 64, G, fmt)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    kc, km = oracle.quantize_cache(f16_bits(k), G, 8, fmt)
    vc, vm = oracle.quantize_cache(f16_bits(v), G, 8, fmt)
    assert np.array_equal(c.k_codes[:, :, :T].cpu().numpy(), kc)
    assert np.array_equal(c.v_codes[:, :, :T].cpu().numpy(), vc)
    assert np.array_equal(c.k_meta[:, :, :T].cpu().numpy().view(np.uint16), km)
    assert np.array_equal(c.v_meta[:, :, :T].cpu().numpy().view(np.uint16), vm)
    assert c.seq_lens.tolist() == [T] * 3


@pytest.mark.parametrize("G,g", [(128, 1), (128, 2), (128, 4), (128, 8), (64, 1), (64, 4),
                                 (32, 1), (32, 2)])
def test_decode_attention(kvq, G, g, fmt):
    H = 2
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=H, q_heads=H * g, bits=8, group=G)
    lens = [300, 45, 1]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, max(lens), DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    c = _alloc(kvq, B, H, 320, G, fmt)
    fill_cache(kvq, c, k, v, lens)
    out = torch.full((B, H * g, 128), float("nan"), device=DEV)
    lse = torch.full((B, H * g), float("nan"), device=DEV)
    ws = kvq.alloc_workspace(c, H * g, 0, device=DEV)
    kvq.kvq_decode_attention(c, q, out, lse, ws)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws) == 0
    seg = oracle_segment(k, v, 8, G, fmt)
    ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [lens], 128 ** -0.5)
    assert_close(out, ref, lse, lref, what=f"{fmt} G{G} g{g}")


def test_decode_step(kvq, fmt):
    """Append + attention in one call on an FP8 cache, several steps."""
    H, g, G = 2, 4, 64
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(kv_heads=H, q_heads=H * g, bits=8,
                                                          group=G)
    lens = [100, 7]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, max(lens), DEV, batch=B)
    c = _alloc(kvq, B, H, 128, G, fmt)
    fill_cache(kvq, c, k, v, lens)
    ws = kvq.alloc_workspace(c, H * g, 0, device=DEV)
    hist_k = [[k[b, :, :lens[b]]] for b in range(B)]
    hist_v = [[v[b, :, :lens[b]]] for b in range(B)]
    cur = list(lens)
    for s in range(3):
        kn, vn = workloads.kv_tokens(wl, 1, DEV, stream_extra=40 + s, batch=B)
        q = workloads.queries(wl, DEV, step=s, batch=B)
        out = torch.empty((B, H * g, 128), device=DEV)
        lse = torch.empty((B, H * g), device=DEV)
        kvq.kvq_decode_step(c, kn, vn, q, out, lse, ws)
        torch.cuda.synchronize()
        for b in range(B):
            hist_k[b].append(kn[b])
            hist_v[b].append(vn[b])
            cur[b] += 1
        assert c.seq_lens.tolist() == cur
        T = max(cur)
        kk = torch.zeros((B, H, T, 128), dtype=torch.float16, device=DEV)
        vv = torch.zeros_like(kk)
        for b in range(B):
            kk[b, :, :cur[b]] = torch.cat(hist_k[b], 1)
            vv[b, :, :cur[b]] = torch.cat(hist_v[b], 1)
        seg = oracle_segment(kk, vv, 8, G, fmt)
        ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [cur], 128 ** -0.5)
        assert_close(out, ref, lse, lref, what=f"{fmt} step {s}")
        for b in range(B):
            n = cur[b]
            assert np.array_equal(c.k_codes[b, :, :n].cpu().numpy(), seg["k_codes"][b, :, :n])
            assert np.array_equal(c.v_meta[b, :, :n].cpu().numpy().view(np.uint16),
                                  seg["v_meta"][b, :, :n])
