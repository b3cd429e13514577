"""GPU parity of the symmetric INT8 KV format (KV-cache page, INT8 item:
scale amax / 127, round, clamp; the oracle's reading R15): codes and scales
written by kvq_quantize_append byte for byte equal to the oracle's (both the
per-sequence append kernel and the bulk kernel), and decode attention over
them within the attention tolerance of the fp64 oracle."""
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


def _alloc(kvq, B, H, max_tokens, G):
    c = kvq.QuantizedKVCache.allocate(B, H, 128, max_tokens, 8, G, DEV,
                                      fmt=kvq.KVQ_FMT_INT8_SYM)
    c.k_codes.fill_(0x80)  # stale codes (-128) and NaN scales in unused slots
    c.v_codes.fill_(0x7F)
    c.k_meta.view(torch.int16).fill_(-1)
    c.v_meta.view(torch.int16).fill_(-1)
    return c


def _adversarial(k, v):
    k[0, 0, 0] = 0.0
    k[0, 0, 1] = 3.0
    k[0, 0, 2] = (torch.randn(128, device=DEV) * 1e-6).half()
    k[0, 0, 3] = (torch.randn(128, device=DEV) * 20000).clamp(-60000, 60000).half()
    # exact ties at s = 1 (amax 127): x.5 values round to even
    row = torch.tensor([127.0, -127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5], device=DEV)
    k[0, 1, 4] = row.repeat(16).half()
    v[1, 0, 5] = -0.0


@pytest.mark.parametrize("H,T", [(2, 7), (4, 77)])  # under 8 tokens: append kernel; 77: bulk
@pytest.mark.parametrize("G", [32, 64, 128])
def test_quantize_bit_exact(kvq, G, H, T):
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(batch=3, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV)
    _adversarial(k, v)
    c = _alloc(kvq, 3, H, 128, G)
    c.seq_lens.copy_(torch.tensor([0, 5, 60], dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    kc, km = oracle.quantize_cache(f16_bits(k), G, 8, "sym8")
    vc, vm = oracle.quantize_cache(f16_bits(v), G, 8, "sym8")
    for b, st in enumerate([0, 5, 60]):
        n = min(T, 128 - st)
        p = slice(st, st + n)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b, :, :n])
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b, :, :n])
        assert np.array_equal(c.k_meta[b, :, p].cpu().numpy().view(np.uint16), km[b, :, :n])
        assert np.array_equal(c.v_meta[b, :, p].cpu().numpy().view(np.uint16), vm[b, :, :n])
    assert c.seq_lens.tolist() == [min(st + T, 128) for st in (0, 5, 60)]


@pytest.mark.parametrize("G,g", [(128, 1), (128, 2), (128, 4), (128, 8), (64, 1), (64, 4),
                                 (32, 1), (32, 2)])
def test_decode_attention(kvq, G, g):
    H = 2
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=H, q_heads=H * g, bits=8, group=G)
    lens = [300, 45, 1]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, max(lens), DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    c = _alloc(kvq, B, H, 320, G)
    fill_cache(kvq, c, k, v, lens)
    out = torch.full((B, H * g, 128), float("nan"), device=DEV)
    lse = torch.full((B, H * g), float("nan"), device=DEV)
    ws = kvq.alloc_workspace(c, H * g, 0, device=DEV)
    kvq.kvq_decode_attention(c, q, out, lse, ws)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws) == 0
    seg = oracle_segment(k, v, 8, G, "sym8")
    ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [lens], 128 ** -0.5)
    assert_close(out, ref, lse, lref, what=f"sym8 G{G} g{g}")


def test_decode_step(kvq):
    """Append + attention in one call on a symmetric INT8 cache, several
    steps."""
    H, g, G = 2, 4, 64
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(kv_heads=H, q_heads=H * g, bits=8,
                                                          group=G)
    lens = [100, 7]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, max(lens), DEV, batch=B)
    c = _alloc(kvq, B, H, 128, G)
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
        seg = oracle_segment(kk, vv, 8, G, "sym8")
        ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [cur], 128 ** -0.5)
        assert_close(out, ref, lse, lref, what=f"sym8 step {s}")
        for b in range(B):
            n = cur[b]
            assert np.array_equal(c.k_codes[b, :, :n].cpu().numpy(), seg["k_codes"][b, :, :n])
            assert np.array_equal(c.v_meta[b, :, :n].cpu().numpy().view(np.uint16),
                                  seg["v_meta"][b, :, :n])
