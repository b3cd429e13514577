"""GPU parity of kvq_decode_step (quantize-on-write of one new token per
(sequence, KV head) inside the split-K kernel for the tokens-on-M formats,
then attention over the cache including it) against the fp64 oracle on the
same seeded fp16 inputs, through both its one-call and its two-call forms."""
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


def _poison(c):
    c.k_codes.fill_(0x5A)
    c.v_codes.fill_(0xA5)
    c.k_meta.view(torch.int16).fill_(-1)  # NaN scales in unused slots
    c.v_meta.view(torch.int16).fill_(-1)


# (bits, G, g): tokens-on-M formats (one launch) and one 16-row format
# (G64, g = 8: the append kernel, then the attention)
FORMATS = [(8, 128, 1), (4, 64, 4), (2, 32, 1), (4, 32, 2), (2, 128, 8), (4, 64, 8)]


@pytest.mark.parametrize("two_calls", [False, True])
@pytest.mark.parametrize("bits,G,g", FORMATS)
def test_decode_step_matches_append_then_attention(kvq, bits, G, g, two_calls):
    H = 2
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=H, q_heads=H * g, bits=bits,
                                                     group=G)
    lens = [254, 37, 0, 129]  # the first reaches max_tokens = 256 and then drops tokens
    B, T0, max_tokens, steps = len(lens), max(lens), 256, 4
    k, v = workloads.kv_tokens(wl, T0, DEV, batch=B)
    c = kvq.QuantizedKVCache.allocate(B, H, 128, max_tokens, bits, G, DEV)
    _poison(c)
    fill_cache(kvq, c, k, v, lens)
    ws = kvq.alloc_workspace(c, H * g, 0, device=DEV)
    # host mirror of every sequence's fp16 history, in cache order
    hist_k = [[k[b, :, :lens[b]]] for b in range(B)]
    hist_v = [[v[b, :, :lens[b]]] for b in range(B)]
    cur = list(lens)
    for s in range(steps):
        kn, vn = workloads.kv_tokens(wl, 1, DEV, stream_extra=20 + s, batch=B)
        q = workloads.queries(wl, DEV, step=s, batch=B)
        out = torch.full((B, H * g, 128), float("nan"), device=DEV)
        lse = torch.full((B, H * g), float("nan"), device=DEV)
        if two_calls:
            kvq.kvq_decode_step_partials(c, kn, vn, q, out, lse, ws)
            kvq.kvq_decode_merge(c, q, out, lse, ws)
        else:
            kvq.kvq_decode_step(c, kn, vn, q, out, lse, ws)
        torch.cuda.synchronize()
        assert kvq.workspace_error_word(ws) == 0
        for b in range(B):
            if cur[b] < max_tokens:
                hist_k[b].append(kn[b])
                hist_v[b].append(vn[b])
                cur[b] += 1
        assert c.seq_lens.tolist() == cur, f"step {s}: seq_lens"
        # the oracle's cache of the same history, padded to one length
        T = max(cur)
        kk = torch.zeros((B, H, T, 128), dtype=torch.float16, device=DEV)
        vv = torch.zeros_like(kk)
        for b in range(B):
            hk = torch.cat(hist_k[b], 1)
            hv = torch.cat(hist_v[b], 1)
            kk[b, :, :hk.shape[1]] = hk
            vv[b, :, :hv.shape[1]] = hv
        seg = oracle_segment(kk, vv, bits, G)
        ref, lref = oracle.decode_attention(q_bits(q), q.dtype == torch.bfloat16, [seg], [cur],
                                            128 ** -0.5)
        mask = np.array([n > 0 for n in cur])
        assert_close(out, ref, lse, lref, mask=mask, what=f"bits{bits} G{G} g{g} step {s}")
        assert torch.all(out[~torch.as_tensor(mask, device=DEV)] == 0)
    # the cache holds exactly the oracle's codes and (scale, zero) of every token
    for b in range(B):
        n = cur[b]
        if n == 0:
            continue
        np.testing.assert_array_equal(c.k_codes[b, :, :n].cpu().numpy(), seg["k_codes"][b, :, :n])
        np.testing.assert_array_equal(c.v_codes[b, :, :n].cpu().numpy(), seg["v_codes"][b, :, :n])
        km = c.k_meta[b, :, :n].cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(km.reshape(seg["k_meta"][b, :, :n].shape),
                                      seg["k_meta"][b, :, :n])


@pytest.mark.parametrize("bits,G,g", [(4, 64, 4), (8, 128, 1), (4, 64, 8)])
def test_attention_call_equals_two_phase_on_one_workspace(kvq, bits, G, g):
    """kvq_decode_attention agrees with kvq_decode_partials + kvq_decode_merge
    and with the oracle, call after call on one workspace (its counters
    return to zero)."""
    H = 2
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=H, q_heads=H * g, bits=bits,
                                                     group=G)
    lens = [2000, 777, 1]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, max(lens), DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    c = kvq.QuantizedKVCache.allocate(B, H, 128, 2048, bits, G, DEV)
    _poison(c)
    fill_cache(kvq, c, k, v, lens)
    ws = kvq.alloc_workspace(c, H * g, 0, device=DEV)
    seg = oracle_segment(k, v, bits, G)
    ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [lens], 128 ** -0.5)
    outs = []
    for rep in range(3):
        out = torch.full((B, H * g, 128), float("nan"), device=DEV)
        lse = torch.full((B, H * g), float("nan"), device=DEV)
        kvq.kvq_decode_attention(c, q, out, lse, ws)
        torch.cuda.synchronize()
        assert kvq.workspace_error_word(ws) == 0
        assert_close(out, ref, lse, lref, what=f"call {rep}")
        outs.append(out.clone())
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    out2 = torch.full_like(outs[0], float("nan"))
    lse2 = torch.full((B, H * g), float("nan"), device=DEV)
    kvq.kvq_decode_partials(c, q, out2, lse2, ws)
    kvq.kvq_decode_merge(c, q, out2, lse2, ws)
    torch.cuda.synchronize()
    assert_close(out2, ref, lse2, lref, what="two-phase merge")
    d = (out2 - outs[0]).abs().max().item()
    assert d <= 1e-5 * max(1.0, outs[0].abs().max().item())
