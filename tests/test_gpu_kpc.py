"""GPU parity of per-channel K grouping (KV-cache page, INT8 item: the Key is
quantized per channel; the oracle's reading R16: blocks of 32 tokens, one
(s, z) per channel and block): K codes and block meta written by
kvq_quantize_append byte for byte equal to the oracle's, V per token as
before."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import f16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
TB = 32


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def _alloc(kvq, B, H, cap, bits, G):
    c = kvq.QuantizedKVCache.allocate(B, H, 128, cap, bits, G, DEV, k_axis=kvq.KVQ_AXIS_CHANNEL)
    c.k_codes.fill_(0xA5)
    c.v_codes.fill_(0x5A)
    c.k_meta.view(torch.int16).fill_(-1)
    c.v_meta.view(torch.int16).fill_(-1)
    return c


@pytest.mark.parametrize("H,T", [(2, 64), (4, 160)])  # V rows per sequence 128 / 640
@pytest.mark.parametrize("bits,G", [(4, 64), (8, 128), (2, 32), (4, 32)])
def test_quantize_channels_bit_exact(kvq, bits, G, H, T):
    B, cap = 4, 192
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV)
    k[0, 0, 3, 5] = 300.0  # an outlier inside one channel's block
    c = _alloc(kvq, B, H, cap, bits, G)
    start = [0, 32, 5, 96]  # sequence 2 is off a block boundary: left untouched
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [min(s + T, cap) if s % TB == 0 else s for s in start]
    kc, km = oracle.quantize_cache_channels(f16_bits(k), bits)
    vc, vm = oracle.quantize_cache(f16_bits(v), G, bits)
    for b, st in enumerate(start):
        if st % TB:
            assert (c.k_codes[b] == 0xA5).all() and (c.v_codes[b] == 0x5A).all()
            assert (c.k_meta[b].view(torch.int16) == -1).all()
            continue
        n = min(T, cap - st)
        p = slice(st, st + n)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b, :, :n])
        blk = slice(st // TB, (st + n) // TB)
        assert np.array_equal(c.k_meta[b, :, blk].cpu().numpy().view(np.uint16),
                              km[b, :, :n // TB])
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b, :, :n])
        assert np.array_equal(c.v_meta[b, :, p].cpu().numpy().view(np.uint16), vm[b, :, :n])
        assert (c.k_codes[b, :, :st] == 0xA5).all()
        assert (c.k_meta[b, :, :st // TB].view(torch.int16) == -1).all()


@pytest.mark.parametrize("bits", [4, 2])
def test_quantize_channels_many_blocks(kvq, bits):
    """Thousands of 32-token blocks, several per CTA of the persistent channel
    kernel (its copy ring runs over many blocks), a few of them on the clamped
    path: sequence 1's last block runs past max_tokens and is dropped,
    sequence 2 is off a block boundary and left untouched."""
    B, H, T, cap = 3, 8, 8192, 8192
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV)
    # blocks that take the clamped path: a constant channel (the scale floor
    # puts |z| far past 2048) and a channel block spanning a huge range
    k[1, 2, 64:96, 7] = 3.0
    k[0, 5, 4096:4128, 100] = torch.linspace(-60000.0, 60000.0, 32)
    c = _alloc(kvq, B, H, cap, bits, 64)
    start = [0, 32, 7]
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [T, cap, 7]
    kc, km = oracle.quantize_cache_channels(f16_bits(k), bits)
    for b, st in enumerate(start[:2]):
        n = min(T, cap - st)
        assert np.array_equal(c.k_codes[b, :, st:st + n].cpu().numpy(), kc[b, :, :n])
        assert np.array_equal(c.k_meta[b, :, st // TB:(st + n) // TB].cpu().numpy().view(np.uint16),
                              km[b, :, :n // TB])
    assert (c.k_codes[2] == 0xA5).all() and (c.k_meta[2].view(torch.int16) == -1).all()


@pytest.mark.parametrize("bits", [4, 2, 8])
def test_quantize_channels_bf16_bit_exact(kvq, bits):
    """bf16 K/V (reading R19) through the per-channel K kernel and the
    per-token V kernel, against the oracle's bf16 path: thousands of blocks,
    several per CTA, and (at 4 and 8 bits) one channel block holding the
    hand-worked bf16 group of tests/golden (values beyond the fp16 range) four
    times over."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                    "bf16_worked_example.json")))
    B, H, T, cap = 2, 8, 4096, 4096 + 64
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV, dtype=torch.bfloat16)
    vals = torch.tensor(g["values"], dtype=torch.float32).to(torch.bfloat16)
    if (max(g["values"]) - min(g["values"])) / ((1 << bits) - 1) <= 65504:
        # planted where its scale fits fp16 (at 2 bits it does not, and the
        # header leaves such a group's codes unspecified)
        k[1, 3, 96:128, 9] = vals.repeat(TB // len(g["values"])).to(DEV)
    c = _alloc(kvq, B, H, cap, bits, 64)
    start = [0, 32]
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [T, T + 32]

    def b16(t):
        return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kc, km = oracle.quantize_cache_channels(b16(k), bits, in_dtype="bf16")
    vc, vm = oracle.quantize_cache(b16(v), 64, bits, in_dtype="bf16")
    if bits == g["bits"]:  # the worked block's scale and zero point
        assert int(km[1, 3, 3, 9, 0]) == int(g["scale_f16"], 16)
        assert int(km[1, 3, 3, 9, 1]) == int(g["zero_f16"], 16)
    for b, st in enumerate(start):
        p = slice(st, st + T)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b]), b
        assert np.array_equal(c.k_meta[b, :, st // TB:(st + T) // TB].cpu().numpy().view(np.uint16),
                              km[b]), b
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b]), b
        assert np.array_equal(c.v_meta[b, :, p].cpu().numpy().view(np.uint16), vm[b]), b


def _kpc_segment(k, v, bits, G):
    kc, km = oracle.quantize_cache_channels(f16_bits(k), bits)
    vc, vm = oracle.quantize_cache(f16_bits(v), G, bits)
    return dict(k_codes=kc, k_meta=km, v_codes=vc, v_meta=vm, bits=bits, group=G,
                k_channels=True)


@pytest.mark.parametrize("bits,G,g", [(4, 64, 4), (8, 128, 1), (4, 128, 4), (4, 128, 1)])
def test_decode_attention_channels(kvq, bits, G, g):
    """Attention over a per-channel-K cache (lengths on block boundaries, one
    sequence empty), then together with an fp16 residual segment holding
    each sequence's unfinished block: the KIVI-style pair."""
    from gpu_util import assert_close, fill_cache, fill_fp16_segment, q_bits
    H = 2
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(kv_heads=H, q_heads=H * g, bits=bits,
                                                          group=G)
    lens = [320, 64, 0, 32]
    B, T = len(lens), max(lens)
    k, v = workloads.kv_tokens(wl, T, DEV, batch=B)
    k[1, 0, 40, 3] = 250.0  # an outlier channel value inside one block
    q = workloads.queries(wl, DEV, batch=B)
    c = _alloc(kvq, B, H, 320, bits, G)
    fill_cache(kvq, c, k, v, lens)
    seg = _kpc_segment(k, v, bits, G)
    ws = kvq.alloc_workspace(c, H * g, 0, device=DEV)
    out = torch.full((B, H * g, 128), float("nan"), device=DEV)
    lse = torch.full((B, H * g), float("nan"), device=DEV)
    kvq.kvq_decode_attention(c, q, out, lse, ws)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws) == 0
    ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [lens], 128 ** -0.5)
    mask = np.array([n > 0 for n in lens])
    assert_close(out, ref, lse, lref, mask=mask, what=f"kpc b{bits} G{G} g{g}")
    # with the unfinished blocks in an fp16 segment
    rlens = [17, 31, 5, 0]
    kr, vr = workloads.kv_tokens(wl, 32, DEV, stream_extra=7, batch=B)
    r = kvq.QuantizedKVCache.allocate(B, H, 128, 64, 16, 128, DEV)
    fill_fp16_segment(r, kr, vr, rlens)
    segs = [c, r]
    ws2 = kvq.alloc_workspace(segs, H * g, 0, device=DEV)
    out2 = torch.full((B, H * g, 128), float("nan"), device=DEV)
    lse2 = torch.full((B, H * g), float("nan"), device=DEV)
    kvq.kvq_decode_attention(segs, q, out2, lse2, ws2)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws2) == 0
    rseg = dict(k_codes=f16_bits(kr).view(np.uint8).reshape(B, H, 32, -1),
                v_codes=f16_bits(vr).view(np.uint8).reshape(B, H, 32, -1), k_meta=None,
                v_meta=None, bits=16, group=128)
    ref2, lref2 = oracle.decode_attention(q_bits(q), False, [seg, rseg], [lens, rlens],
                                          128 ** -0.5)
    assert_close(out2, ref2, lse2, lref2, what=f"kpc + fp16 residual b{bits} G{G} g{g}")
