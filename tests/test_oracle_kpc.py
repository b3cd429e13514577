"""Pins of the oracle's per-channel K grouping (KV-cache page, INT8 item: the
Key is quantized per channel; reading R16: blocks of 32 tokens, one (s, z) per
channel and block).  Per-channel quantization of a block is per-token group
quantization of the transposed block, whose formula is pinned elsewhere; the
codes must also land at their channel's bit offset of each token row, keep
the half-step bound, and give attention equal to torch's on the dequantized
values."""
import numpy as np
import torch

import oracle

T = oracle.KPC_BLOCK


def _unpack(codes, bits, n):
    """Codes [rows, n * bits / 8] -> integers [rows, n] (element j at bit j * bits)."""
    j = np.arange(n)
    byte = codes[:, (j * bits) // 8].astype(np.int64)
    return (byte >> ((j * bits) % 8)) & ((1 << bits) - 1)


def _block(rng, scale=3.0):
    x = rng.standard_normal((T, 128)) * scale
    x[:, 5] = np.linspace(-40, 90, T)       # one channel with its own range
    x[:, 77] = 2.5                          # a constant channel
    return x.astype(np.float16)


def test_block_is_per_token_quantization_of_the_transposed_block():
    rng = np.random.default_rng(21)
    for bits in (2, 4, 8):
        x = _block(rng)
        codes, meta = oracle.quantize_block_channels(x.view(np.uint16), bits)
        ct, mt = oracle.quantize_rows(np.ascontiguousarray(x.T).view(np.uint16), T, bits)
        assert np.array_equal(meta, mt[:, 0, :])
        assert np.array_equal(_unpack(codes, bits, 128), _unpack(ct, bits, T).T)


def test_channel_codes_sit_at_their_bit_offset():
    """Channel 5 spans [-40, 90] over the block: its codes run 0 .. qmax in
    token order, at bits 5 * b of every row; the constant channel 77 gets one
    code throughout."""
    rng = np.random.default_rng(22)
    x = _block(rng)
    codes, meta = oracle.quantize_block_channels(x.view(np.uint16), 4)
    c = _unpack(codes, 4, 128)
    assert c[0, 5] == 0 and c[-1, 5] == 15
    assert np.all(np.diff(c[:, 5]) >= 0)
    assert len(set(c[:, 77].tolist())) == 1
    s5 = meta[5, 0:1].view(np.float16)[0]
    assert abs(float(s5) - 130.0 / 15) < 0.01


def test_half_step_bound_per_channel():
    rng = np.random.default_rng(23)
    for bits in (2, 4, 8):
        x = _block(rng, scale=rng.choice([1e-3, 1.0, 200.0]))
        codes, meta = oracle.quantize_block_channels(x.view(np.uint16), bits)
        xh = oracle.dequantize_block_channels(codes, meta, 128, bits)
        s = meta[:, 0].view(np.float16).astype(np.float64)
        ok = np.abs(x.astype(np.float64) - xh) <= s[None, :] / 2 * (1 + 2.0**-12)
        # the constant channel 77 (2.5) hits the 1e-5 scale floor and its zero
        # point saturates at -65504 (reading R4's stated consequence): every
        # other channel keeps the bound
        assert np.all(np.delete(ok, 77, axis=1))
        assert meta[77, 1] == np.float16(-65504).view(np.uint16)


def test_attention_over_a_per_channel_segment_matches_torch():
    rng = np.random.default_rng(24)
    B, H, L, g = 2, 2, 3 * T, 4
    k = (rng.standard_normal((B, H, L, 128)) * 2).astype(np.float16)
    v = rng.standard_normal((B, H, L, 128)).astype(np.float16)
    q = rng.standard_normal((B, H * g, 128)).astype(np.float16)
    kc, km = oracle.quantize_cache_channels(k.view(np.uint16), 4)
    vc, vm = oracle.quantize_cache(v.view(np.uint16), 64, 4)
    seg = dict(k_codes=kc, k_meta=km, v_codes=vc, v_meta=vm, bits=4, group=64, k_channels=True)
    lens = np.array([L, 2 * T])
    o, lse = oracle.decode_attention(q.view(np.uint16), False, [seg], [lens], 128 ** -0.5)
    for b in range(B):
        for h in range(H):
            n = int(lens[b])
            K = oracle.dequantize_channels(kc[b, h], km[b, h], n, 128, 4)
            V = oracle.dequantize_rows(vc[b, h, :n], vm[b, h, :n], 128, 64, 4)
            qq = torch.from_numpy(q[b, h * g:(h + 1) * g].astype(np.float64))
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq[None, :, None], torch.from_numpy(K)[None, None].expand(1, g, n, 128),
                torch.from_numpy(V)[None, None].expand(1, g, n, 128), scale=128 ** -0.5)
            assert np.allclose(o[b, h * g:(h + 1) * g], ref[0, :, 0].numpy(), atol=1e-12)


def test_bf16_block_with_the_worked_example_in_one_channel():
    """bf16 input (reading R19) through the per-channel path: channel 9 of a
    block holds the hand-worked bf16 INT4 group of tests/golden (values beyond
    the fp16 range), four times over, so its min and max, and hence its
    scale, zero point and codes, are the fixture's."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                    "bf16_worked_example.json")))
    pat = np.array([int(h, 16) for h in g["bf16_patterns"]], np.uint16)
    rng = np.random.default_rng(25)
    x = torch.from_numpy(rng.standard_normal((T, 128)).astype(np.float32))
    xb = x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16).copy()
    xb[:, 9] = np.tile(pat, T // len(pat))
    codes, meta = oracle.quantize_block_channels(xb, 4, in_dtype="bf16")
    assert _unpack(codes, 4, 128)[:, 9].tolist() == g["codes"] * (T // len(pat))
    assert int(meta[9, 0]) == int(g["scale_f16"], 16)
    assert int(meta[9, 1]) == int(g["zero_f16"], 16)


def test_bf16_block_of_fp16_values_matches_the_fp16_path():
    """A bf16 block whose values are all fp16 values gives exactly the codes
    and (s, z) of its fp16 form (both widen to the same fp32 values)."""
    rng = np.random.default_rng(26)
    for bits in (2, 4, 8):
        x = torch.from_numpy(_block(rng).astype(np.float32))
        xb = x.to(torch.bfloat16).float()
        assert torch.equal(xb.half().float(), xb)
        b16 = xb.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)
        f16 = xb.to(torch.float16).contiguous().view(torch.int16).numpy().view(np.uint16)
        cb, mb = oracle.quantize_block_channels(b16, bits, in_dtype="bf16")
        cf, mf = oracle.quantize_block_channels(f16, bits)
        assert np.array_equal(cb, cf) and np.array_equal(mb, mf), bits
