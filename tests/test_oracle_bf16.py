"""Pins of the oracle's bfloat16 input path (kvq_quantize_append with bf16
K/V: the KV-cache page's caches come in bf16 as well as fp16).  The values
are read exactly into fp32 and the group arithmetic that follows is the fp16
path's, so the pins are:
  - a hand-derived INT4 group of bf16 values beyond the fp16 range
    (tests/golden/bf16_worked_example.json);
  - bf16 rows whose values are all fp16 values give exactly the codes, scales
    and zero points of the (separately pinned) fp16 path, in every format;
  - the half-step bound |x - x_hat| <= s/2 on random bf16 groups;
  - each code is the nearest grid point, found exactly with fractions."""
import json
import os
from fractions import Fraction

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def _f16_bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float16).contiguous().view(torch.int16).numpy().view(np.uint16)


def test_bf16_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "bf16_worked_example.json")))
    pat = np.array([int(h, 16) for h in g["bf16_patterns"]], np.uint16)
    vals = torch.tensor(g["values"], dtype=torch.float32)
    assert np.array_equal(_bf16_bits(vals), pat)  # the fixture's patterns are the values
    codes, meta = oracle.quantize_rows(pat[None], g["group"], g["bits"], in_dtype="bf16")
    unpacked = [(codes[0, j // 2] >> (4 * (j % 2))) & 15 for j in range(g["group"])]
    assert unpacked == g["codes"]
    assert int(meta[0, 0, 0]) == int(g["scale_f16"], 16)
    assert int(meta[0, 0, 1]) == int(g["zero_f16"], 16)


def test_bf16_rows_of_fp16_values_match_the_fp16_path():
    gen = torch.Generator().manual_seed(11)
    x = torch.randn((64, 128), generator=gen) * 3
    x[5] *= 1000.0                      # large, still fp16 values after bf16 rounding
    x[9] = 0.0
    x[17, :7] = torch.tensor([0.5, -0.5, 1.5, 2.5, -2.5, 3.5, 4.5])  # ties
    xb = x.to(torch.bfloat16).float()   # bf16 values ...
    assert torch.equal(xb.half().float(), xb)  # ... that are all fp16 values
    b16, f16 = _bf16_bits(xb), _f16_bits(xb)
    for fmt, bits, groups in (("int", 2, (32, 64, 128)), ("int", 4, (32, 64, 128)),
                              ("int", 8, (32, 64, 128)), ("fp8", 8, (64, 128)),
                              ("sym8", 8, (64, 128)), ("e5m2", 8, (64, 128))):
        for G in groups:
            cb, mb = oracle.quantize_rows(b16, G, bits, fmt, in_dtype="bf16")
            cf, mf = oracle.quantize_rows(f16, G, bits, fmt)
            assert np.array_equal(cb, cf), (fmt, bits, G)
            assert np.array_equal(mb, mf), (fmt, bits, G)


def _unpack(codes, D, bits):
    out = np.zeros((codes.shape[0], D), np.int64)
    for j in range(D):
        out[:, j] = (codes[:, (j * bits) // 8] >> ((j * bits) % 8)) & ((1 << bits) - 1)
    return out


def test_bf16_half_step_bound_and_nearest_code():
    gen = torch.Generator().manual_seed(12)
    x = torch.randn((40, 128), generator=gen)
    # rows from 1e-3 to 1e4: every group's (max - min) / qmax stays an fp16
    # value (the scale is stored in fp16; wider groups are out of contract)
    x[::4] *= torch.logspace(-3, 4, 10)[:, None]
    xb = x.to(torch.bfloat16).float().numpy().astype(np.float64)
    pat = _bf16_bits(x)
    for bits in (2, 4, 8):
        for G in (32, 64, 128):
            codes, meta = oracle.quantize_rows(pat, G, bits, in_dtype="bf16")
            c = _unpack(codes, 128, bits)
            s = meta[..., 0].view(np.float16).astype(np.float64).repeat(G, axis=1)
            z = meta[..., 1].view(np.float16).astype(np.float64).repeat(G, axis=1)
            xhat = (c - z) * s
            ok = np.abs(z) <= 2048  # z exact in fp16 (R4): the bound holds
            assert np.all(np.abs(xb - xhat)[ok] <= s[ok] / 2 * (1 + 2.0 ** -22)), (bits, G)
            # nearest code of [0, 2^bits - 1] to x / s + z, ties to even, exactly
            qmax = (1 << bits) - 1
            for r in range(0, xb.shape[0], 7):
                for j in range(0, 128, 5):
                    t = Fraction(float(xb[r, j])) / Fraction(float(s[r, j])) + Fraction(
                        float(z[r, j]))
                    fl = t.numerator // t.denominator
                    frac = t - fl
                    near = fl + (1 if frac > Fraction(1, 2) or
                                 (frac == Fraction(1, 2) and fl % 2 == 1) else 0)
                    assert c[r, j] == min(max(near, 0), qmax), (bits, G, r, j)
