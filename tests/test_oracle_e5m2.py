"""Pins of the oracle's FP8 E5M2 format (KV-cache page, FP8 item: E4M3 or
E5M2; reading R17): the codec against torch's float8_e5m2 on every code and
on every midpoint between neighbouring values (ties), a hand-derived group,
and the rounding bound of the group quantization."""
import json
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e5m2_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e5m2).float().numpy().astype(np.float64)
    assert np.all((mine == ref) | (np.isnan(mine) & np.isnan(ref)))


def test_encode_matches_torch_on_midpoints_and_random_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e5m2).float().numpy().astype(np.float64)
    fin = np.unique(vals[np.isfinite(vals)])
    rng = np.random.default_rng(31)
    x = np.concatenate([(fin[:-1] + fin[1:]) / 2, fin,
                        rng.standard_normal(4000) * rng.choice([1e-4, 1, 300, 20000], 4000)])
    x = np.clip(x, -57344, 57344).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f32_to_e5m2(x), ref)
    # saturation instead of infinity past the largest finite value
    assert oracle.f32_to_e5m2(np.array([1e6, -1e9], np.float32)).tolist() == [0x7B, 0xFB]


def test_worked_group():
    with open(os.path.join(GOLDEN, "e5m2_worked_example.json")) as f:
        ex = json.load(f)
    for g in ex["groups"]:
        code, s16 = oracle.quantize_group_e5m2(np.asarray(g["x"], np.float16).view(np.uint16))
        assert code.tolist() == g["codes"]
        assert s16 == int(g["s16"], 16)


def test_rounding_bound():
    """Every value is within half an E5M2 step (relative 2^-3 of its
    magnitude, or half the subnormal step) of its dequantized value."""
    rng = np.random.default_rng(32)
    x = (rng.standard_normal((200, 128)) * rng.choice([1e-3, 1, 60], (200, 1))).astype(np.float16)
    codes, meta = oracle.quantize_rows(x.view(np.uint16), 64, 8, "e5m2")
    xh = oracle.dequantize_rows(codes, meta, 128, 64, 8, "e5m2")
    s = np.repeat(meta[:, :, 0].view(np.float16).astype(np.float64), 64, axis=1)
    a = np.abs(x.astype(np.float64))
    bound = np.maximum(a * 2.0**-3, s * 2.0**-17) * (1 + 2.0**-10)
    assert np.all(np.abs(x.astype(np.float64) - xh) <= bound)
    assert np.all(np.isfinite(xh))
