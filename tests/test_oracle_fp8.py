"""Pins of the oracle's FP8 E4M3 format (KV-cache page, FP8 KV cache with a
dynamic scale; reading R14 of oracle/kvq_oracle.c): the codec against
PyTorch's float8_e4m3fn (a library routine), a hand-derived group, and the
rounding bound of the dequantized values."""
import json
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_to_f64(codes)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    same = (v == t) | (np.isnan(v) & np.isnan(t))
    assert same.all()
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and v[0x7E] == 448.0 and v[0x01] == 2.0**-9


def test_encode_round_trips_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    v = oracle.e4m3_to_f64(codes)
    fin = ~np.isnan(v)
    assert np.array_equal(oracle.f32_to_e4m3(v[fin].astype(np.float32)), codes[fin])


def test_encode_matches_torch_including_ties():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 40, rng.standard_normal(20000) * 0.01])
    x = np.clip(x, -448, 448).astype(np.float32)
    # every midpoint between neighbouring finite values (exact ties)
    v = np.unique(oracle.e4m3_to_f64(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f32_to_e4m3(x), ref)


def test_saturation_and_nan():
    c = oracle.f32_to_e4m3(np.array([1000.0, -1000.0, np.inf, -np.inf, np.nan, -0.0], np.float32))
    assert c.tolist() == [0x7E, 0xFE, 0x7E, 0xFE, 0x7F, 0x80]


def test_worked_groups():
    ex = json.load(open(os.path.join(GOLDEN, "fp8_worked_example.json")))
    for g in ex["groups"]:
        x16 = np.asarray(g["x"], np.float16)
        assert np.array_equal(x16.astype(np.float64), np.asarray(g["x"]))  # exact in fp16
        code, s16 = oracle.quantize_group_fp8(x16.view(np.uint16))
        assert code.tolist() == g["codes"] and s16 == int(g["s16"], 16)
        if "x_hat" in g:
            meta = np.array([[[s16, 0]]], np.uint16)
            xh = oracle.dequantize_rows(code[None], meta, len(code), len(code), 8, "fp8")
            assert xh[0].tolist() == g["x_hat"]


def test_rows_rounding_bound():
    """Every element is within half an E4M3 step of x / s, times s: relative
    2^-4 for normal values, 2^-10 s in the subnormal range (plus the fp32
    rounding of the division)."""
    rng = np.random.default_rng(5)
    G, D = 64, 128
    x = np.concatenate([rng.standard_normal((300, D)), rng.standard_normal((100, D)) * 40,
                        rng.standard_normal((50, D)) * 1e-3]).astype(np.float16)
    codes, meta = oracle.quantize_rows(x.view(np.uint16), G, 8, "fp8")
    assert np.all(meta[..., 1] == 0)
    xh = oracle.dequantize_rows(codes, meta, D, G, 8, "fp8")
    s = np.repeat(meta[..., 0].view(np.float16).astype(np.float64), G, axis=1)
    xd = x.astype(np.float64)
    bound = np.maximum(np.abs(xd) * 2.0**-4, s * 2.0**-10) * (1 + 2.0**-20) + np.abs(xd) * 2.0**-23
    assert np.all(np.abs(xd - xh) <= bound)
    # the group maximum lands on at most 448 steps of s, and s is the stored
    # scale rounded up from amax / 448
    amax = np.abs(xd).reshape(-1, D // G, G).max(-1)
    sg = meta[..., 0].view(np.float16).astype(np.float64)
    assert np.all(amax / sg <= 448.0)
    assert np.all(sg >= np.maximum(amax / 448, 1e-5) * (1 - 2.0**-23))
