"""Pins of the oracle's symmetric INT8 format (KV-cache page, INT8 item:
scale = amax / 127, round, clamp to [-128, 127]; reading R15): hand-derived
groups, the page's own torch formulation on random groups, the half-step
error bound, and the two's complement dequantization."""
import json
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _f16(x):
    return np.asarray(x, np.float16).view(np.uint16)


def test_worked_groups():
    with open(os.path.join(GOLDEN, "sym8_worked_example.json")) as f:
        ex = json.load(f)
    for g in ex["groups"]:
        code, s16 = oracle.quantize_group_sym8(_f16(g["x"]))
        assert code.tolist() == g["codes"], g
        assert s16 == int(g["s16"], 16), g


def _listing_in_torch(x16: np.ndarray, G: int):
    """The page's listing on one group per row of G values (the scale of a
    group reduced over its values, round, clamp, int8), with the scale kept
    in fp16 rounded up from its fp32 value and floored at 1e-5 (R15)."""
    x = torch.from_numpy(x16.view(np.float16)).float().reshape(-1, G)
    s32 = torch.clamp(x.abs().amax(dim=-1, keepdim=True) / 127.0, min=1e-5)
    s16 = s32.half()
    up = s16.float() < s32
    s16 = torch.where(up, torch.nextafter(s16, torch.full_like(s16, float("inf"))), s16)
    q = torch.round(x / s16.float()).clamp(-128, 127).to(torch.int8)
    return q.reshape(x16.shape[0], -1), s16.reshape(x16.shape[0], -1)


def test_matches_the_page_listing_in_torch():
    rng = np.random.default_rng(11)
    for G in (32, 64, 128):
        rows = []
        for scale in (1e-7, 1e-3, 1.0, 30.0, 3000.0):
            rows.append(rng.standard_normal((40, 128)) * scale)
        rows.append(np.round(rng.standard_normal((40, 128)) * 4) / 2)  # many exact .5 ties
        x16 = np.clip(np.concatenate(rows), -65504, 65504).astype(np.float16).view(np.uint16)
        codes, meta = oracle.quantize_rows(x16, G, 8, "sym8")
        ref_q, ref_s = _listing_in_torch(x16, G)
        assert np.array_equal(codes.view(np.int8), ref_q.numpy())
        assert np.array_equal(meta[:, :, 0], ref_s.view(torch.int16).numpy().view(np.uint16))
        assert np.all(meta[:, :, 1] == 0)


def test_half_step_bound_and_code_range():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal((300, 128)) * rng.choice([1e-3, 1, 50], (300, 1))).astype(np.float16)
    codes, meta = oracle.quantize_rows(x.view(np.uint16), 64, 8, "sym8")
    c = codes.view(np.int8).astype(np.int64)
    assert c.min() >= -127 and c.max() <= 127  # the rounded-up scale keeps |x / s| <= 127
    xh = oracle.dequantize_rows(codes, meta, 128, 64, 8, "sym8")
    s = np.repeat(meta[:, :, 0].view(np.float16).astype(np.float64), 64, axis=1)
    assert np.all(np.abs(x.astype(np.float64) - xh) <= s / 2 * (1 + 2.0**-12))


def test_dequantize_is_signed_code_times_scale():
    codes = np.array([[0, 1, 127, 128, 129, 255, 200, 56]], np.uint8)
    meta = np.array([[[np.float16(0.25).view(np.uint16), 0]]], np.uint16)
    xh = oracle.dequantize_rows(codes, meta, 8, 8, 8, "sym8")
    assert xh.tolist() == [[0.0, 0.25, 31.75, -32.0, -31.75, -0.25, -14.0, 14.0]]
