"""Pins of the oracle's Oaken group-shift codec ("大模型KV缓存量化技术：原理、
优化与实践" page, sections 3.1, 3.2.1, 3.2.2; reading R18): hand-derived rows,
brute force over the inner grid, the reduction to the 4-bit group quantizer
when a row's own range is the offline one, the half-step bounds of both
zones, and the slot invariants (outer elements only, ascending dims, at most
16, the rest zero)."""
import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _unpack4(codes):
    j = np.arange(codes.shape[1] * 2)
    return (codes[:, j // 2].astype(np.int64) >> ((j % 2) * 4)) & 15


def _params():
    # (s_in, z_in, s_out, outer_bits): fp16 inner scales, several zero points
    return [(0.125, 8, 0.25, 5), (0.0625, 3, 0.3, 6), (2.0, 12, 1.7, 7), (0.01171875, 0, 0.05, 5),
            (1.0, 15, 0.5, 6)]


def _rows(rng, s_in, z_in, n=300, D=128):
    t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
    span = t_hi - t_lo
    x = rng.uniform(t_lo - 0.6 * span, t_hi + 0.6 * span, (n, D))
    x[: n // 3] = rng.uniform(t_lo, t_hi, (n // 3, D))           # all inner
    k = rng.integers(-2, 18, (n // 4, D)) - z_in                 # on the grid and ties
    x[n // 3: n // 3 + n // 4] = (k + rng.choice([0.0, 0.5], (n // 4, D))) * s_in
    return x.astype(np.float16).view(np.uint16)


def test_worked_rows():
    with open(os.path.join(GOLDEN, "oaken_worked_example.json")) as f:
        ex = json.load(f)
    for r in ex["rows"]:
        x = np.asarray(r["x"], np.float16).view(np.uint16)[None]
        codes, slots = oracle.oaken_quantize_rows(x, r["s_in"], r["z_in"], r["s_out"],
                                                  r["outer_bits"])
        assert codes[0].tolist() == r["codes"], r
        assert slots[0].tolist() == [int(v, 16) for v in r["slots"]], r
        xh = oracle.oaken_dequantize_rows(codes, slots, x.shape[1], r["s_in"], r["z_in"],
                                          r["s_out"])
        assert xh[0].tolist() == r["x_hat"], r


def test_inner_codes_are_the_nearest_grid_point():
    """Brute force: an inner element's code is the c in [0, 15] whose grid
    value (c - z_in) * s_in is nearest to v, ties to the even integer
    c - z_in (round half to even of v / s_in)."""
    rng = np.random.default_rng(21)
    for s_in, z_in, s_out, b in _params():
        x16 = _rows(rng, s_in, z_in, n=60)
        codes, _ = oracle.oaken_quantize_rows(x16, s_in, z_in, s_out, b)
        c = _unpack4(codes)
        v = x16.view(np.float16).astype(np.float64)
        t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
        inner = (v >= t_lo) & (v <= t_hi)
        grid = (np.arange(16) - z_in) * s_in
        dist = np.abs(v[..., None] - grid)
        best = dist.min(-1, keepdims=True)
        cand = dist <= best * (1 + 1e-12) + 1e-300
        # among equidistant codes, the one with c - z_in even
        even = ((np.arange(16) - z_in) % 2 == 0)
        pick = np.where(cand.sum(-1) > 1, np.argmax(cand & even, -1), np.argmax(cand, -1))
        assert np.array_equal(c[inner], pick[inner])


def test_reduces_to_the_group_quantizer():
    """A row whose minimum is T_lo and maximum T_hi has the group quantizer's
    scale s_in and zero point z_in (R2-R5 with G = D, bits 4), and no
    outliers: its Oaken codes are that quantizer's codes."""
    rng = np.random.default_rng(22)
    for s_in, z_in, s_out, b in _params():
        t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
        x = rng.uniform(t_lo, t_hi, (50, 128))
        x[:, 3], x[:, 77] = t_lo, t_hi
        x16 = x.astype(np.float16).view(np.uint16)
        codes, slots = oracle.oaken_quantize_rows(x16, s_in, z_in, s_out, b)
        gc, gm = oracle.quantize_rows(x16, 128, 4)
        assert np.all(gm[:, 0, 0] == np.float16(s_in).view(np.uint16))
        assert np.all(gm[:, 0, 1].view(np.float16) == z_in)
        assert np.array_equal(codes, gc)
        assert np.all(slots == 0)


def test_half_step_bounds_and_slots():
    rng = np.random.default_rng(23)
    for s_in, z_in, s_out, b in _params():
        x16 = _rows(rng, s_in, z_in)
        codes, slots = oracle.oaken_quantize_rows(x16, s_in, z_in, s_out, b)
        xh = oracle.oaken_dequantize_rows(codes, slots, 128, s_in, z_in, s_out)
        v = x16.view(np.float16).astype(np.float64)
        c = _unpack4(codes)
        t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
        inner = (v >= t_lo) & (v <= t_hi)
        hi, lo = v > t_hi, v < t_lo
        err = np.abs(v - xh)
        assert np.all(err[inner] <= s_in / 2 * (1 + 2.0**-20))
        assert np.all(c[hi] == 15) and np.all(c[lo] == 0)
        m_max = 2**b - 1
        for r in range(v.shape[0]):
            dims = np.nonzero(hi[r] | lo[r])[0]
            kept = dims[:16]
            sl = slots[r]
            assert np.all(sl[len(kept):] == 0)
            assert np.array_equal(sl[:len(kept)] & 0xFF, kept)
            d = (sl[:len(kept)] >> 8).astype(np.uint8).view(np.int8).astype(np.int64)
            assert np.all(np.where(hi[r, kept], d >= 0, d <= 0))
            assert np.all(np.abs(d) <= m_max)
            # an outlier with a slot and an uncapped magnitude is within s_out / 2
            shift = np.where(hi[r, kept], v[r, kept] - t_hi, t_lo - v[r, kept])
            unc = shift / s_out < m_max - 0.5
            assert np.all(err[r, kept][unc] <= s_out / 2 * (1 + 2.0**-20) + 1e-12)
            # a capped one is below its true value's magnitude, never past it
            assert np.all(np.abs(xh[r, kept][~unc]) <= np.abs(v[r, kept][~unc]))
            # dropped outliers reconstruct to their threshold
            for j in dims[16:]:
                assert xh[r, j] == (t_hi if hi[r, j] else t_lo)


def test_dense_sparse_equals_the_page_dequantization():
    """x_hat of an outlier is T_hi + m * s_out (Delta > 0) or T_lo - m * s_out
    (Delta < 0): the page's T + Delta_hat, with the dense part supplying T."""
    rng = np.random.default_rng(24)
    s_in, z_in, s_out, b = 0.25, 5, 0.4, 6
    t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
    x = np.concatenate([rng.uniform(t_hi, t_hi + 20, (40, 8)),
                        rng.uniform(t_lo - 20, t_lo, (40, 8))], 1)
    x16 = x.astype(np.float16).view(np.uint16)
    codes, slots = oracle.oaken_quantize_rows(x16, s_in, z_in, s_out, b)
    xh = oracle.oaken_dequantize_rows(codes, slots, 16, s_in, z_in, s_out)
    m = (slots >> 8).astype(np.uint8).view(np.int8).astype(np.float64)
    assert np.array_equal(slots & 0xFF, np.tile(np.arange(16), (40, 1)))
    so = float(np.float32(s_out))  # the plane's parameters are fp32
    expect = np.where(np.arange(16) < 8, t_hi + m * so, t_lo + m * so)
    assert np.array_equal(xh, expect)


def test_bf16_worked_row():
    """bf16 input (reading R19) through the Oaken encoder: the hand-worked row
    of tests/golden/oaken_bf16_worked_example.json, with outliers beyond the
    fp16 range on both sides (capped magnitudes), values on the thresholds
    (inner), a zero-magnitude outlier and two halfway magnitudes."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                    "oaken_bf16_worked_example.json")))
    import torch
    vals = torch.tensor(g["values"], dtype=torch.float32)
    pat = np.array([int(h, 16) for h in g["bf16_patterns"]], np.uint16)
    assert np.array_equal(vals.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16), pat)
    codes, slots = oracle.oaken_quantize_rows(pat[None], g["s_in"], g["z_in"], g["s_out"],
                                              g["outer_bits"], in_dtype="bf16")
    assert [(int(codes[0, j // 2]) >> (4 * (j % 2))) & 15 for j in range(8)] == g["codes"]
    want = [int(h, 16) for h in g["slots"]]
    assert slots[0, :len(want)].tolist() == want
    assert not slots[0, len(want):].any()


def test_bf16_rows_of_fp16_values_match_the_fp16_path():
    """bf16 rows whose values are all fp16 values (outliers included) give
    exactly the fp16 path's codes and slots."""
    import torch
    gen = torch.Generator().manual_seed(31)
    x = torch.randn((48, 128), generator=gen) * 2
    x[:, 7] *= 40.0
    x[:, 90] *= -25.0
    x[3, :20] = torch.linspace(-60.0, 60.0, 20)
    xb = x.to(torch.bfloat16).float()
    assert torch.equal(xb.half().float(), xb)
    b16 = xb.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)
    f16 = xb.to(torch.float16).contiguous().view(torch.int16).numpy().view(np.uint16)
    for params in ((0.25, 8, 0.5, 5), (0.125, 3, 0.05, 7), (0.5, 0, 2.0, 6)):
        cb, sb = oracle.oaken_quantize_rows(b16, *params, in_dtype="bf16")
        cf, sf = oracle.oaken_quantize_rows(f16, *params)
        assert np.array_equal(cb, cf) and np.array_equal(sb, sf), params
