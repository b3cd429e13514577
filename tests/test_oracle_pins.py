"""Pins for the CPU oracle: every check here compares the oracle with
something other than itself -- hand-derived values from the pages' formulas
(tests/golden), library routines (numpy/torch fp16 rounding, torch
scaled-dot-product attention, scipy log-sum-exp), closed forms and brute
force on tiny inputs."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _f16(vals):
    return np.asarray(vals, np.float16).view(np.uint16)


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- fp16 codec

def test_f16_decode_exhaustive_matches_numpy():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_bits_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f16_roundtrip_exhaustive():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16).astype(np.float32)
    back = oracle.f32_to_f16_bits(f)
    ok = ~np.isnan(f)
    assert np.array_equal(back[ok], h[ok])


def test_f16_encode_matches_numpy_and_torch_rne():
    rng = np.random.default_rng(1)
    parts = [
        rng.standard_normal(400_000).astype(np.float32),
        (rng.standard_normal(200_000) * 3e4).astype(np.float32),           # near overflow
        (rng.standard_normal(200_000) * 1e-6).astype(np.float32),          # subnormal range
        rng.uniform(-70000, 70000, 100_000).astype(np.float32),
        rng.integers(0, 2**32, 300_000, dtype=np.uint64).astype(np.uint32).view(np.float32),
    ]
    # exact ties: midpoints between adjacent fp16 values (normal and subnormal)
    h = np.arange(0, 0x7bff, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    parts.append(mid[(mid.astype(np.float64) == (lo + hi) / 2)])
    x = np.concatenate(parts)
    x = x[np.isfinite(x)]
    ours = oracle.f32_to_f16_bits(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    t = torch.from_numpy(x[:200_000]).half().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours[:200_000], t)


def test_f16_round_up_is_smallest_not_below():
    rng = np.random.default_rng(2)
    x = np.abs(rng.standard_normal(20_000)).astype(np.float32) * 10 + 1e-5
    up = oracle.f32_to_f16_bits_up(x)
    v = up.view(np.float16).astype(np.float64)
    below = (up - 1).view(np.float16).astype(np.float64)
    assert np.all(v >= x.astype(np.float64))
    assert np.all(below < x.astype(np.float64))


# ---------------------------------------------------------------- quantization

def test_quant_worked_examples(golden_dir):
    ex = _load(golden_dir, "quant_worked_examples.json")
    for g in ex["groups"]:
        code, s16, z16 = oracle.quantize_group(_f16(g["x"]), g["bits"])
        assert list(code) == g["codes"], g["name"]
        assert s16 == int(g["s16"], 16), g["name"]
        assert z16 == int(g["z16"], 16), g["name"]


def _row_from_rule(name):
    j = np.arange(128)
    if "INT4" in name:
        return np.where(j < 64, j % 16, -((j - 64) % 16)).astype(np.float16)
    return (j % 4).astype(np.float16)


def test_quant_row_packing_examples(golden_dir):
    ex = _load(golden_dir, "quant_worked_examples.json")
    for r in ex["rows"]:
        x = _row_from_rule(r["name"]).view(np.uint16)[None]
        codes, meta = oracle.quantize_rows(x, r["group"], r["bits"])
        assert codes[0].tobytes().hex() == r["codes_hex"], r["name"]
        want = np.array([[int(a, 16), int(b, 16)] for a, b in r["meta"]], np.uint16)
        assert np.array_equal(meta[0], want), r["name"]


def _random_groups(rng, n, G):
    """Mixed group populations: N(0,1), channel outliers, all-positive,
    all-negative, tiny ranges, large magnitudes."""
    out = []
    for k in range(n):
        kind = k % 6
        if kind == 0:
            x = rng.standard_normal(G)
        elif kind == 1:
            x = rng.standard_normal(G)
            x[rng.integers(0, G, 2)] *= 20
        elif kind == 2:
            x = rng.uniform(1, 9, G)
        elif kind == 3:
            x = -rng.uniform(0.5, 3, G)
        elif kind == 4:
            x = 0.25 + rng.standard_normal(G) * 1e-3
        else:
            x = rng.standard_normal(G) * 3000
        out.append(x.astype(np.float16))
    return np.stack(out)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_quant_code_is_nearest_grid_point_bruteforce(bits, G):
    """Each code is the argmin over all codes c in [0, qmax] of
    |x/s - (c - z)| (exact rational arithmetic), ties to the even multiple."""
    rng = np.random.default_rng(bits * 1000 + G)
    qmax = (1 << bits) - 1
    groups = _random_groups(rng, 36, G)
    for x16 in groups:
        code, s16, z16 = oracle.quantize_group(x16.view(np.uint16), bits)
        s = Fraction(float(np.uint16(s16).view(np.float16)))
        z = Fraction(float(np.uint16(z16).view(np.float16)))
        for xv, c in zip(x16.astype(np.float64), code):
            t = Fraction(float(xv)) / s
            # skip elements whose exact quotient sits within an fp32 ulp of a
            # rounding boundary (the division is rounded before round())
            frac = t - math.floor(t)
            if abs(frac - Fraction(1, 2)) < abs(t) * Fraction(1, 2**22) + Fraction(1, 2**40):
                continue
            best = min(range(qmax + 1), key=lambda cc: (abs(t - (cc - z)), (cc - z) % 2))
            assert c == best


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_dequant_error_at_most_half_step(bits, G):
    """|x - x_hat| <= s/2 (up to the fp32 rounding of x/s) for every element
    of every group whose zero point is exact in fp16 (|z| <= 2048)."""
    rng = np.random.default_rng(7 + bits + G)
    groups = _random_groups(rng, 600, G)
    codes, meta = oracle.quantize_rows(groups.view(np.uint16), G, bits)
    xh = oracle.dequantize_rows(codes, meta, G, G, bits)
    s = meta[:, 0, 0].view(np.float16).astype(np.float64)
    z = meta[:, 0, 1].view(np.float16).astype(np.float64)
    x = groups.astype(np.float64)
    ok = np.abs(z) <= 2048
    assert ok.mean() > 0.8
    err = np.abs(x - xh)
    bound = s[:, None] / 2 + np.abs(x) * 2.0**-23 + s[:, None] * 2.0**-20
    assert np.all(err[ok] <= bound[ok])


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_codes_in_range_and_extremes(bits):
    rng = np.random.default_rng(11 + bits)
    G = 64
    qmax = (1 << bits) - 1
    groups = _random_groups(rng, 300, G)
    for x16 in groups[::5]:
        code, s16, z16 = oracle.quantize_group(x16.view(np.uint16), bits)
        assert code.max() <= qmax
        z = float(np.uint16(z16).view(np.float16))
        if abs(z) <= 2048:
            # min maps to 0 exactly; max maps to qmax or qmax - 1 (s rounded up)
            assert code[np.argmin(x16)] == 0
            assert code[np.argmax(x16)] in (qmax, qmax - 1)


def test_scale_matches_static_formula_and_codes_agree_within_one():
    """s equals (max - min)/(2^b - 1) (static-quantization page 2.1) up to the
    fp16 round-up, and codes agree within 1 with that page's
    round((x - min)/scale)."""
    rng = np.random.default_rng(5)
    for bits in (2, 4, 8):
        qmax = (1 << bits) - 1
        for x16 in _random_groups(rng, 60, 64)[::1]:
            code, s16, z16 = oracle.quantize_group(x16.view(np.uint16), bits)
            x = x16.astype(np.float64)
            s = float(np.uint16(s16).view(np.float16))
            s_ref = max((x.max() - x.min()) / qmax, 1e-5)
            assert s_ref <= s <= s_ref * (1 + 2.0**-10) + 2.0**-24
            if abs(float(np.uint16(z16).view(np.float16))) <= 2048:
                alt = np.clip(np.round((x - x.min()) / s), 0, qmax)
                assert np.max(np.abs(alt - code)) <= 1


def test_scale_floor_and_constant_groups():
    for v in (0.0, 1e-4, -0.5, 0.25):
        code, s16, z16 = oracle.quantize_group(_f16([v] * 32), 4)
        assert s16 == 0x00A8  # fp16(1e-5), rounded up
        assert len(set(code.tolist())) == 1


def test_groups_run_along_head_dim():
    """An outlier in one group changes that group's scale and no other."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 128)).astype(np.float16)
    _, m0 = oracle.quantize_rows(x.view(np.uint16), 64, 4)
    y = x.copy()
    y[2, 70] = 50
    _, m1 = oracle.quantize_rows(y.view(np.uint16), 64, 4)
    diff = np.argwhere(m0[..., 0] != m1[..., 0])
    assert diff.tolist() == [[2, 1]]


def test_bits16_rows_are_stored_raw():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 128)).astype(np.float16)
    codes, _ = oracle.quantize_rows(x.view(np.uint16), 128, 16)
    assert codes.tobytes() == x.tobytes()
    back = oracle.dequantize_rows(codes, None, 128, 128, 16)
    assert np.array_equal(back, x.astype(np.float64))


# ---------------------------------------------------------------- attention

def test_attention_two_token_hand_expansion(golden_dir):
    ex = _load(golden_dir, "attention_two_tokens.json")
    o, lse = oracle.attention(np.array(ex["q"]), np.array(ex["K"]), np.array(ex["V"]),
                              ex["scale"])
    np.testing.assert_allclose(o, ex["o"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, ex["lse"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("g,L,D", [(1, 1, 8), (1, 37, 16), (8, 100, 128), (4, 513, 64)])
def test_attention_matches_torch_sdpa(g, L, D):
    rng = np.random.default_rng(g * 7 + L)
    q = rng.standard_normal((g, D))
    K = rng.standard_normal((L, D)) * 2
    V = rng.standard_normal((L, D))
    scale = 1 / math.sqrt(D)
    o, lse = oracle.attention(q, K, V, scale)
    tq = torch.from_numpy(q)[None, :, None, :]           # [1, g, 1, D]
    tk = torch.from_numpy(K)[None, None].expand(1, g, L, D)
    tv = torch.from_numpy(V)[None, None].expand(1, g, L, D)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=0, atol=1e-12)
    from scipy.special import logsumexp
    np.testing.assert_allclose(lse, logsumexp(scale * q @ K.T, axis=1), rtol=1e-13)


def test_attention_closed_forms():
    rng = np.random.default_rng(9)
    D = 16
    q = rng.standard_normal((2, D))
    V = rng.standard_normal((5, D))
    # one token: output is that token's value, lse its score
    K1 = rng.standard_normal((1, D))
    o, lse = oracle.attention(q, K1, V[:1], 0.3)
    np.testing.assert_array_equal(o, np.repeat(V[:1], 2, 0))
    np.testing.assert_allclose(lse, 0.3 * q @ K1[0], rtol=1e-15)
    # identical keys: output is the mean of V
    K = np.repeat(K1, 5, 0)
    o, _ = oracle.attention(q, K, V, 0.3)
    np.testing.assert_allclose(o, np.repeat(V.mean(0, keepdims=True), 2, 0), atol=1e-14)
    # one key whose score is 60 above the rest dominates
    qd = np.zeros((1, D))
    qd[0, 0] = 1.0
    Kd = np.zeros((5, D))
    Kd[3, 0] = 60.0
    o, lse = oracle.attention(qd, Kd, V, 1.0)
    np.testing.assert_allclose(o[0], V[3], atol=1e-24 + 10 * math.exp(-60) * np.abs(V).max())
    # permuting tokens leaves the output unchanged
    K = rng.standard_normal((5, D))
    p = rng.permutation(5)
    o1, l1 = oracle.attention(q, K, V, 0.5)
    o2, l2 = oracle.attention(q, K[p], V[p], 0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)


def test_blockwise_merge_equals_direct():
    """Cocktail 3.2.3: attention computed per block and merged equals the
    unchunked computation, including empty blocks."""
    rng = np.random.default_rng(10)
    g, L, D = 8, 700, 128
    q = rng.standard_normal((g, D))
    K = rng.standard_normal((L, D)) * 3
    V = rng.standard_normal((L, D))
    o, lse = oracle.attention(q, K, V, 0.1)
    for bounds in ([0, L], [0, 1, L], [0, 100, 100, 333, 690, L], list(range(0, L + 1, 32)) + [L]):
        bounds = sorted(set(bounds)) if bounds[-1] != L else bounds
        bounds = list(dict.fromkeys(bounds))
        ob, lb = oracle.attention_blocks(q, K, V, 0.1, bounds)
        np.testing.assert_allclose(ob, o, atol=1e-12)
        np.testing.assert_allclose(lb, lse, atol=1e-12)


def test_packed_attention_equals_dequantize_then_attend():
    rng = np.random.default_rng(12)
    L, D, G = 300, 128, 64
    x = (rng.standard_normal((2, L, D)) * 2).astype(np.float16)
    kc, km = oracle.quantize_rows(x[0].view(np.uint16), G, 4)
    vc, vm = oracle.quantize_rows(x[1].view(np.uint16), G, 8)
    q16 = rng.standard_normal((4, D)).astype(np.float16).view(np.uint16)
    o1, l1 = oracle.attention_packed(q16, False, kc, km, 4, vc, vm, 8, G, L, 0.0883)
    K = oracle.dequantize_rows(kc, km, D, G, 4)
    V = oracle.dequantize_rows(vc, vm, D, G, 8)
    qd = q16.view(np.float16).astype(np.float64)
    o2, l2 = oracle.attention(qd, K, V, 0.0883)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


# ---------------------------------------------------------------- Cocktail search

def test_chunk_threshold_toy(golden_dir):
    ex = _load(golden_dir, "chunk_threshold_toy.json")
    sim, bits = oracle.chunk_assign(np.array(ex["chunks"], np.float32),
                                    np.array(ex["query"], np.float32), ex["alpha"], ex["beta"])
    assert sim.tolist() == ex["sims"]
    assert bits.tolist() == ex["classes"]
    perm, counts = oracle.chunk_partition(bits)
    assert perm.tolist() == ex["perm"]
    assert counts.tolist() == ex["counts"]


def test_chunk_similarity_matches_numpy_and_partition_is_stable():
    rng = np.random.default_rng(13)
    emb = rng.standard_normal((1024, 768)).astype(np.float32)
    qe = emb[rng.choice(1024, 20, replace=False)].mean(0) + 0.1 * rng.standard_normal(768)
    qe = qe.astype(np.float32)
    sim, bits = oracle.chunk_assign(emb, qe, 0.6, 0.1)
    e64, q64 = emb.astype(np.float64), qe.astype(np.float64)
    ref = e64 @ q64 / (np.linalg.norm(e64, axis=1) * np.linalg.norm(q64))
    np.testing.assert_allclose(sim, ref, rtol=1e-12, atol=1e-15)
    lo = sim.min() + (sim.max() - sim.min()) * 0.6
    hi = sim.max() - (sim.max() - sim.min()) * 0.1
    want = np.where(sim > hi, 16, np.where(sim > lo, 4, 2))
    assert np.array_equal(bits, want)
    perm, counts = oracle.chunk_partition(bits)
    assert sorted(perm.tolist()) == list(range(1024))
    rank = {16: 0, 4: 1, 2: 2}
    keys = [(rank[int(bits[i])], int(i)) for i in perm]
    assert keys == sorted(keys)
    assert counts.tolist() == [int((bits == 16).sum()), int((bits == 4).sum()),
                               int((bits == 2).sum())]


# ---------------------------------------------------------------- KV size

def test_kv_size_worked_example(golden_dir):
    ex = _load(golden_dir, "kv_size_worked_example.json")
    n = oracle.kv_elements(ex["layers"], ex["kv_heads"], ex["head_dim"], ex["seq_len"],
                           ex["batch"])
    assert n == ex["elements"]
    assert abs(n / ex["page_elements_approx"] - 1) < 0.01
    assert n * 2 == ex["fp16_bytes"]
    assert abs(n * 2 / 1e9 - ex["page_bytes_approx_gb"]) < 1.0
