"""Mutation check of the oracle's pins.

Each case plants one plausible mistake in a temporary copy of the oracle's C
source (never in the oracle itself), rebuilds the copy, and asserts that at
least one pin -- a hand-derived fixture, a library routine or a closed form
-- now fails.  A mutant that survives would mean the pins cannot tell that
mistake from the real thing."""
import importlib.util
import json
import math
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
GOLDEN = os.path.join(ROOT, "tests", "golden")

# (name, original text, mutated text)
MUTANTS = [
    ("bf16 read as fp16", "return in_bf16 ? kvqo_bf16_to_f32(x[j]) : kvqo_f16_to_f32(x[j]);",
     "return kvqo_f16_to_f32(x[j]);"),
    ("round half away from zero", "float c = rintf(kvqo_in(x, j, in_bf16) / s) + z;",
     "float c = roundf(kvqo_in(x, j, in_bf16) / s) + z;"),
    ("scale rounded to nearest", "uint16_t s16 = kvqo_f32_to_f16_up(s32);",
     "uint16_t s16 = kvqo_f32_to_f16(s32);"),
    ("zero point clamped to code range", "    uint16_t z16 = kvqo_f32_to_f16(zf);",
     "    if (zf < 0.0f) zf = 0.0f; if (zf > qmax) zf = qmax;\n    uint16_t z16 = kvqo_f32_to_f16(zf);"),
    ("no scale floor", "    if (s32 < 1e-5f)\n        s32 = 1e-5f;", ""),
    ("zero point sign flipped", "float zf = rintf(-mn / s) + 0.0f;", "float zf = rintf(mn / s) + 0.0f;"),
    ("negative zero kept", "float zf = rintf(-mn / s) + 0.0f;", "float zf = rintf(-mn / s);"),
    ("2^bits levels", "const float qmax = (float)((1 << bits) - 1);",
     "const float qmax = (float)(1 << bits);"),
    ("high nibble first", "cr[bitpos / 8] |= (uint8_t)(tmp[j] << (bitpos % 8));",
     "cr[bitpos / 8] |= (uint8_t)(tmp[j] << (8 - bits - bitpos % 8));"),
    ("dequant adds zero point", "out[r * D + e] = (c - z) * s;", "out[r * D + e] = (c + z) * s;"),
    ("score not scaled", "score[t] = scale * acc;", "score[t] = acc;"),
    ("lse in log2", "lse[h] = m + log(l);\n    }\n    free(score);",
     "lse[h] = m + log2(l);\n    }\n    free(score);"),
    ("merge drops block weights", "l += w * lb[b];", "l += lb[b];"),
    ("FP16 threshold inclusive", "if (sim[i] > t_high)", "if (sim[i] >= t_high)"),
    ("query norm missing", "sim[i] = dot / (nq * sqrt(cc));", "sim[i] = dot / sqrt(cc);"),
    ("INT2 before INT4", "static const uint8_t order[3] = {16, 4, 2};",
     "static const uint8_t order[3] = {16, 2, 4};"),
    ("f16 rounding truncates", "if (rest > 0x1000u || (rest == 0x1000u && (h & 1u)))",
     "if (rest > 0x1000u)"),
    ("e4m3 ties away from zero", "double r = rint(a / quantum) * quantum;",
     "double r = round(a / quantum) * quantum;"),
    ("e4m3 without subnormal spacing", "double quantum = ldexp(1.0, (e < -6 ? -6 : e) - 3);",
     "double quantum = ldexp(1.0, e - 3);"),
    ("e4m3 exponent bias 8", "v = ldexp((double)(8 + m), e - 10);",
     "v = ldexp((double)(8 + m), e - 11);"),
    ("fp8 scale from another maximum", "float s32 = amax / 448.0f;", "float s32 = amax / 464.0f;"),
    ("sym8 ties away from zero", "float c = rintf(kvqo_in(x, j, in_bf16) / s);",
     "float c = roundf(kvqo_in(x, j, in_bf16) / s);"),
    ("sym8 scale over 128 levels", "float s32 = amax / 127.0f;", "float s32 = amax / 128.0f;"),
    ("sym8 offset-binary codes", "code[j] = (uint8_t)(int8_t)c;",
     "code[j] = (uint8_t)(int)(c + 128.0f);"),
    ("sym8 dequant unsigned", ": (fmt == 3) ? kvqo_e5m2_to_f64(c) : (double)(int8_t)c;",
     ": (fmt == 3) ? kvqo_e5m2_to_f64(c) : (double)c;"),
    ("per-channel block read transposed", "col[t] = x[(int64_t)t * D + d];",
     "col[t] = x[(int64_t)d * T + t];"),
    ("per-channel codes at the token offset", "codes[t * row_bytes + bitpos / 8] |= (uint8_t)(tmp[t] << (bitpos % 8));",
     "codes[d * (row_bytes / 4) + (t * bits) / 8] |= (uint8_t)(tmp[t] << ((t * bits) % 8));"),
    ("per-channel dequant ignores the zero point", "out[(int64_t)t * D + d] = (c - z) * s;",
     "out[(int64_t)t * D + d] = c * s;"),
    ("e5m2 ties away from zero", "double quantum = ldexp(1.0, (e < -14 ? -14 : e) - 2);\n    double r = rint(a / quantum) * quantum;",
     "double quantum = ldexp(1.0, (e < -14 ? -14 : e) - 2);\n    double r = round(a / quantum) * quantum;"),
    ("e5m2 exponent bias 16", "v = ldexp((double)(4 + m), e - 17);", "v = ldexp((double)(4 + m), e - 18);"),
    ("e5m2 scale from the E4M3 maximum", "float s32 = amax / 57344.0f;", "float s32 = amax / 448.0f;"),
    ("oaken high side shifted by the low threshold", "const float delta = v - t_hi;",
     "const float delta = v - t_lo;"),
    ("oaken outer ties away from zero", "float m = rintf(delta / s_out);", "float m = roundf(delta / s_out);"),
    ("oaken inner zero point dropped", "float cf = rintf(v / s_in) + z;", "float cf = rintf(v / s_in);"),
    ("oaken upper threshold one step high", "const float t_hi = (15.0f - z) * s_in;",
     "const float t_hi = (16.0f - z) * s_in;"),
    ("oaken outer magnitude one bit short", "const float m_max = (float)((1 << outer_bits) - 1);",
     "const float m_max = (float)((1 << (outer_bits - 1)) - 1);"),
]


def _build_mutant(tmp_path, orig, new):
    src = open(os.path.join(ORACLE_DIR, "kvq_oracle.c")).read()
    assert orig in src, orig
    d = tmp_path / "oracle_mutant"
    d.mkdir()
    (d / "kvq_oracle.c").write_text(src.replace(orig, new, 1))
    shutil.copy(os.path.join(ORACLE_DIR, "__init__.py"), d / "__init__.py")
    spec = importlib.util.spec_from_file_location("oracle_mutant_" + str(abs(hash(new))),
                                                  str(d / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _pins(o):
    """Yield (pin name, passed) for a compact set of the oracle's pins."""
    ex = _golden("quant_worked_examples.json")
    ok = True
    for g in ex["groups"]:
        with np.errstate(all="ignore"):
            code, s16, z16 = o.quantize_group(np.asarray(g["x"], np.float16).view(np.uint16),
                                              g["bits"])
        ok &= (list(code) == g["codes"] and s16 == int(g["s16"], 16)
               and z16 == int(g["z16"], 16))
    yield "quant worked examples", ok

    j = np.arange(128)
    x = np.where(j < 64, j % 16, -((j - 64) % 16)).astype(np.float16).view(np.uint16)[None]
    codes, _ = o.quantize_rows(x, 64, 4)
    yield "packing example", codes[0].tobytes().hex() == ex["rows"][0]["codes_hex"]

    rng = np.random.default_rng(0)
    G, bits = 64, 4
    xs = np.concatenate([rng.standard_normal((200, G)), rng.uniform(1, 9, (200, G))]).astype(np.float16)
    with np.errstate(all="ignore"):
        c, m = o.quantize_rows(xs.view(np.uint16), G, bits)
        xh = o.dequantize_rows(c, m, G, G, bits)
    s = m[:, 0, 0].view(np.float16).astype(np.float64)
    err = np.abs(xs.astype(np.float64) - xh)
    yield "half-step bound", bool(np.all(err <= s[:, None] / 2 * (1 + 2.0**-12) + 1e-12))

    h = np.arange(0, 0x7c00, dtype=np.uint32).astype(np.uint16)
    lo = h[:-1].view(np.float16).astype(np.float64)
    hi = h[1:].view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    yield "fp16 ties vs numpy", bool(np.array_equal(o.f32_to_f16_bits(mid),
                                                    mid.astype(np.float16).view(np.uint16)))

    a = _golden("attention_two_tokens.json")
    oo, ll = o.attention(np.array(a["q"]), np.array(a["K"]), np.array(a["V"]), a["scale"])
    yield "two-token expansion", bool(np.allclose(oo, a["o"], atol=1e-14)
                                      and np.allclose(ll, a["lse"], atol=1e-14))

    q = rng.standard_normal((4, 32))
    K = rng.standard_normal((50, 32))
    V = rng.standard_normal((50, 32))
    oo, ll = o.attention(q, K, V, 0.2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None], torch.from_numpy(K)[None, None].expand(1, 4, 50, 32),
        torch.from_numpy(V)[None, None].expand(1, 4, 50, 32), scale=0.2)[0, :, 0].numpy()
    lref = np.log(np.exp(0.2 * q @ K.T).sum(1))
    yield "torch sdpa", bool(np.allclose(oo, ref, atol=1e-12) and np.allclose(ll, lref, atol=1e-12))
    ob, lb = o.attention_blocks(q, K * 3, V, 0.2, [0, 7, 7, 30, 50])
    od, ld = o.attention(q, K * 3, V, 0.2)
    yield "blocks equal direct", bool(np.allclose(ob, od, atol=1e-12) and np.allclose(lb, ld, atol=1e-12))

    f8 = _golden("fp8_worked_example.json")
    ok = True
    for g in f8["groups"]:
        code, s16 = o.quantize_group_fp8(np.asarray(g["x"], np.float16).view(np.uint16))
        ok &= code.tolist() == g["codes"] and s16 == int(g["s16"], 16)
    yield "fp8 worked groups", bool(ok)
    codes = np.arange(256, dtype=np.uint8)
    v8 = o.e4m3_to_f64(codes)
    t8 = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    yield "e4m3 decode vs torch", bool(np.all((v8 == t8) | (np.isnan(v8) & np.isnan(t8))))
    fin = np.unique(t8[~np.isnan(t8)])
    mids = np.concatenate([(fin[:-1] + fin[1:]) / 2, rng.standard_normal(2000) * 30]).astype(np.float32)
    mids = np.clip(mids, -448, 448)
    yield "e4m3 encode vs torch", bool(np.array_equal(
        o.f32_to_e4m3(mids), torch.from_numpy(mids).to(torch.float8_e4m3fn).view(torch.uint8).numpy()))

    s8 = _golden("sym8_worked_example.json")
    ok = True
    for g in s8["groups"]:
        code, s16 = o.quantize_group_sym8(np.asarray(g["x"], np.float16).view(np.uint16))
        ok &= code.tolist() == g["codes"] and s16 == int(g["s16"], 16)
    yield "sym8 worked groups", bool(ok)
    c8 = np.array([[0, 1, 127, 128, 255]], np.uint8)
    m8 = np.array([[[np.float16(0.5).view(np.uint16), 0]]], np.uint16)
    yield "sym8 dequant", o.dequantize_rows(c8, m8, 5, 5, 8, "sym8").tolist() == [
        [0.0, 0.5, 63.5, -64.0, -0.5]]

    rng_k = np.random.default_rng(5)
    xk = (rng_k.standard_normal((32, 128)) * 3).astype(np.float16)
    xk[:, 5] = np.linspace(-40, 90, 32)
    ck, mk = o.quantize_block_channels(xk.view(np.uint16), 4)
    ctr, mtr = o.quantize_rows(np.ascontiguousarray(xk.T).view(np.uint16), 32, 4)
    jj = np.arange(128)
    un = (ck[:, jj // 2].astype(np.int64) >> ((jj % 2) * 4)) & 15
    jt = np.arange(32)
    unt = (ctr[:, jt // 2].astype(np.int64) >> ((jt % 2) * 4)) & 15
    yield "per-channel = transposed per-token", bool(np.array_equal(mk, mtr[:, 0, :])
                                                      and np.array_equal(un, unt.T))
    xh = o.dequantize_block_channels(ck, mk, 128, 4)
    sk = mk[:, 0].view(np.float16).astype(np.float64)
    yield "per-channel half-step bound", bool(np.all(np.abs(xk.astype(np.float64) - xh)
                                                     <= sk[None, :] / 2 * (1 + 2.0**-12)))

    e5 = _golden("e5m2_worked_example.json")
    ok = True
    for g in e5["groups"]:
        code, s16 = o.quantize_group_e5m2(np.asarray(g["x"], np.float16).view(np.uint16))
        ok &= code.tolist() == g["codes"] and s16 == int(g["s16"], 16)
    yield "e5m2 worked group", bool(ok)
    c5 = np.arange(256, dtype=np.uint8)
    v5 = o.e5m2_to_f64(c5)
    t5 = torch.from_numpy(c5).view(torch.float8_e5m2).float().numpy().astype(np.float64)
    yield "e5m2 decode vs torch", bool(np.all((v5 == t5) | (np.isnan(v5) & np.isnan(t5))))
    f5 = np.unique(t5[np.isfinite(t5)])
    m5 = np.clip((f5[:-1] + f5[1:]) / 2, -57344, 57344).astype(np.float32)
    yield "e5m2 encode vs torch", bool(np.array_equal(
        o.f32_to_e5m2(m5), torch.from_numpy(m5).to(torch.float8_e5m2).view(torch.uint8).numpy()))

    b = _golden("bf16_worked_example.json")
    pat = np.array([int(h, 16) for h in b["bf16_patterns"]], np.uint16)[None]
    cb, mb = o.quantize_rows(pat, b["group"], b["bits"], in_dtype="bf16")
    ub = [(int(cb[0, j // 2]) >> (4 * (j % 2))) & 15 for j in range(b["group"])]
    yield "bf16 worked group", (ub == b["codes"] and int(mb[0, 0, 0]) == int(b["scale_f16"], 16)
                                and int(mb[0, 0, 1]) == int(b["zero_f16"], 16))

    ok = True
    for r in _golden("oaken_worked_example.json")["rows"]:
        x = np.asarray(r["x"], np.float16).view(np.uint16)[None]
        c, sl = o.oaken_quantize_rows(x, r["s_in"], r["z_in"], r["s_out"], r["outer_bits"])
        xh = o.oaken_dequantize_rows(c, sl, x.shape[1], r["s_in"], r["z_in"], r["s_out"])
        ok &= (c[0].tolist() == r["codes"] and sl[0].tolist() == [int(v, 16) for v in r["slots"]]
               and xh[0].tolist() == r["x_hat"])
    yield "oaken worked rows", bool(ok)

    t = _golden("chunk_threshold_toy.json")
    sim, cls = o.chunk_assign(np.array(t["chunks"], np.float32), np.array(t["query"], np.float32),
                              t["alpha"], t["beta"])
    perm, _ = o.chunk_partition(cls)
    yield "threshold toy", (sim.tolist() == t["sims"] and cls.tolist() == t["classes"]
                            and perm.tolist() == t["perm"])

    emb = rng.standard_normal((64, 24)).astype(np.float32)
    qe = (3 * rng.standard_normal(24)).astype(np.float32)
    sim, _ = o.chunk_assign(emb, qe, 0.6, 0.1)
    e64, q64 = emb.astype(np.float64), qe.astype(np.float64)
    ref = e64 @ q64 / (np.linalg.norm(e64, axis=1) * np.linalg.norm(q64))
    yield "cosine vs numpy", bool(np.allclose(sim, ref, rtol=1e-12, atol=1e-15))


def test_real_oracle_passes_compact_pins():
    import oracle
    failed = [name for name, ok in _pins(oracle) if not ok]
    assert failed == []


@pytest.mark.parametrize("name,orig,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, orig, new):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    mod = _build_mutant(tmp_path, orig, new)
    results = dict(_pins(mod))
    assert not all(results.values()), f"mutant '{name}' passed every pin: {results}"
