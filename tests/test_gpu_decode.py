"""GPU parity of kvq_decode_attention against the fp64 oracle on the same
seeded fp16 inputs: max-abs <= 2e-3 and relative L2 <= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_close, f16_bits, fill_cache, fill_fp16_segment, oracle_segment, q_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def _poison(c):
    c.k_codes.fill_(0x77)
    c.v_codes.fill_(0x88)
    if c.k_meta is not None:
        c.k_meta.view(torch.int16).fill_(-1)  # NaN patterns in unused slots
        c.v_meta.view(torch.int16).fill_(-1)


def _run(kvq, segs, q, max_len_hint=0):
    B, Hq, D = q.shape
    out = torch.full((B, Hq, D), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    ws = kvq.alloc_workspace(segs, Hq, max_len_hint, device=DEV)
    kvq.kvq_decode_attention(segs, q, out, lse, ws, max_len_hint=max_len_hint)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws) == 0
    return out, lse


def _case(kvq, wl, lens, max_tokens, max_len_hint=0, T=None):
    B = len(lens)
    T = T or max(lens)
    k, v = workloads.kv_tokens(wl, T, DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    c = kvq.QuantizedKVCache.allocate(B, wl.kv_heads, 128, max_tokens, wl.bits, wl.group, DEV)
    _poison(c)
    fill_cache(kvq, c, k, v, lens)
    out, lse = _run(kvq, c, q, max_len_hint)
    seg = oracle_segment(k, v, wl.bits, wl.group)
    ref, lref = oracle.decode_attention(q_bits(q), q.dtype == torch.bfloat16, [seg], [lens],
                                        128 ** -0.5)
    return out, lse, ref, lref


BASES = {
    "int4_g64_gqa8": workloads.WORKLOADS["llama3_8b_gqa_int4"],
    "int8_g128_mha_bf16": workloads.WORKLOADS["llama2_7b_mha_int8"],
    "int4_g64_mha_tiny": workloads.WORKLOADS["tiny"],
    "int4_g64_long": workloads.WORKLOADS["long_gqa_int4"],
}


@pytest.mark.parametrize("name", list(BASES))
def test_workload_shapes_small(kvq, name):
    base = BASES[name]
    g = base.group_ratio
    wl = base.scaled(kv_heads=2, q_heads=2 * g)
    lens = [37, 300, 16]
    out, lse, ref, lref = _case(kvq, wl, lens, 320)
    assert_close(out, ref, lse, lref, what=name)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128])
@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_bits_groups_ratios(kvq, bits, G, g):
    if (128 // G) * g > 16:
        pytest.skip("unsupported combination (more than 16 group x head rows)")
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=2, q_heads=2 * g, bits=bits,
                                                     group=G)
    lens = [129, 250]
    out, lse, ref, lref = _case(kvq, wl, lens, 256)
    assert_close(out, ref, lse, lref, what=f"bits{bits} G{G} g{g}")


@pytest.mark.parametrize("hint", [0, 64, 100000])
def test_split_counts_do_not_change_results(kvq, hint):
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(kv_heads=1, q_heads=8)
    lens = [1000, 777]
    out, lse, ref, lref = _case(kvq, wl, lens, 1024, max_len_hint=hint)
    assert_close(out, ref, lse, lref, what=f"hint {hint}")


@pytest.mark.parametrize("B,H,L", [(2, 2, 5000), (1, 1, 65536)])
def test_many_partials_and_the_two_call_form(kvq, B, H, L):
    """Plans of 40 and of 410 partials per query head (one sequence and one
    KV head over 65536 tokens: the merge kernel's largest thread groups),
    through the one-call attention and the two-call form (kvq_decode_partials
    + kvq_decode_merge), against the oracle."""
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=4 * H)
    lens = [L] + [L - 777] * (B - 1)
    out, lse, ref, lref = _case(kvq, wl, lens, workloads.round_up(L, 64))
    assert_close(out, ref, lse, lref, what=f"attention B{B} H{H} L{L}")
    k, v = workloads.kv_tokens(wl, L, DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    c = kvq.QuantizedKVCache.allocate(B, H, 128, workloads.round_up(L, 64), 4, 64, DEV)
    fill_cache(kvq, c, k, v, lens)
    ws = kvq.alloc_workspace(c, 4 * H, 0, device=DEV)
    o2 = torch.full((B, 4 * H, 128), float("nan"), device=DEV)
    l2 = torch.full((B, 4 * H), float("nan"), device=DEV)
    kvq.kvq_decode_partials(c, q, o2, l2, ws)
    kvq.kvq_decode_merge(c, q, o2, l2, ws)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws) == 0
    assert_close(o2, ref, l2, lref, what=f"two-call B{B} H{H} L{L}")


def test_edge_lengths(kvq):
    """Empty sequence (out 0, lse -inf), one token, exact tile multiples, the
    full capacity, and a tail of one token past a tile."""
    wl = workloads.WORKLOADS["tiny"].scaled(kv_heads=2, q_heads=4)
    lens = [0, 1, 16, 64, 17, 128]
    out, lse, ref, lref = _case(kvq, wl, lens, 128)
    o = out.cpu().numpy()
    assert np.all(o[0] == 0.0)
    assert np.all(np.isneginf(lse.cpu().numpy()[0]))
    mask = np.ones(len(lens), bool)
    mask[0] = False
    assert_close(out, ref, lse, lref, mask=mask, what="edge lengths")
    # one token: the output is that token's dequantized value
    seg = oracle_segment(*workloads.kv_tokens(wl, 128, DEV, batch=len(lens)), wl.bits, wl.group)
    v1 = oracle.dequantize_rows(seg["v_codes"][1, 0, :1], seg["v_meta"][1, 0, :1], 128, 64, 4)
    np.testing.assert_allclose(o[1, 0], v1[0], atol=1e-5)


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_fp16_segment(kvq, g):
    """Raw fp16 rows (Cocktail's FP16 class), ragged lengths, NaN bytes past
    the valid length, one to eight query heads per KV head."""
    wl = workloads.WORKLOADS["cocktail_mixed"].scaled(kv_heads=3, q_heads=3 * g)
    lens = [45, 100]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, 100, DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    c = kvq.QuantizedKVCache.allocate(B, 3, 128, 128, 16, 128, DEV)
    c.k_codes.fill_(0xFF)
    c.v_codes.fill_(0xFF)  # NaN fp16 everywhere first
    fill_fp16_segment(c, k, v, lens)
    c.k_codes[0, :, 45:].fill_(0xFF)
    c.v_codes[0, :, 45:].fill_(0xFF)
    out, lse = _run(kvq, c, q)
    seg = oracle_segment(k, v, 16, 128)
    ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [lens], 128 ** -0.5)
    assert_close(out, ref, lse, lref, what=f"fp16 segment g{g}")


@pytest.mark.parametrize("bits,G,g", [(2, 32, 1), (2, 32, 2), (4, 64, 4), (8, 128, 8),
                                      (2, 64, 8), (4, 32, 4)])
def test_large_magnitude_values(kvq, bits, G, g):
    """V entries in the tens of thousands (INT2 scales near 3 * 10^4): the
    weights p * s_V fed to the fp16 tensor-core operand must stay finite.
    Compared after dividing by the magnitude, so the tolerance applies to the
    N(0, 1)-sized values."""
    mag = 500.0  # the x20 outlier channels reach ~45000, inside fp16 range
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=2, q_heads=2 * g, bits=bits,
                                                     group=G)
    lens = [200, 97]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, 200, DEV, batch=B)
    v = (v.float() * mag).half()
    assert torch.isfinite(v).all() and v.abs().max() > 2.0e4
    q = workloads.queries(wl, DEV, batch=B)
    c = kvq.QuantizedKVCache.allocate(B, 2, 128, 256, bits, G, DEV)
    _poison(c)
    fill_cache(kvq, c, k, v, lens)
    out, lse = _run(kvq, c, q)
    seg = oracle_segment(k, v, bits, G)
    ref, lref = oracle.decode_attention(q_bits(q), q.dtype == torch.bfloat16, [seg], [lens],
                                        128 ** -0.5)
    assert_close(out / mag, ref / mag, lse, lref, what=f"large values bits{bits} G{G} g{g}")


@pytest.mark.parametrize("bits,G,g", [(4, 128, 1), (4, 128, 2), (8, 128, 8), (4, 64, 4),
                                      (2, 32, 2), (2, 64, 8)])
def test_rising_scores_rescale(kvq, bits, G, g):
    """Keys whose magnitude grows along the sequence make every head's running
    max rise stage after stage, at different stages for different heads, so
    the accumulators are rescaled many times."""
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=2, q_heads=2 * g, bits=bits,
                                                     group=G)
    lens = [600, 333]
    B = len(lens)
    T = max(lens)
    k, v = workloads.kv_tokens(wl, T, DEV, batch=B)
    ramp = torch.linspace(0.2, 3.0, T, device=DEV).view(1, 1, T, 1)
    k = (k.float() * ramp).half()
    q = workloads.queries(wl, DEV, batch=B)
    c = kvq.QuantizedKVCache.allocate(B, 2, 128, 640, bits, G, DEV)
    _poison(c)
    fill_cache(kvq, c, k, v, lens)
    out, lse = _run(kvq, c, q, max_len_hint=64)  # one split: one long running max
    seg = oracle_segment(k, v, bits, G)
    ref, lref = oracle.decode_attention(q_bits(q), q.dtype == torch.bfloat16, [seg], [lens],
                                        128 ** -0.5)
    assert_close(out, ref, lse, lref, what=f"rising scores bits{bits} G{G} g{g}")


@pytest.mark.parametrize("bits,G,g", [(8, 128, 1), (4, 64, 4), (2, 32, 1), (4, 128, 8),
                                      (2, 64, 2), (4, 32, 4), (16, 128, 4)])
def test_dominant_token_precision(kvq, bits, G, g):
    """One token whose key is a large multiple of every query gets all the
    weight: the output must equal that token's dequantized V to ~1e-6
    relative.  The weights p * s_V enter the tensor cores as two fp16 parts;
    rounding them to one fp16 value would show here as errors near 2^-12."""
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(kv_heads=2, q_heads=2 * g, bits=bits,
                                                     group=G)
    lens = [150, 61]
    B, T = len(lens), max(lens)
    k, v = workloads.kv_tokens(wl, T, DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    star = [97, 13]
    qh = q.view(B, 2, g, 128).float().sum(2)  # per KV head: the sum of its queries
    for bi, ts in enumerate(star):
        kk = qh[bi] / qh[bi].norm(dim=-1, keepdim=True) * 60.0
        k[bi, :, ts] = kk.half()
    v = (v.float() * 4.0).half()
    c = kvq.QuantizedKVCache.allocate(B, 2, 128, 192, bits, G, DEV)
    _poison(c)
    if bits == 16:
        fill_fp16_segment(c, k, v, lens)
    else:
        fill_cache(kvq, c, k, v, lens)
    out, _ = _run(kvq, c, q)
    seg = oracle_segment(k, v, bits, G)
    ref, _ = oracle.decode_attention(q_bits(q), q.dtype == torch.bfloat16, [seg], [lens],
                                     128 ** -0.5)
    o = out.cpu().numpy().astype(np.float64)
    scale = np.abs(ref).max()
    err = np.abs(o - ref).max() / scale
    assert err < 2e-5, f"bits{bits} G{G} g{g}: max error {err:.2e} of max |out|"


def test_mixed_segments_equal_unchunked(kvq):
    """Three segments (FP16, INT4, INT2) of one sequence merged by log-sum-exp
    equal attention over all their tokens (Cocktail page 3.2.3)."""
    B, H = 2, 3
    wl = workloads.WORKLOADS["cocktail_mixed"].scaled(kv_heads=H, q_heads=H)
    q = workloads.queries(wl, DEV, batch=B)
    lens = [[32, 64], [96, 0], [500, 320]]
    segs, osegs = [], []
    for i, (bits, G) in enumerate(((16, 128), (4, 32), (2, 32))):
        k, v = workloads.kv_tokens(wl, max(lens[i]), DEV, stream_extra=10 + i, batch=B)
        c = kvq.QuantizedKVCache.allocate(B, H, 128, 512, bits, G, DEV)
        _poison(c)
        if bits == 16:
            fill_fp16_segment(c, k, v, lens[i])
        else:
            fill_cache(kvq, c, k, v, lens[i])
        segs.append(c)
        osegs.append(oracle_segment(k, v, bits, G))
    out, lse = _run(kvq, segs, q)
    ref, lref = oracle.decode_attention(q_bits(q), False, osegs, lens, 128 ** -0.5)
    assert_close(out, ref, lse, lref, what="mixed segments")


def test_decode_steps_with_append(kvq):
    """Append one token per sequence, attend, repeat (the decode loop)."""
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=2, kv_heads=2, q_heads=16)
    B, ctx = 2, 200
    k, v = workloads.kv_tokens(wl, ctx, DEV)
    c = kvq.QuantizedKVCache.allocate(B, 2, 128, 256, 4, 64, DEV)
    _poison(c)
    fill_cache(kvq, c, k, v, [ctx, ctx])
    ks, vs = [k], [v]
    for step in range(5):
        kn, vn = workloads.kv_tokens(wl, 1, DEV, stream_extra=1 + step)
        kvq.kvq_quantize_append(c, kn, vn, 1, advance_seq_lens=True)
        ks.append(kn)
        vs.append(vn)
        q = workloads.queries(wl, DEV, step=step)
        out, lse = _run(kvq, c, q)
        seg = oracle_segment(torch.cat(ks, 2), torch.cat(vs, 2), 4, 64)
        n = ctx + step + 1
        ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [[n, n]], 128 ** -0.5)
        assert_close(out, ref, lse, lref, what=f"step {step}")
    assert c.seq_lens.tolist() == [ctx + 5] * 2


def _full_size(kvq, name, pairs, steps=1):
    """Full-size workload in the benchmark's launch configuration, the oracle
    evaluated on sampled (sequence, KV head) pairs."""
    wl = workloads.WORKLOADS[name]
    B, H, L = wl.batch, wl.kv_heads, wl.context
    max_tokens = workloads.round_up(L + 64, 64)
    k, v = workloads.kv_tokens(wl, L, DEV)
    c = kvq.QuantizedKVCache.allocate(B, H, 128, max_tokens, wl.bits, wl.group, DEV)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, L, advance_seq_lens=True)
    kn, vn = workloads.kv_tokens(wl, 1, DEV, stream_extra=1)
    kvq.kvq_quantize_append(c, kn, vn, 1, advance_seq_lens=True)
    q = workloads.queries(wl, DEV)
    out, lse = _run(kvq, c, q, max_len_hint=L + 1)
    g = wl.group_ratio
    ref = np.full((B, wl.q_heads, 128), np.nan)
    lref = np.full((B, wl.q_heads), np.nan)
    mask = np.zeros((B, wl.q_heads), bool)
    for b, h in pairs:
        kk = torch.cat([k[b:b + 1, h:h + 1], kn[b:b + 1, h:h + 1]], 2)
        vv = torch.cat([v[b:b + 1, h:h + 1], vn[b:b + 1, h:h + 1]], 2)
        seg = oracle_segment(kk, vv, wl.bits, wl.group)
        qq = q[b:b + 1, h * g:(h + 1) * g]
        r, lr = oracle.decode_attention(q_bits(qq), q.dtype == torch.bfloat16, [seg], [[L + 1]],
                                        128 ** -0.5)
        ref[b, h * g:(h + 1) * g] = r[0]
        lref[b, h * g:(h + 1) * g] = lr[0]
        mask[b, h * g:(h + 1) * g] = True
    assert_close(out, ref, lse, lref, mask=mask, what=name)


def test_full_size_llama2_mha_int8_sampled(kvq):
    _full_size(kvq, "llama2_7b_mha_int8", [(0, 0), (3, 17), (15, 31), (7, 5)])


def test_full_size_llama3_gqa_int4_sampled(kvq):
    _full_size(kvq, "llama3_8b_gqa_int4", [(0, 0), (31, 7), (12, 3)])


def test_full_size_long_context_sampled(kvq):
    _full_size(kvq, "long_gqa_int4", [(0, 0), (0, 5)])


def _large_query_case(kvq, bits, G, g, q_dtype, mag, zero_channel):
    """K, V and queries N(0, 1), then one query element per head at `mag`
    (dim 5).
    With zero_channel, K's dim 5 is 0 on every token and dims 0..G-1 are
    |N(0, 1)|, so that group's minimum is 0, its zero point +0 and dim 5's
    code exactly 0: the large element contributes exactly nothing, and any
    overflow of it inside the kernel shows as NaN."""
    H, B, T = 2, 2, 200
    gen = torch.Generator(device=DEV)
    gen.manual_seed(77)
    k = torch.randn((B, H, T, 128), generator=gen, device=DEV).half()
    v = torch.randn((B, H, T, 128), generator=gen, device=DEV).half()
    if zero_channel:
        k[..., :G] = k[..., :G].abs()
        k[..., 5] = 0.0
    else:
        # the large element meets a key channel scaled so that q_5 k_5 stays
        # near N(0, 20^2): moderate scores, as the tensor cores' accumulation
        # (not fp32 rounding alone) limits the precision of much larger ones
        k[..., 5] = (k[..., 5].float() * (20.0 / mag)).half()
    qf = torch.randn((B, H * g, 128), generator=gen, device=DEV)
    qf[..., 5] = mag
    qf[:, ::2, 5] = -mag  # both signs
    q = qf.to(torch.bfloat16 if q_dtype == "bf16" else torch.float16)
    assert torch.isfinite(q).all()
    lens = [T, 151]
    c = kvq.QuantizedKVCache.allocate(B, H, 128, 256, bits, G, DEV)
    _poison(c)
    fill_cache(kvq, c, k, v, lens)
    out, lse = _run(kvq, c, q)
    seg = oracle_segment(k, v, bits, G)
    ref, lref = oracle.decode_attention(q_bits(q), q_dtype == "bf16", [seg], [lens],
                                        128 ** -0.5)
    return out, lse, ref, lref


@pytest.mark.parametrize("bits,G,g,q_dtype,mag", [
    (2, 32, 2, "f16", 2000.0), (2, 128, 8, "f16", 2000.0), (4, 64, 4, "f16", 5000.0),
    (4, 128, 1, "f16", 60000.0), (4, 64, 8, "f16", 5000.0), (2, 32, 4, "f16", 2000.0),
    (8, 128, 1, "f16", 60000.0), (4, 64, 4, "bf16", 1.0e5), (8, 128, 1, "bf16", 3.0e5),
    (2, 32, 2, "bf16", 1.0e6)])
def test_large_query_elements_do_not_overflow(kvq, bits, G, g, q_dtype, mag):
    """A query element the kernels lift past the fp16 range (INT2 codes lift
    query elements by up to 2^6, INT4 by 2^4) or a bf16 query above 65504:
    the staged row is scaled down by a power of two and its scores scaled
    back up, so the result is finite and within the attention tolerance of
    the oracle (the large element meets exact-zero codes here, so the fp32
    scores are as well conditioned as for N(0, 1) queries)."""
    out, lse, ref, lref = _large_query_case(kvq, bits, G, g, q_dtype, mag, zero_channel=True)
    assert_close(out, ref, lse, lref, what=f"large q bits{bits} G{G} g{g} {q_dtype} {mag}")


@pytest.mark.parametrize("bits,G,g,mag", [(4, 64, 4, 5000.0), (2, 32, 2, 2000.0),
                                          (4, 64, 8, 5000.0), (2, 128, 8, 1000.0)])
def test_large_query_elements_meet_real_keys(kvq, bits, G, g, mag):
    """The same large elements against keys whose channel 5 is scaled to
    keep the products q_5 k_5 moderate: the large elements still meet real,
    nonzero codes (and would overflow without the row shift), and the
    result is within the attention tolerance.  A score is formed as
    s (sum q c - z sum q) with the codes' sum accumulated by the tensor
    cores, so its absolute error grows with |q_5| z rather than with the
    score: with 2-bit groups of 128 and eight heads per KV head the
    tolerance holds up to |q_5| of about 1000 (the header states the
    limit)."""
    out, lse, ref, lref = _large_query_case(kvq, bits, G, g, "f16", mag, zero_channel=False)
    assert_close(out, ref, lse, lref, what=f"large q, real keys bits{bits} G{G} g{g}")
