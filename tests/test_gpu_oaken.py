"""GPU parity of the Oaken group-shift codec ("大模型KV缓存量化技术：原理、优化与
实践" page, sections 3.1, 3.2.1, 3.2.2; the oracle's reading R18): codes and
outlier slots written by kvq_quantize_append byte for byte equal to the
oracle's (ragged starts, the capacity edge, thresholds, ties, rows with more
outliers than slots, bf16 rows); decode attention over them within the attention
tolerance of the fp64 oracle (g = 1, 2, 4, 8; ragged, empty and one-token
lengths; bf16 queries; several split counts; rising scores); the decode
step (append, then attention); and the full-size workload in the
benchmark's launch configuration on sampled (sequence, KV head) pairs."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_close, f16_bits, q_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
WL = workloads.WORKLOADS["llama3_8b_gqa_oaken"]
KP, VP = workloads.oaken_params(WL, "k"), workloads.oaken_params(WL, "v")
TIES = (0.25, 8, 0.5, 6)  # T_lo = -2, T_hi = 1.75; outlier ties at 0.25 + k / 2


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def _alloc(kvq, B, H, max_tokens, kp=KP, vp=VP):
    c = kvq.QuantizedKVCache.allocate(B, H, 128, max_tokens, 4, 128, DEV,
                                      fmt=kvq.KVQ_FMT_OAKEN, k_oaken=kp, v_oaken=vp)
    c.k_codes.fill_(0xA5)  # stale codes and slots in unused rows
    c.v_codes.fill_(0x5A)
    c.k_meta.fill_(-1)
    c.v_meta.fill_(0x1234)
    return c


def _segment(k, v, kp=KP, vp=VP):
    kc, ks = oracle.oaken_quantize_cache(f16_bits(k), kp)
    vc, vs = oracle.oaken_quantize_cache(f16_bits(v), vp)
    return dict(k_codes=kc, v_codes=vc, k_meta=ks, v_meta=vs, bits=4, group=128, fmt="oaken",
                k_oaken=kp, v_oaken=vp)


def _fill(kvq, c, k, v, lens):
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, k.shape[2], advance_seq_lens=True)
    c.seq_lens.copy_(torch.as_tensor(np.asarray(lens, np.int32), device=DEV))


def _run(kvq, c, q, max_len_hint=0):
    B, Hq, D = q.shape
    out = torch.full((B, Hq, D), float("nan"), device=DEV)
    lse = torch.full((B, Hq), float("nan"), device=DEV)
    ws = kvq.alloc_workspace(c, Hq, max_len_hint, device=DEV)
    kvq.kvq_decode_attention(c, q, out, lse, ws, max_len_hint=max_len_hint)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws) == 0
    return out, lse


def _adversarial(k, v, kp):
    s_in, z_in, s_out, _ = kp
    t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
    grid = (torch.arange(-z_in, 16 - z_in, device=DEV).float() * s_in)
    k[0, 0, 0] = grid.repeat(8)[:128].half()                          # on the grid
    k[0, 0, 1] = ((grid + 0.5 * s_in).repeat(8)[:128]).half()         # inner ties
    k[0, 0, 2] = torch.where(torch.arange(128, device=DEV) % 2 == 0,  # every value outer
                             torch.tensor(t_hi + 40.0 * s_out + 1.0, device=DEV),
                             torch.tensor(t_lo - 3.0 * s_out - 1.0, device=DEV)).half()
    k[0, 0, 3, :64] = t_lo
    k[0, 0, 3, 64:] = t_hi
    k[0, 1, 4] = (torch.randn(128, device=DEV) * 2e4).clamp(-6e4, 6e4).half()
    k[0, 1, 5] = (torch.randn(128, device=DEV) * 1e-6).half()         # subnormals
    v[1, 0, 5] = -0.0
    v[1, 0, 6, :20] = torch.tensor(t_hi + 0.25 + 0.5 * np.arange(20), device=DEV).half()  # ties


@pytest.mark.parametrize("params", ["calibrated", "ties"])
@pytest.mark.parametrize("H,T", [(2, 41), (4, 77)])
def test_quantize_bit_exact(kvq, params, H, T):
    kp, vp = (KP, VP) if params == "calibrated" else (TIES, TIES)
    wl = WL.scaled(batch=3, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV)
    _adversarial(k, v, kp)
    c = _alloc(kvq, 3, H, 128, kp, vp)
    starts = [0, 5, 60]
    c.seq_lens.copy_(torch.tensor(starts, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    kc, ks = oracle.oaken_quantize_cache(f16_bits(k), kp)
    vc, vs = oracle.oaken_quantize_cache(f16_bits(v), vp)
    assert (ks != 0).sum(-1).max() == 16  # a row with more outliers than slots
    for b, st in enumerate(starts):
        n = min(T, 128 - st)
        p = slice(st, st + n)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b, :, :n])
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b, :, :n])
        assert np.array_equal(c.k_meta[b, :, p].cpu().numpy().view(np.uint16), ks[b, :, :n])
        assert np.array_equal(c.v_meta[b, :, p].cpu().numpy().view(np.uint16), vs[b, :, :n])
        # rows before the start and past the capacity are untouched
        assert np.all(c.k_codes[b, :, :st].cpu().numpy() == 0xA5)
    assert c.seq_lens.tolist() == [min(st + T, 128) for st in starts]


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_decode_attention(kvq, g):
    H = 2
    wl = WL.scaled(kv_heads=H, q_heads=H * g)
    lens = [300, 45, 1, 64]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, max(lens), DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    c = _alloc(kvq, B, H, 320)
    _fill(kvq, c, k, v, lens)
    out, lse = _run(kvq, c, q)
    seg = _segment(k, v)
    ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [lens], 128 ** -0.5)
    assert_close(out, ref, lse, lref, what=f"oaken g{g}")
    # one token: the output is that token's dequantized V row
    v1 = oracle.oaken_dequantize_rows(seg["v_codes"][2, 0, :1], seg["v_meta"][2, 0, :1], 128,
                                      *VP[:3])
    np.testing.assert_allclose(out[2, 0].cpu().numpy(), v1[0], atol=1e-5)


def test_edge_lengths_and_bf16(kvq):
    """Empty sequence (out 0, lse -inf), tile multiples and tails, the full
    capacity, bf16 queries."""
    wl = WL.scaled(kv_heads=2, q_heads=8, q_dtype="bf16")
    lens = [0, 32, 33, 31, 128, 97]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, 128, DEV, batch=B)
    q = workloads.queries(wl, DEV, batch=B)
    assert q.dtype == torch.bfloat16
    c = _alloc(kvq, B, 2, 128)
    _fill(kvq, c, k, v, lens)
    out, lse = _run(kvq, c, q)
    o = out.cpu().numpy()
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse.cpu().numpy()[0]))
    ref, lref = oracle.decode_attention(q_bits(q), True, [_segment(k, v)], [lens], 128 ** -0.5)
    mask = np.ones(B, bool)
    mask[0] = False
    assert_close(out, ref, lse, lref, mask=mask, what="oaken edges bf16")


@pytest.mark.parametrize("hint", [64, 0, 4096])
def test_split_counts_and_rising_scores(kvq, hint):
    """Keys growing along the sequence make the running max rise tile after
    tile (many rescales); the split count follows the hint."""
    wl = WL.scaled(kv_heads=1, q_heads=4)
    lens = [1000, 777]
    B, T = len(lens), max(lens)
    k, v = workloads.kv_tokens(wl, T, DEV, batch=B)
    k = (k.float() * torch.linspace(0.2, 3.0, T, device=DEV).view(1, 1, T, 1)).half()
    q = workloads.queries(wl, DEV, batch=B)
    c = _alloc(kvq, B, 1, 1024)
    _fill(kvq, c, k, v, lens)
    out, lse = _run(kvq, c, q, max_len_hint=hint)
    ref, lref = oracle.decode_attention(q_bits(q), False, [_segment(k, v)], [lens], 128 ** -0.5)
    assert_close(out, ref, lse, lref, what=f"oaken hint {hint}")


def test_decode_step(kvq):
    """kvq_decode_step on an Oaken cache: the append, then attention over the
    cache with the new token, several steps."""
    H, g = 2, 4
    wl = WL.scaled(kv_heads=H, q_heads=H * g)
    lens = [100, 7]
    B = len(lens)
    k, v = workloads.kv_tokens(wl, max(lens), DEV, batch=B)
    c = _alloc(kvq, B, H, 128)
    _fill(kvq, c, k, v, lens)
    ws = kvq.alloc_workspace(c, H * g, 0, device=DEV)
    hist_k = [[k[b, :, :lens[b]]] for b in range(B)]
    hist_v = [[v[b, :, :lens[b]]] for b in range(B)]
    cur = list(lens)
    for s in range(3):
        kn, vn = workloads.kv_tokens(wl, 1, DEV, stream_extra=40 + s, batch=B)
        q = workloads.queries(wl, DEV, step=s, batch=B)
        out = torch.empty((B, H * g, 128), device=DEV)
        lse = torch.empty((B, H * g), device=DEV)
        kvq.kvq_decode_step(c, kn, vn, q, out, lse, ws)
        torch.cuda.synchronize()
        for b in range(B):
            hist_k[b].append(kn[b])
            hist_v[b].append(vn[b])
            cur[b] += 1
        assert c.seq_lens.tolist() == cur
        T = max(cur)
        kk = torch.zeros((B, H, T, 128), dtype=torch.float16, device=DEV)
        vv = torch.zeros_like(kk)
        for b in range(B):
            kk[b, :, :cur[b]] = torch.cat(hist_k[b], 1)
            vv[b, :, :cur[b]] = torch.cat(hist_v[b], 1)
        seg = _segment(kk, vv)
        ref, lref = oracle.decode_attention(q_bits(q), False, [seg], [cur], 128 ** -0.5)
        assert_close(out, ref, lse, lref, what=f"oaken step {s}")
        for b in range(B):
            n = cur[b]
            assert np.array_equal(c.k_codes[b, :, :n].cpu().numpy(), seg["k_codes"][b, :, :n])
            assert np.array_equal(c.v_meta[b, :, :n].cpu().numpy().view(np.uint16),
                                  seg["v_meta"][b, :, :n])


def test_full_size_sampled(kvq):
    """The full workload (B 32, 32/8 heads, 8192 tokens) with the benchmark's
    cache capacity and length hint, the oracle on sampled pairs; the codes
    and slots of those pairs compared too."""
    B, H, L = WL.batch, WL.kv_heads, WL.context
    max_tokens = workloads.round_up(L + WL.steps + 1, 64)
    k, v = workloads.kv_tokens(WL, L, DEV)
    c = _alloc(kvq, B, H, max_tokens)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, L, advance_seq_lens=True)
    q = workloads.queries(WL, DEV)
    out, lse = _run(kvq, c, q, max_len_hint=L)
    g = WL.group_ratio
    ref = np.full((B, WL.q_heads, 128), np.nan)
    lref = np.full((B, WL.q_heads), np.nan)
    mask = np.zeros((B, WL.q_heads), bool)
    for b, h in [(0, 0), (31, 7), (12, 3)]:
        seg = _segment(k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1])
        assert np.array_equal(c.k_codes[b, h, :L].cpu().numpy(), seg["k_codes"][0, 0])
        assert np.array_equal(c.v_meta[b, h, :L].cpu().numpy().view(np.uint16), seg["v_meta"][0, 0])
        qq = q[b:b + 1, h * g:(h + 1) * g]
        r, lr = oracle.decode_attention(q_bits(qq), False, [seg], [[L]], 128 ** -0.5)
        ref[b, h * g:(h + 1) * g] = r[0]
        lref[b, h * g:(h + 1) * g] = lr[0]
        mask[b, h * g:(h + 1) * g] = True
    assert_close(out, ref, lse, lref, mask=mask, what="llama3_8b_gqa_oaken")


@pytest.mark.parametrize("n_new", [3, 160])
def test_bf16_quantize_bit_exact(kvq, n_new):
    """bf16 K/V (reading R19) through the append kernel (3 tokens) and the
    bulk kernel (160), against the oracle's bf16 path: the workload's rows,
    the hand-worked bf16 row of tests/golden (outliers beyond the fp16 range,
    values on the thresholds, halfway magnitudes) and a row of values far
    beyond fp16, byte for byte in codes and slots."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                                    "oaken_bf16_worked_example.json")))
    params = (g["s_in"], g["z_in"], g["s_out"], g["outer_bits"])
    B, H = 2, 4
    wl = WL.scaled(batch=B, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, n_new, DEV, dtype=torch.bfloat16)
    k[1, 2, 1, :8] = torch.tensor(g["values"], dtype=torch.float32).to(torch.bfloat16).to(DEV)
    v[0, 1, 0] = (torch.randn(128, device=DEV) * 1e6).to(torch.bfloat16)
    c = _alloc(kvq, B, H, 256, kp=params, vp=params)
    start = [0, 37]
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, n_new, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [s + n_new for s in start]

    def b16(t):
        return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kc, ks = oracle.oaken_quantize_cache(b16(k), params, in_dtype="bf16")
    vc, vs = oracle.oaken_quantize_cache(b16(v), params, in_dtype="bf16")
    assert ks[1, 2, 1, :5].tolist() == [int(h, 16) for h in g["slots"]]
    for b, st in enumerate(start):
        p = slice(st, st + n_new)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b]), b
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b]), b
        assert np.array_equal(c.k_meta[b, :, p].cpu().numpy().view(np.uint16), ks[b]), b
        assert np.array_equal(c.v_meta[b, :, p].cpu().numpy().view(np.uint16), vs[b]), b
        assert (c.k_codes[b, :, :st] == 0xA5).all() and (c.v_codes[b, :, st + n_new:] == 0x5A).all()
