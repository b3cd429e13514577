"""GPU parity of the Cocktail chunk search (kvq_chunk_assign), the reorder
(kvq_chunk_reorder) and mixed-precision decode over the reordered cache."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_close, f16_bits, q_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def test_chunk_assign_bit_exact(kvq):
    wl = workloads.WORKLOADS["cocktail_mixed"].scaled(batch=3)
    emb, qemb = workloads.chunk_embeddings(wl, DEV)
    B, n = 3, wl.n_chunks
    bits = torch.zeros((B, n), dtype=torch.uint8, device=DEV)
    sim = torch.zeros((B, n), dtype=torch.float64, device=DEV)
    kvq.kvq_chunk_assign(emb, qemb, wl.alpha, wl.beta, bits, sim)
    torch.cuda.synchronize()
    e, qe = emb.cpu().numpy(), qemb.cpu().numpy()
    for b in range(B):
        s_ref, c_ref = oracle.chunk_assign(e[b], qe[b], wl.alpha, wl.beta)
        assert np.array_equal(sim[b].cpu().numpy().view(np.uint64), s_ref.view(np.uint64))
        assert np.array_equal(bits[b].cpu().numpy(), c_ref)
        counts = np.bincount(c_ref, minlength=17)[[16, 4, 2]]
        assert counts[0] >= 1 and counts.sum() == n


def test_chunk_assign_rounds_and_partial_tile(kvq):
    """More chunks than threads of the CTA (several rounds) and an embedding
    width that leaves a partial last tile: similarities bit for bit."""
    B, n, E = 2, 2500, 100
    g = torch.Generator(device=DEV)
    g.manual_seed(17)
    emb = torch.randn((B, n, E), generator=g, device=DEV)
    qemb = torch.randn((B, E), generator=g, device=DEV)
    bits = torch.zeros((B, n), dtype=torch.uint8, device=DEV)
    sim = torch.zeros((B, n), dtype=torch.float64, device=DEV)
    kvq.kvq_chunk_assign(emb, qemb, 0.6, 0.1, bits, sim)
    torch.cuda.synchronize()
    e, qe = emb.cpu().numpy(), qemb.cpu().numpy()
    for b in range(B):
        s_ref, c_ref = oracle.chunk_assign(e[b], qe[b], 0.6, 0.1)
        assert np.array_equal(sim[b].cpu().numpy().view(np.uint64), s_ref.view(np.uint64))
        assert np.array_equal(bits[b].cpu().numpy(), c_ref)


def test_chunk_assign_threshold_toy(kvq, golden_dir):
    import json
    import os
    ex = json.load(open(os.path.join(golden_dir, "chunk_threshold_toy.json")))
    emb = torch.tensor(ex["chunks"], dtype=torch.float32, device=DEV)[None]
    qe = torch.tensor(ex["query"], dtype=torch.float32, device=DEV)[None]
    bits = torch.zeros((1, emb.shape[1]), dtype=torch.uint8, device=DEV)
    sim = torch.zeros((1, emb.shape[1]), dtype=torch.float64, device=DEV)
    kvq.kvq_chunk_assign(emb, qe, ex["alpha"], ex["beta"], bits, sim)
    assert sim[0].tolist() == ex["sims"]
    assert bits[0].tolist() == ex["classes"]


def _segments(kvq, B, H, cap, G):
    segs = []
    for bits in (16, 4, 2):
        c = kvq.QuantizedKVCache.allocate(B, H, 128, cap, bits, G, DEV)
        c.k_codes.fill_(0xFF)
        c.v_codes.fill_(0xFF)
        if c.k_meta is not None:
            c.k_meta.view(torch.int16).fill_(-1)
            c.v_meta.view(torch.int16).fill_(-1)
        segs.append(c)
    return segs


def _check_reorder(kvq, wl, B, H, ctx, chunk_bits_np, oracle_bits=None, G=32):
    """chunk_bits_np goes to the kernel; oracle_bits (default the same) are
    the classes the oracle partitions by."""
    if oracle_bits is None:
        oracle_bits = chunk_bits_np
    T = wl.chunk_tokens
    n = ctx // T
    k, v = workloads.kv_tokens(wl, ctx, DEV, batch=B)
    segs = _segments(kvq, B, H, workloads.round_up(ctx, 64), G)
    cb = torch.from_numpy(chunk_bits_np).to(DEV)
    perm = torch.full((B, n), -1, dtype=torch.int32, device=DEV)
    kvq.kvq_chunk_reorder(segs, k, v, T, cb, perm)
    torch.cuda.synchronize()
    k16, v16 = f16_bits(k), f16_bits(v)
    oseg_lens = []
    osegs = [dict(k_codes=[], v_codes=[], k_meta=[], v_meta=[]) for _ in range(3)]
    for b in range(B):
        p_ref, counts = oracle.chunk_partition(oracle_bits[b])
        assert perm[b].tolist() == p_ref.tolist()
        lens = [int(x) * T for x in counts]
        oseg_lens.append(lens)
        assert [int(s.seq_lens[b]) for s in segs] == lens
        start = 0
        for i, (bits, cnt) in enumerate(zip((16, 4, 2), counts)):
            idx = p_ref[start:start + cnt]
            start += cnt
            tok = (idx[:, None] * T + np.arange(T)[None]).reshape(-1)
            for side, src in (("k", k16), ("v", v16)):
                rows = src[b][:, tok]  # [H, cnt*T, 128]
                got = getattr(segs[i], f"{side}_codes")[b, :, :cnt * T].cpu().numpy()
                if bits == 16:
                    assert np.array_equal(got.view(np.uint16).reshape(rows.shape), rows)
                else:
                    ec, em = oracle.quantize_cache(rows, G, bits)
                    assert np.array_equal(got, ec)
                    gm = getattr(segs[i], f"{side}_meta")[b, :, :cnt * T].cpu().numpy()
                    assert np.array_equal(gm.view(np.uint16), em)
    return k, v, segs, oseg_lens


def test_reorder_small_all_classes(kvq):
    wl = workloads.WORKLOADS["cocktail_mixed"].scaled(kv_heads=3, q_heads=3)
    B, H, ctx = 2, 3, 2048
    rng = np.random.default_rng(1)
    cbits = rng.choice(np.array([16, 4, 2], np.uint8), size=(B, ctx // 32), p=[0.1, 0.3, 0.6])
    cbits[1, :] = 2          # a sequence with a single class
    cbits[1, 5] = 7          # an unknown value counts as INT2
    cls = np.where(cbits == 7, 2, cbits).astype(np.uint8)
    k, v, segs, lens = _check_reorder(kvq, wl, B, H, ctx, cbits, oracle_bits=cls)
    # mixed decode over the reordered segments equals plain attention over
    # the original (unreordered) tokens with each chunk's own precision
    q = workloads.queries(wl, DEV, batch=B)
    out = torch.empty((B, H, 128), device=DEV)
    lse = torch.empty((B, H), device=DEV)
    ws = kvq.alloc_workspace(segs, H, device=DEV)
    kvq.kvq_decode_attention(segs, q, out, lse, ws)
    torch.cuda.synchronize()
    ref = np.zeros((B, H, 128))
    lref = np.zeros((B, H))
    k16, v16 = f16_bits(k), f16_bits(v)
    for b in range(B):
        for h in range(H):
            Ks, Vs = [], []
            for c in range(ctx // 32):
                rows_k = k16[b, h, c * 32:(c + 1) * 32]
                rows_v = v16[b, h, c * 32:(c + 1) * 32]
                bits = int(cls[b, c])
                kc, km = oracle.quantize_rows(rows_k, 32, bits)
                vc, vm = oracle.quantize_rows(rows_v, 32, bits)
                Ks.append(oracle.dequantize_rows(kc, km, 128, 32, bits))
                Vs.append(oracle.dequantize_rows(vc, vm, 128, 32, bits))
            qd = q[b, h:h + 1].float().cpu().numpy().astype(np.float64)
            o, l = oracle.attention(qd, np.concatenate(Ks), np.concatenate(Vs), 128 ** -0.5)
            ref[b, h], lref[b, h] = o[0], l[0]
    assert_close(out, ref, lse, lref, what="mixed decode vs original order")


def test_cocktail_full_size_sampled(kvq):
    """Full Cocktail workload: 8 sequences x 40 heads x 32768 tokens, chunk
    classes from the GPU search, reorder, decode; oracle on sampled heads."""
    wl = workloads.WORKLOADS["cocktail_mixed"]
    B, H, ctx, T = wl.batch, wl.kv_heads, wl.context, wl.chunk_tokens
    n = wl.n_chunks
    emb, qemb = workloads.chunk_embeddings(wl, DEV)
    cb = torch.zeros((B, n), dtype=torch.uint8, device=DEV)
    kvq.kvq_chunk_assign(emb, qemb, wl.alpha, wl.beta, cb)
    e, qe = emb.cpu().numpy(), qemb.cpu().numpy()
    cb_np = cb.cpu().numpy()
    for b in range(B):
        assert np.array_equal(cb_np[b], oracle.chunk_assign(e[b], qe[b], wl.alpha, wl.beta)[1])
    del emb
    k, v = workloads.kv_tokens(wl, ctx, DEV)
    segs = _segments(kvq, B, H, ctx, 32)
    perm = torch.empty((B, n), dtype=torch.int32, device=DEV)
    kvq.kvq_chunk_reorder(segs, k, v, T, cb, perm)
    q = workloads.queries(wl, DEV)
    out = torch.empty((B, H, 128), device=DEV)
    lse = torch.empty((B, H), device=DEV)
    ws = kvq.alloc_workspace(segs, H, max_len_hint=ctx, device=DEV)
    kvq.kvq_decode_attention(segs, q, out, lse, ws, max_len_hint=ctx)
    torch.cuda.synchronize()
    ref = np.full((B, H, 128), np.nan)
    lref = np.full((B, H), np.nan)
    mask = np.zeros((B, H), bool)
    for b, h in ((0, 0), (5, 39), (7, 11)):
        p_ref, counts = oracle.chunk_partition(cb_np[b])
        assert perm[b].tolist() == p_ref.tolist()
        osegs, lens = [], []
        start = 0
        for bits, cnt in zip((16, 4, 2), counts):
            idx = p_ref[start:start + cnt]
            start += cnt
            tok = torch.from_numpy((idx[:, None] * T + np.arange(T)[None]).reshape(-1)).to(DEV)
            kk = k[b:b + 1, h:h + 1, tok]
            vv = v[b:b + 1, h:h + 1, tok]
            from gpu_util import oracle_segment
            osegs.append(oracle_segment(kk, vv, bits, 32))
            lens.append([int(cnt) * T])
        r, lr = oracle.decode_attention(q_bits(q[b:b + 1, h:h + 1]), False, osegs, lens,
                                        128 ** -0.5)
        ref[b, h], lref[b, h], mask[b, h] = r[0, 0], lr[0, 0], True
    assert_close(out, ref, lse, lref, mask=mask, what="cocktail full size")


@pytest.mark.parametrize("G", [64, 128])
def test_reorder_chunk16_groups(kvq, G):
    """16-token chunks (two 8-row units each) and the larger group sizes:
    gathered rows and codes byte for byte against the oracle's partition."""
    wl = workloads.WORKLOADS["cocktail_mixed"].scaled(kv_heads=2, q_heads=2, chunk_tokens=16)
    B, H, ctx = 3, 2, 1024
    rng = np.random.default_rng(3)
    cbits = rng.choice(np.array([16, 4, 2], np.uint8), size=(B, ctx // 16), p=[0.2, 0.3, 0.5])
    cbits[2, :] = 4
    _check_reorder(kvq, wl, B, H, ctx, cbits, G=G)
