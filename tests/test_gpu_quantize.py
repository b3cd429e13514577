"""GPU parity of quantize-on-write (kvq_quantize_append) against the oracle:
codes, scales and zero points compared byte for byte."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import f16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


DEV = "cuda"


def _alloc(kvq, B, H, max_tokens, bits, G):
    c = kvq.QuantizedKVCache.allocate(B, H, 128, max_tokens, bits, G, DEV)
    # stale bytes everywhere (NaN meta patterns) so unwritten slots are visible
    c.k_codes.fill_(0xA5)
    c.v_codes.fill_(0x5A)
    c.k_meta.view(torch.int16).fill_(-1)
    c.v_meta.view(torch.int16).fill_(-1)
    return c


def _expect(k, v, bits, G):
    kc, km = oracle.quantize_cache(f16_bits(k), G, bits)
    vc, vm = oracle.quantize_cache(f16_bits(v), G, bits)
    return kc, km, vc, vm


def _meta_bits(t):
    return t.cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_bulk_quantize_bit_exact(kvq, bits, G):
    wl = workloads.WORKLOADS["long_gqa_int4"].scaled(batch=3, kv_heads=2, q_heads=2)
    T = 37  # several row pairs and a ragged tail
    k, v = workloads.kv_tokens(wl, T, DEV)
    c = _alloc(kvq, 3, 2, 64, bits, G)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    kc, km, vc, vm = _expect(k, v, bits, G)
    assert np.array_equal(c.k_codes[:, :, :T].cpu().numpy(), kc)
    assert np.array_equal(c.v_codes[:, :, :T].cpu().numpy(), vc)
    assert np.array_equal(_meta_bits(c.k_meta[:, :, :T]), km)
    assert np.array_equal(_meta_bits(c.v_meta[:, :, :T]), vm)
    assert c.seq_lens.tolist() == [T] * 3
    # untouched slots keep their stale bytes
    assert (c.k_codes[:, :, T:] == 0xA5).all()


@pytest.mark.parametrize("bits,G", [(4, 64), (8, 128), (2, 32)])
def test_append_at_ragged_positions(kvq, bits, G):
    B, H = 3, 4
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    c = _alloc(kvq, B, H, 128, bits, G)
    start = [0, 5, 17]
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    for step in range(3):
        k, v = workloads.kv_tokens(wl, 2, DEV, stream_extra=1 + step)
        kvq.kvq_quantize_append(c, k, v, 2, advance_seq_lens=True)
        kc, km, vc, vm = _expect(k, v, bits, G)
        for b in range(B):
            p = start[b] + 2 * step
            assert np.array_equal(c.k_codes[b, :, p:p + 2].cpu().numpy(), kc[b])
            assert np.array_equal(c.v_codes[b, :, p:p + 2].cpu().numpy(), vc[b])
            assert np.array_equal(_meta_bits(c.k_meta[b, :, p:p + 2]), km[b])
            assert np.array_equal(_meta_bits(c.v_meta[b, :, p:p + 2]), vm[b])
    assert c.seq_lens.tolist() == [s + 6 for s in start]
    # no advance: lengths stay, data still written
    k, v = workloads.kv_tokens(wl, 1, DEV, stream_extra=99)
    kvq.kvq_quantize_append(c, k, v, 1, advance_seq_lens=False)
    assert c.seq_lens.tolist() == [s + 6 for s in start]


def _adversarial_rows():
    """Token rows built from hand-picked groups: constant groups, fp16
    extremes, subnormals, exact .5 ties, all-positive and all-negative groups,
    a single outlier."""
    rng = np.random.default_rng(123)
    rows = []
    specials = [
        np.full(128, 3.0), np.zeros(128), np.full(128, -0.0),
        np.tile([-1, 0, 0.5, 2], 32), np.tile([-1, 1.5, 0, 2], 32),
        np.tile([10, 11, 12, 13], 32), -np.tile([10, 11, 12, 13], 32),
        np.tile([65504, -65504], 64), np.tile([65504, 65504, 0, 1], 32),
        np.tile([6e-8, 0, -6e-8, 1.2e-7], 32), np.tile([6.1e-5, 3e-5, 1e-6, 0], 32),
        np.arange(128) % 16, -(np.arange(128) % 16), (np.arange(128) % 4) * 0.25,
    ]
    for s in specials:
        rows.append(s.astype(np.float16))
    x = rng.standard_normal(128)
    x[7] = 300
    rows.append(x.astype(np.float16))
    for _ in range(17):
        rows.append((rng.standard_normal(128) * rng.choice([1e-3, 1, 50])).astype(np.float16))
    # exact ties: x = (k + 0.5) * s with s a power of two
    for sc in (0.25, 1.0, 4.0):
        t = (rng.integers(-6, 6, 128) + 0.5) * sc
        t[0], t[1] = -8 * sc, 7 * sc
        rows.append(t.astype(np.float16))
    return np.stack(rows)


@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("G", [32, 64, 128])
def test_adversarial_groups_bit_exact(kvq, bits, G):
    rows = _adversarial_rows()
    n = rows.shape[0]
    k = torch.from_numpy(rows).to(DEV).view(1, 1, n, 128).contiguous()
    v = torch.from_numpy(rows[::-1].copy()).to(DEV).view(1, 1, n, 128).contiguous()
    c = _alloc(kvq, 1, 1, 64, bits, G)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, n, advance_seq_lens=True)
    kc, km, vc, vm = _expect(k, v, bits, G)
    assert np.array_equal(c.k_codes[:, :, :n].cpu().numpy(), kc)
    assert np.array_equal(_meta_bits(c.k_meta[:, :, :n]), km)
    assert np.array_equal(c.v_codes[:, :, :n].cpu().numpy(), vc)
    assert np.array_equal(_meta_bits(c.v_meta[:, :, :n]), vm)


def test_capacity_is_enforced_on_device(kvq):
    B, H = 2, 2
    wl = workloads.WORKLOADS["tiny"].scaled(batch=B, kv_heads=H, q_heads=H)
    c = _alloc(kvq, B, H, 64, 4, 64)
    c.seq_lens.copy_(torch.tensor([62, 10], dtype=torch.int32))
    k, v = workloads.kv_tokens(wl, 4, DEV)
    kvq.kvq_quantize_append(c, k, v, 4, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [64, 14]
    kc, km, vc, vm = _expect(k, v, 4, 64)
    assert np.array_equal(c.k_codes[0, :, 62:64].cpu().numpy(), kc[0, :, :2])
    assert np.array_equal(c.k_codes[1, :, 10:14].cpu().numpy(), kc[1])


def test_prefill_full_size_long_context_sampled(kvq):
    """131072-token bulk prefill of the long-context workload (1 x 8 KV heads,
    INT4 G64), compared on 4096 sampled rows of K and of V."""
    wl = workloads.WORKLOADS["long_gqa_int4"]
    T = wl.context
    k, v = workloads.kv_tokens(wl, T, DEV)
    c = kvq.QuantizedKVCache.allocate(1, wl.kv_heads, 128, T, 4, 64, DEV)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [T]
    rng = np.random.default_rng(0)
    h = rng.integers(0, wl.kv_heads, 4096)
    t = rng.integers(0, T, 4096)
    t[:16] = np.arange(T - 16, T)
    for src, codes, meta in ((k, c.k_codes, c.k_meta), (v, c.v_codes, c.v_meta)):
        x = f16_bits(src[0, h, t])
        ec, em = oracle.quantize_rows(x, 64, 4)
        assert np.array_equal(codes[0, h, t].cpu().numpy(), ec)
        assert np.array_equal(_meta_bits(meta[0, h, t]), em)


# ---- the bulk (prefill) kernel: eight or more tokens per sequence


def _alloc_fmt(kvq, B, H, max_tokens, bits, G, fmt):
    f = {"fp8": kvq.KVQ_FMT_FP8_E4M3, "e5m2": kvq.KVQ_FMT_FP8_E5M2}.get(fmt, kvq.KVQ_FMT_INT)
    c = kvq.QuantizedKVCache.allocate(B, H, 128, max_tokens, bits, G, DEV, fmt=f)
    c.k_codes.fill_(0xA5)
    c.v_codes.fill_(0x5A)
    c.k_meta.view(torch.int16).fill_(-1)
    c.v_meta.view(torch.int16).fill_(-1)
    return c


BULK_FORMATS = [(b, G, "int") for b in (2, 4, 8) for G in (32, 64, 128)] + \
               [(8, G, f) for G in (32, 64, 128) for f in ("fp8", "e5m2")]


@pytest.mark.parametrize("bits,G,fmt", BULK_FORMATS)
def test_bulk_kernel_ragged_starts_and_capacity(kvq, bits, G, fmt):
    """77 tokens per (sequence, KV head) over 4 heads (616 rows per
    sequence: the bulk kernel), appended at start positions 0, 3 and 60 of a
    128-token cache: the third sequence's last 9 tokens fall past capacity
    and are dropped; every written row equals the oracle's, every other slot
    keeps its bytes."""
    B, H, T, cap = 3, 4, 77, 128
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV)
    c = _alloc_fmt(kvq, B, H, cap, bits, G, fmt)
    start = [0, 3, 60]
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [min(s + T, cap) for s in start]
    kc, km = oracle.quantize_cache(f16_bits(k), G, bits, fmt)
    vc, vm = oracle.quantize_cache(f16_bits(v), G, bits, fmt)
    for b in range(B):
        n = min(T, cap - start[b])
        p = slice(start[b], start[b] + n)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b, :, :n])
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b, :, :n])
        assert np.array_equal(_meta_bits(c.k_meta[b, :, p]), km[b, :, :n])
        assert np.array_equal(_meta_bits(c.v_meta[b, :, p]), vm[b, :, :n])
        assert (c.k_codes[b, :, :start[b]] == 0xA5).all()
        assert (c.v_codes[b, :, start[b] + n:] == 0x5A).all()
        assert (c.k_meta[b, :, start[b] + n:].view(torch.int16) == -1).all()


@pytest.mark.parametrize("bits,G,fmt", [(8, 128, "int"), (4, 64, "int"), (2, 32, "int"),
                                        (4, 128, "int"), (8, 64, "fp8"), (8, 32, "e5m2")])
def test_bulk_kernel_scale_sweep_and_adversarial(kvq, bits, G, fmt):
    """Groups whose magnitudes sweep the fp16 range (2^-24 .. 2^15, so the
    scale runs from its 1e-5 floor to above 100), offsets that push the zero
    point to its clamp, and the hand-picked adversarial rows, all through the
    bulk kernel; codes, scales and zero points byte for byte."""
    rng = np.random.default_rng(7)
    rows = []
    for e in range(-24, 16):
        for off in (0.0, 3.0, -40.0):
            x = rng.standard_normal(128) * 2.0 ** e + off * 2.0 ** max(e, 0)
            rows.append(np.clip(x, -65504, 65504).astype(np.float16))
    rows = np.concatenate([np.stack(rows), _adversarial_rows()])
    n = rows.shape[0]  # tokens per (sequence, head): the bulk kernel
    H = 4
    k = torch.from_numpy(np.stack([rows] * H)).to(DEV).view(1, H, n, 128).contiguous()
    v = torch.from_numpy(np.stack([rows[::-1]] * H)).to(DEV).view(1, H, n, 128).contiguous()
    k[0, 1] = -k[0, 1]
    c = _alloc_fmt(kvq, 1, H, 192, bits, G, fmt)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, n, advance_seq_lens=True)
    assert torch.isfinite(k.float()).all()
    kc, km = oracle.quantize_cache(f16_bits(k), G, bits, fmt)
    vc, vm = oracle.quantize_cache(f16_bits(v), G, bits, fmt)
    assert np.array_equal(c.k_codes[:, :, :n].cpu().numpy(), kc)
    assert np.array_equal(_meta_bits(c.k_meta[:, :, :n]), km)
    assert np.array_equal(c.v_codes[:, :, :n].cpu().numpy(), vc)
    assert np.array_equal(_meta_bits(c.v_meta[:, :, :n]), vm)
