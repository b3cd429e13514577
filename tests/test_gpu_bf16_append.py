"""GPU parity of quantize-on-write with bfloat16 K/V input (kvq_quantize_append
with KVQ_BF16: the KV-cache page's caches come in bf16 as well as fp16)
against the oracle's bf16 path: codes, scales and zero points byte for byte,
through the one-CTA-per-sequence append kernel and the bulk kernel, in every
token-grouped format; and attention over a bf16-written cache within the
attention tolerance."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_util import assert_close, q_bits

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def kvq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _alloc(kvq, B, H, cap, bits, G, fmt):
    f = {"fp8": kvq.KVQ_FMT_FP8_E4M3, "e5m2": kvq.KVQ_FMT_FP8_E5M2,
         "sym8": kvq.KVQ_FMT_INT8_SYM}.get(fmt, kvq.KVQ_FMT_INT)
    c = kvq.QuantizedKVCache.allocate(B, H, 128, cap, bits, G, DEV, fmt=f)
    c.k_codes.fill_(0xA5)
    c.v_codes.fill_(0x5A)
    c.k_meta.view(torch.int16).fill_(-1)
    c.v_meta.view(torch.int16).fill_(-1)
    return c


def _meta(t):
    return t.cpu().numpy().view(np.uint16)


FORMATS = [(b, G, "int") for b in (2, 4, 8) for G in (32, 64, 128)] + \
          [(8, G, f) for G in (32, 64, 128) for f in ("fp8", "e5m2", "sym8")]


def _check_rows(c, k, v, bits, G, fmt, start, n_rows, untouched=True):
    """Rows start[b] .. start[b] + n_rows[b] - 1 of sequence b hold the
    oracle's codes and (s, z) of k[b], v[b]; with `untouched`, every slot
    before and after them still holds its stale bytes."""
    kc, km = oracle.quantize_cache(bits16(k), G, bits, fmt, in_dtype="bf16")
    vc, vm = oracle.quantize_cache(bits16(v), G, bits, fmt, in_dtype="bf16")
    for b in range(k.shape[0]):
        n = n_rows[b]
        p = slice(start[b], start[b] + n)
        assert np.array_equal(c.k_codes[b, :, p].cpu().numpy(), kc[b, :, :n]), b
        assert np.array_equal(c.v_codes[b, :, p].cpu().numpy(), vc[b, :, :n]), b
        assert np.array_equal(_meta(c.k_meta[b, :, p]), km[b, :, :n]), b
        assert np.array_equal(_meta(c.v_meta[b, :, p]), vm[b, :, :n]), b
        if untouched:
            assert (c.k_codes[b, :, :start[b]] == 0xA5).all()
            assert (c.v_codes[b, :, start[b] + n:] == 0x5A).all()


@pytest.mark.parametrize("bits,G,fmt", FORMATS)
def test_bf16_append_kernel_bit_exact(kvq, bits, G, fmt):
    """Two tokens per (sequence, KV head) at ragged start positions, three
    steps: the one-CTA-per-sequence append kernel."""
    B, H = 3, 4
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    c = _alloc(kvq, B, H, 128, bits, G, fmt)
    start = [0, 5, 17]
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    for step in range(3):
        k, v = workloads.kv_tokens(wl, 2, DEV, stream_extra=1 + step, dtype=torch.bfloat16)
        kvq.kvq_quantize_append(c, k, v, 2, advance_seq_lens=True)
        _check_rows(c, k, v, bits, G, fmt, [s + 2 * step for s in start], [2] * B,
                    untouched=False)
    assert c.seq_lens.tolist() == [s + 6 for s in start]
    for b in range(B):  # slots outside the six written rows keep their bytes
        assert (c.k_codes[b, :, :start[b]] == 0xA5).all()
        assert (c.v_codes[b, :, start[b] + 6:] == 0x5A).all()
        assert (c.k_meta[b, :, start[b] + 6:].view(torch.int16) == -1).all()


@pytest.mark.parametrize("bits,G,fmt", FORMATS)
def test_bf16_bulk_kernel_ragged_starts_and_capacity(kvq, bits, G, fmt):
    """77 tokens per (sequence, KV head) over 4 heads (the bulk kernel) at
    start positions 0, 3 and 60 of a 128-token cache; the third sequence's
    last 9 tokens are dropped at capacity."""
    B, H, T, cap = 3, 4, 77, 128
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=H)
    k, v = workloads.kv_tokens(wl, T, DEV, dtype=torch.bfloat16)
    c = _alloc(kvq, B, H, cap, bits, G, fmt)
    start = [0, 3, 60]
    c.seq_lens.copy_(torch.tensor(start, dtype=torch.int32))
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    assert c.seq_lens.tolist() == [min(s + T, cap) for s in start]
    _check_rows(c, k, v, bits, G, fmt, start, [min(T, cap - s) for s in start])


def _sweep_rows(fmt):
    """bf16 rows whose groups sweep magnitudes from bf16 subnormals to values
    far beyond the fp16 range, each group's scale inside fp16 (the encodable
    range stated in the header): spreads 2^-133 .. 2^13 around offsets up to
    3 * 2^23, constant groups up to 2^40 for the integer formats, ties."""
    rng = np.random.default_rng(17)
    rows = []
    for e in range(-40, 14):
        for off in (0.0, 3.0, -40.0):
            rows.append(rng.standard_normal(128) * 2.0 ** e + off * 2.0 ** max(e, 0))
    rows.append(rng.integers(-8, 8, 128) * 2.0 ** -133)       # bf16 subnormals
    rows.append(1e5 + rng.standard_normal(128) * 100.0)
    rows.append(-3e6 + rng.standard_normal(128) * 1e4)
    for cst in (3e6, -7.5e5, 2.0 ** 20):
        rows.append(np.full(128, cst))
    if fmt == "int":
        rows.append(np.full(128, 2.0 ** 40))
        rows.append(np.full(128, -(2.0 ** 33)))
    for sc in (0.25, 1.0, 4.0, 2.0 ** 12):  # exact ties x = (k + 0.5) s
        t = (rng.integers(-6, 6, 128) + 0.5) * sc
        t[0], t[1] = -8 * sc, 7 * sc
        rows.append(t)
    return torch.tensor(np.stack(rows), dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("bits,G,fmt", [(8, 128, "int"), (4, 64, "int"), (2, 32, "int"),
                                        (4, 128, "int"), (8, 64, "fp8"), (8, 32, "e5m2"),
                                        (8, 128, "sym8")])
def test_bf16_scale_sweep_bulk_kernel(kvq, bits, G, fmt):
    rows = _sweep_rows(fmt)
    n, H = rows.shape[0], 4   # n >= 8 tokens per (sequence, head): the bulk kernel
    k = torch.stack([rows] * H).view(1, H, n, 128).to(DEV).contiguous()
    v = torch.stack([rows.flip(0)] * H).view(1, H, n, 128).to(DEV).contiguous()
    k[0, 1] = -k[0, 1]
    cap = ((n + 63) // 64) * 64
    c = _alloc(kvq, 1, H, cap, bits, G, fmt)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, n, advance_seq_lens=True)
    _check_rows(c, k, v, bits, G, fmt, [0], [n])
    # the same rows, a few at a time, through the append kernel
    c2 = _alloc(kvq, 1, H, cap, bits, G, fmt)
    c2.seq_lens.zero_()
    for i in range(0, n, 4):   # fewer than 8 tokens a call: the append kernel
        m = min(4, n - i)
        kvq.kvq_quantize_append(c2, k[:, :, i:i + m].contiguous(), v[:, :, i:i + m].contiguous(),
                                m, advance_seq_lens=True)
    assert torch.equal(c2.k_codes[:, :, :n], c.k_codes[:, :, :n])
    assert torch.equal(c2.v_meta[:, :, :n].view(torch.int16), c.v_meta[:, :, :n].view(torch.int16))


def test_bf16_written_cache_attention(kvq):
    """Attention over a cache written from bf16 K/V (Llama-3 GQA shape, INT4
    G64, 2 sequences of ragged length) against the oracle's attention over its
    own bf16 quantization of the same rows."""
    B, H, Hq, T = 2, 2, 8, 700
    wl = workloads.WORKLOADS["llama3_8b_gqa_int4"].scaled(batch=B, kv_heads=H, q_heads=Hq)
    k, v = workloads.kv_tokens(wl, T, DEV, dtype=torch.bfloat16)
    q = workloads.queries(wl, DEV)
    c = kvq.QuantizedKVCache.allocate(B, H, 128, 768, 4, 64, DEV)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, T, advance_seq_lens=True)
    lens = np.array([T, 333], np.int32)
    c.seq_lens.copy_(torch.from_numpy(lens).to(DEV))
    ws = kvq.alloc_workspace(c, Hq, T, device=DEV)
    out = torch.empty((B, Hq, 128), device=DEV)
    lse = torch.empty((B, Hq), device=DEV)
    kvq.kvq_decode_attention(c, q, out, lse, ws, max_len_hint=T)
    kc, km = oracle.quantize_cache(bits16(k), 64, 4, in_dtype="bf16")
    vc, vm = oracle.quantize_cache(bits16(v), 64, 4, in_dtype="bf16")
    seg = dict(k_codes=kc, v_codes=vc, k_meta=km, v_meta=vm, bits=4, group=64)
    ref, lref = oracle.decode_attention(q_bits(q), q.dtype == torch.bfloat16, [seg], [lens],
                                        128 ** -0.5)
    torch.cuda.synchronize()
    assert kvq.workspace_error_word(ws) == 0
    assert_close(out, ref, lse, lref, what="bf16-written INT4 cache")
