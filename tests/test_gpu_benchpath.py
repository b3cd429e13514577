"""GPU parity of the exact launches the benchmark times: kvq_decode_step (the
new token's quantize-on-write, the split-K attention and the in-kernel
log-sum-exp merge, one kernel) at the full workload shapes, with the
benchmark's cache capacity and length hint, over consecutive steps.

For every step: the appended token's codes and (scale, zero) of every
(sequence, KV head) are compared byte for byte with the oracle's quantization
of the same fp16 row (Cocktail page 3.2.2 formula), seq_lens advances by one,
and the attention of sampled (sequence, KV head) pairs is compared with the
fp64 oracle over the whole history (TurboQuant page 2.3: dequantization
inside the products; Cocktail page 3.2.3: the merged pieces equal the
unchunked attention) within 2e-3 max-abs and 1e-3 relative L2."""
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


def _bench_path(kvq, name, pairs, steps):
    wl = workloads.WORKLOADS[name]
    B, H, Hq, D, ctx = wl.batch, wl.kv_heads, wl.q_heads, wl.head_dim, wl.context
    g = wl.group_ratio
    episode = wl.steps
    max_tokens = workloads.round_up(ctx + episode + 1, 64)  # as the benchmark
    hint = ctx + episode
    k, v = workloads.kv_tokens(wl, ctx, DEV)
    c = kvq.QuantizedKVCache.allocate(B, H, D, max_tokens, wl.bits, wl.group, DEV)
    c.seq_lens.zero_()
    kvq.kvq_quantize_append(c, k, v, ctx, advance_seq_lens=True)
    ws = kvq.alloc_workspace(c, Hq, hint, device=DEV)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=DEV)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    hist_k = {p: [k[p[0], p[1]]] for p in pairs}
    hist_v = {p: [v[p[0], p[1]]] for p in pairs}
    for s in range(steps):
        kn, vn = workloads.kv_tokens(wl, 1, DEV, stream_extra=1 + s)
        q = workloads.queries(wl, DEV, step=s)
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        kvq.kvq_decode_step(c, kn, vn, q, out, lse, ws, max_len_hint=hint)
        torch.cuda.synchronize()
        assert kvq.workspace_error_word(ws) == 0
        L = ctx + s + 1
        assert c.seq_lens.tolist() == [L] * B, f"step {s}: seq_lens"
        # the appended row of every (sequence, KV head), byte for byte
        for which, x, codes, meta in (("K", kn, c.k_codes, c.k_meta),
                                      ("V", vn, c.v_codes, c.v_meta)):
            rows = f16_bits(x).reshape(B * H, D)
            oc, om = oracle.quantize_rows(rows, wl.group, wl.bits)
            got_c = codes[:, :, L - 1].reshape(B * H, -1).cpu().numpy()
            got_m = meta[:, :, L - 1].reshape(B * H, -1).cpu().numpy().view(np.uint16)
            np.testing.assert_array_equal(got_c, oc, err_msg=f"step {s}: {which} codes")
            np.testing.assert_array_equal(got_m, om.reshape(B * H, -1),
                                          err_msg=f"step {s}: {which} (scale, zero)")
        # attention of the sampled pairs over their whole history
        ref = np.full((B, Hq, D), np.nan)
        lref = np.full((B, Hq), np.nan)
        mask = np.zeros((B, Hq), bool)
        for b, h in pairs:
            hist_k[(b, h)].append(kn[b, h])
            hist_v[(b, h)].append(vn[b, h])
            kk = f16_bits(torch.cat(hist_k[(b, h)], 0))
            vv = f16_bits(torch.cat(hist_v[(b, h)], 0))
            kc, km = oracle.quantize_rows(kk, wl.group, wl.bits)
            vc, vm = oracle.quantize_rows(vv, wl.group, wl.bits)
            seg = dict(k_codes=kc[None, None], k_meta=km[None, None], v_codes=vc[None, None],
                       v_meta=vm[None, None], bits=wl.bits, group=wl.group)
            qq = q[b:b + 1, h * g:(h + 1) * g]
            r, lr = oracle.decode_attention(q_bits(qq), q.dtype == torch.bfloat16, [seg], [[L]],
                                            D ** -0.5)
            ref[b, h * g:(h + 1) * g] = r[0]
            lref[b, h * g:(h + 1) * g] = lr[0]
            mask[b, h * g:(h + 1) * g] = True
        assert_close(out, ref, lse, lref, mask=mask, what=f"{name} step {s}")
        assert torch.all(torch.isfinite(out)) and torch.all(torch.isfinite(lse))


def test_bench_path_llama3_gqa_int4(kvq):
    """Batch 32, 32 query / 8 KV heads, INT4 G64, context 8192: 3 steps."""
    _bench_path(kvq, "llama3_8b_gqa_int4", [(0, 0), (31, 7), (12, 3), (20, 5)], steps=3)


def test_bench_path_llama2_mha_int8_bf16_queries(kvq):
    """Batch 16, 32 heads, INT8 G128, bf16 queries, context 4096: 3 steps."""
    _bench_path(kvq, "llama2_7b_mha_int8", [(0, 0), (15, 31), (7, 12)], steps=3)


def test_bench_path_long_context(kvq):
    """One sequence of 131072 tokens, 32 query / 8 KV heads, INT4 G64: each
    KV head spread over about 74 CTAs, merged in two levels; 2 steps."""
    _bench_path(kvq, "long_gqa_int4", [(0, 0), (0, 7)], steps=2)
