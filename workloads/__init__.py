"""Seeded synthetic inputs for the decode workloads (no quantization or
attention arithmetic lives here).

This module is the one piece shared by the tests, the benchmark and the
smoke check: it only draws random tensors with the shapes, distributions and
outlier structure of the five decode workloads, on whatever torch device it
is given.  Everything random comes from ``torch.Generator`` objects seeded
from the workload seed and a fixed stream id, so a tensor does not depend on
the order in which others were drawn.

The workloads stand in for the pages' Llama-shaped decode layers (no model
weights or datasets are needed): K/V rows are N(0, sigma) with a few
"channel outliers" (whole head_dim channels scaled up for every token, the
phenomenon the TurboQuant page blames for poor global scales), queries are
N(0, 1), and the chunk-level mixed-precision workload draws 768-d chunk
embeddings in place of a retrieval encoder.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

# stream ids: one generator per kind of tensor
_S_CHANNELS, _S_K, _S_V, _S_Q, _S_STEP, _S_EMB, _S_PICK, _S_NOISE = range(8)


@dataclass(frozen=True)
class Outliers:
    """Which K or V channels are scaled, and by how much.

    ``channels`` lists fixed head_dim indices used in every KV head;
    ``fraction`` picks round(fraction * kv_heads * head_dim) (head, dim)
    channels of the layer without replacement; ``per_head`` picks that many
    dims in each KV head.  Exactly one of them is set (or none: no outliers).
    """
    factor: float = 1.0
    channels: Tuple[int, ...] = ()
    fraction: float = 0.0
    per_head: int = 0


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    context: int
    bits: int                 # 2, 4, 8 (16 = raw fp16)
    group: int
    q_dtype: str              # "f16" or "bf16"
    steps: int                # decode steps (appends + attention); 1 = attention only
    append: bool              # a fresh token is quantized and appended each step
    seed: int
    k_outliers: Outliers = Outliers()
    v_outliers: Outliers = Outliers()
    k_sigma: float = 1.0
    v_sigma: float = 1.0
    # chunk-level mixed precision (Cocktail-style)
    chunk_tokens: int = 0
    emb_dim: int = 0
    query_pool: int = 0       # the query embedding averages this many chunk embeddings
    query_noise: float = 0.0
    alpha: float = 0.0
    beta: float = 0.0
    low_bits: Tuple[int, ...] = ()   # bit-widths of the two quantized classes
    fmt: str = "int"          # code format: "int" (asymmetric integer), "fp8" (E4M3, bits 8),
    #                           "e5m2" (E5M2, bits 8), "sym8" (symmetric INT8, bits 8) or
    #                           "oaken" (group-shift codec, bits 4, group = head_dim)
    outer_bits: int = 5       # "oaken": bits of an outlier's shifted magnitude
    k_axis: str = "token"     # K grouping: "token" (groups along head_dim) or "channel"
    #                           (per channel over 32-token blocks; attention only)

    @property
    def group_ratio(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def n_chunks(self) -> int:
        return self.context // self.chunk_tokens if self.chunk_tokens else 0

    def scaled(self, **kw) -> "DecodeWorkload":
        """The same workload at other sizes (tests run reduced copies)."""
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": DecodeWorkload(
        name="tiny", batch=1, q_heads=1, kv_heads=1, head_dim=128, context=256,
        bits=4, group=64, q_dtype="f16", steps=1, append=False, seed=0,
        k_outliers=Outliers(factor=20.0, channels=(3, 77)),
        v_outliers=Outliers(factor=20.0, channels=(3, 77))),
    "llama2_7b_mha_int8": DecodeWorkload(
        name="llama2_7b_mha_int8", batch=16, q_heads=32, kv_heads=32, head_dim=128,
        context=4096, bits=8, group=128, q_dtype="bf16", steps=100, append=True, seed=2,
        k_outliers=Outliers(factor=10.0, fraction=0.01),
        v_outliers=Outliers(factor=10.0, fraction=0.01)),
    "llama3_8b_gqa_int4": DecodeWorkload(
        name="llama3_8b_gqa_int4", batch=32, q_heads=32, kv_heads=8, head_dim=128,
        context=8192, bits=4, group=64, q_dtype="f16", steps=100, append=True, seed=3,
        k_outliers=Outliers(factor=15.0, per_head=4), v_sigma=0.5),
    "cocktail_mixed": DecodeWorkload(
        name="cocktail_mixed", batch=8, q_heads=40, kv_heads=40, head_dim=128,
        context=32768, bits=4, group=32, q_dtype="f16", steps=100, append=False, seed=4,
        chunk_tokens=32, emb_dim=768, query_pool=20, query_noise=0.1, alpha=0.6, beta=0.1,
        low_bits=(4, 2)),
    # the FP8 E4M3 variant of the KV-cache page, on the Llama-2 and Llama-3 shapes
    "llama2_7b_mha_fp8": DecodeWorkload(
        name="llama2_7b_mha_fp8", batch=16, q_heads=32, kv_heads=32, head_dim=128,
        context=4096, bits=8, group=128, q_dtype="bf16", steps=100, append=True, seed=2,
        k_outliers=Outliers(factor=10.0, fraction=0.01),
        v_outliers=Outliers(factor=10.0, fraction=0.01), fmt="fp8"),
    "llama3_8b_gqa_fp8": DecodeWorkload(
        name="llama3_8b_gqa_fp8", batch=32, q_heads=32, kv_heads=8, head_dim=128,
        context=8192, bits=8, group=64, q_dtype="f16", steps=100, append=True, seed=3,
        k_outliers=Outliers(factor=15.0, per_head=4), v_sigma=0.5, fmt="fp8"),
    "llama3_8b_gqa_e5m2": DecodeWorkload(
        name="llama3_8b_gqa_e5m2", batch=32, q_heads=32, kv_heads=8, head_dim=128,
        context=8192, bits=8, group=64, q_dtype="f16", steps=100, append=True, seed=3,
        k_outliers=Outliers(factor=15.0, per_head=4), v_sigma=0.5, fmt="e5m2"),
    "llama2_7b_mha_sym8": DecodeWorkload(
        name="llama2_7b_mha_sym8", batch=16, q_heads=32, kv_heads=32, head_dim=128,
        context=4096, bits=8, group=128, q_dtype="bf16", steps=100, append=True, seed=2,
        k_outliers=Outliers(factor=10.0, fraction=0.01),
        v_outliers=Outliers(factor=10.0, fraction=0.01), fmt="sym8"),
    "llama3_8b_gqa_int4_kpc": DecodeWorkload(
        name="llama3_8b_gqa_int4_kpc", batch=32, q_heads=32, kv_heads=8, head_dim=128,
        context=8192, bits=4, group=64, q_dtype="f16", steps=100, append=False, seed=3,
        k_outliers=Outliers(factor=15.0, per_head=4), v_sigma=0.5, k_axis="channel"),
    "llama3_8b_gqa_oaken": DecodeWorkload(
        name="llama3_8b_gqa_oaken", batch=32, q_heads=32, kv_heads=8, head_dim=128,
        context=8192, bits=4, group=128, q_dtype="f16", steps=100, append=False, seed=3,
        k_outliers=Outliers(factor=15.0, per_head=4), v_sigma=0.5, fmt="oaken"),
    "long_gqa_int4": DecodeWorkload(
        name="long_gqa_int4", batch=1, q_heads=32, kv_heads=8, head_dim=128,
        context=131072, bits=4, group=64, q_dtype="f16", steps=256, append=True, seed=5,
        k_outliers=Outliers(factor=20.0, fraction=0.01),
        v_outliers=Outliers(factor=20.0, fraction=0.01)),
}


def _gen(device, seed: int, stream: int, extra: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + stream * 7919 + extra) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def outlier_mask(wl: DecodeWorkload, which: str) -> torch.Tensor:
    """[kv_heads, head_dim] float32 multipliers (1 or the outlier factor), CPU."""
    spec = wl.k_outliers if which == "k" else wl.v_outliers
    H, D = wl.kv_heads, wl.head_dim
    mult = torch.ones(H, D, dtype=torch.float32)
    g = _gen("cpu", wl.seed, _S_CHANNELS, 0 if which == "k" else 1)
    if spec.channels:
        mult[:, list(spec.channels)] = spec.factor
    elif spec.fraction > 0:
        n = int(round(spec.fraction * H * D))
        idx = torch.randperm(H * D, generator=g)[:n]
        mult.view(-1)[idx] = spec.factor
    elif spec.per_head > 0:
        for h in range(H):
            idx = torch.randperm(D, generator=g)[:spec.per_head]
            mult[h, idx] = spec.factor
    return mult


def kv_tokens(wl: DecodeWorkload, n_tokens: int, device, stream_extra: int = 0,
              batch: Optional[int] = None, dtype: torch.dtype = torch.float16):
    """Fresh K and V rows [B, kv_heads, n_tokens, head_dim] of ``dtype``
    (fp16, or bf16: the same fp32 draws rounded to the other type).

    ``stream_extra`` selects an independent stream (0 = the prompt/context,
    1 + step = the token appended at that decode step)."""
    B = wl.batch if batch is None else batch
    shape = (B, wl.kv_heads, n_tokens, wl.head_dim)
    out = []
    for which, stream, sigma in (("k", _S_K, wl.k_sigma), ("v", _S_V, wl.v_sigma)):
        g = _gen(device, wl.seed, stream, stream_extra)
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        x.mul_(sigma)
        x.mul_(outlier_mask(wl, which).to(device)[None, :, None, :])
        out.append(x.to(dtype))
    return out[0], out[1]


def queries(wl: DecodeWorkload, device, step: int = 0, batch: Optional[int] = None):
    """Query vectors [B, q_heads, head_dim] in the workload's query dtype."""
    B = wl.batch if batch is None else batch
    g = _gen(device, wl.seed, _S_Q, step)
    q = torch.randn((B, wl.q_heads, wl.head_dim), generator=g, device=device,
                    dtype=torch.float32)
    return q.to(torch.bfloat16 if wl.q_dtype == "bf16" else torch.float16)


def chunk_embeddings(wl: DecodeWorkload, device, batch: Optional[int] = None):
    """Chunk embeddings [B, n_chunks, emb_dim] fp32 ~ N(0, 1), and query
    embeddings [B, emb_dim]: the mean of ``query_pool`` distinct random chunk
    embeddings plus N(0, query_noise) noise."""
    B = wl.batch if batch is None else batch
    n, E = wl.n_chunks, wl.emb_dim
    emb = torch.randn((B, n, E), generator=_gen(device, wl.seed, _S_EMB), device=device,
                      dtype=torch.float32)
    gp = _gen("cpu", wl.seed, _S_PICK)
    picks = torch.stack([torch.randperm(n, generator=gp)[:wl.query_pool] for _ in range(B)])
    picks = picks.to(device)
    pooled = torch.stack([emb[b, picks[b]].mean(0) for b in range(B)])
    noise = torch.randn((B, E), generator=_gen(device, wl.seed, _S_NOISE), device=device,
                        dtype=torch.float32)
    return emb, pooled + wl.query_noise * noise


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


# stream of the calibration sample behind the Oaken planes' offline parameters
_CALIBRATION_EXTRA = 1 << 20


def oaken_params(wl: DecodeWorkload, which: str, n_tokens: int = 512):
    """Offline parameters (inner_scale, inner_zero, outer_scale, outer_bits)
    of the K ("k") or V ("v") plane of an "oaken" workload, from percentile
    statistics of a calibration sample drawn like the workload's rows (an
    independent stream, one sequence): the 2.5th and 97.5th percentiles
    bound the 4-bit band, so about 5% of the values fall in the outer zone;
    inner_scale is the smallest fp16 value with 15 steps spanning that band;
    inner_zero puts the low percentile on the grid; outer_scale lets the
    sample's extremes reach the largest outlier magnitude."""
    k, v = kv_tokens(wl, n_tokens, "cpu", stream_extra=_CALIBRATION_EXTRA, batch=1)
    x = (k if which == "k" else v).float().flatten()
    lo = float(torch.quantile(x, 0.025))
    hi = float(torch.quantile(x, 0.975))
    span = torch.tensor((hi - lo) / 15.0, dtype=torch.float32)
    s16 = span.half()
    if s16.float() < span:
        s16 = torch.nextafter(s16, torch.tensor(float("inf"), dtype=torch.float16))
    s_in = float(s16)
    z_in = int(min(max(round(-lo / s_in), 0), 15))
    t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
    reach = max(float(x.max()) - t_hi, t_lo - float(x.min()), s_in)
    s_out = float(torch.tensor(reach / ((1 << wl.outer_bits) - 1), dtype=torch.float32))
    return s_in, z_in, s_out, wl.outer_bits
