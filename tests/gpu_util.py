"""Test-side helpers for the GPU parity tests: build packed caches through the
C ABI, and the oracle's reference for the same seeded fp16 inputs (the oracle
quantizes the inputs itself; nothing it sees comes from the CUDA path)."""
import numpy as np
import torch

import oracle

ATOL = 2e-3      # attention: max-abs error against the fp64 oracle
RTOL_L2 = 1e-3   # attention: relative L2 error


def f16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def q_bits(q: torch.Tensor) -> np.ndarray:
    return f16_bits(q) if q.dtype == torch.float16 else \
        q.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def fill_cache(kvq, cache, k: torch.Tensor, v: torch.Tensor, lens):
    """Write the first lens[b] tokens of k/v ([B, H, T, D] fp16) into a packed
    cache through kvq_quantize_append (one bulk call, then trims seq_lens)."""
    cache.seq_lens.zero_()
    kvq.kvq_quantize_append(cache, k, v, k.shape[2], advance_seq_lens=True)
    cache.seq_lens.copy_(torch.as_tensor(np.asarray(lens, np.int32), device=cache.seq_lens.device))


def fill_fp16_segment(cache, k: torch.Tensor, v: torch.Tensor, lens):
    """A bits-16 segment stores raw fp16 rows: copy them in (data preparation)."""
    T = k.shape[2]
    cache.k_codes[:, :, :T].copy_(k.view(torch.uint8).view(*k.shape[:3], -1))
    cache.v_codes[:, :, :T].copy_(v.view(torch.uint8).view(*v.shape[:3], -1))
    cache.seq_lens.copy_(torch.as_tensor(np.asarray(lens, np.int32), device=cache.seq_lens.device))


def oracle_segment(k: torch.Tensor, v: torch.Tensor, bits: int, group: int, fmt: str = "int"):
    """The oracle's own packed cache of the same fp16 inputs (fmt "fp8": E4M3,
    "sym8": symmetric INT8)."""
    k16, v16 = f16_bits(k), f16_bits(v)
    if bits == 16:
        kc = k16.view(np.uint8).reshape(*k16.shape[:3], -1)
        vc = v16.view(np.uint8).reshape(*v16.shape[:3], -1)
        return dict(k_codes=kc, v_codes=vc, k_meta=None, v_meta=None, bits=16, group=128)
    kc, km = oracle.quantize_cache(k16, group, bits, fmt)
    vc, vm = oracle.quantize_cache(v16, group, bits, fmt)
    return dict(k_codes=kc, v_codes=vc, k_meta=km, v_meta=vm, bits=bits, group=group, fmt=fmt)


def assert_close(out: torch.Tensor, ref: np.ndarray, lse=None, lse_ref=None, mask=None,
                 what=""):
    o = out.detach().cpu().numpy().astype(np.float64)
    if mask is not None:
        o, ref = o[mask], ref[mask]
        if lse is not None:
            lse = lse.detach().cpu().numpy()[mask]
            lse_ref = lse_ref[mask]
    assert np.all(np.isfinite(o)), f"{what}: non-finite output"
    err = np.abs(o - ref).max() if o.size else 0.0
    nrm = np.linalg.norm(ref)
    rel = np.linalg.norm(o - ref) / nrm if nrm > 0 else np.linalg.norm(o - ref)
    assert err <= ATOL, f"{what}: max-abs {err:.3e} > {ATOL}"
    assert rel <= RTOL_L2, f"{what}: rel-L2 {rel:.3e} > {RTOL_L2}"
    if lse is not None:
        l = lse if isinstance(lse, np.ndarray) else lse.detach().cpu().numpy()
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(l), fin), f"{what}: lse finiteness"
        if fin.any():
            e2 = np.abs(l[fin] - lse_ref[fin]).max()
            assert e2 <= ATOL, f"{what}: lse max-abs {e2:.3e}"
    return err, rel
