"""Python binding of libkvq's C ABI (argument marshalling only).

Every function here has the name of the C entry point it calls and does
nothing but turn torch tensors into pointers, call the library, and raise
``KvqError`` on a non-OK status.  All computation happens in the CUDA
kernels of libkvq.so; if the library is missing this module raises on
import -- there is no fallback path.

PyTorch supplies device memory and streams: ``QuantizedKVCache`` allocates
the packed planes as torch tensors and describes them to the library.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_WORKSPACE, \
    KVQ_ERR_CUDA = range(6)
KVQ_F16, KVQ_BF16 = 0, 1
KVQ_FMT_INT, KVQ_FMT_FP8_E4M3, KVQ_FMT_INT8_SYM, KVQ_FMT_FP8_E5M2, KVQ_FMT_OAKEN = 0, 1, 2, 3, 4
KVQ_AXIS_TOKEN, KVQ_AXIS_CHANNEL = 0, 1
KVQ_CHANNEL_BLOCK = 32
KVQ_OAKEN_SLOTS = 16
HEADER_BYTES = 256  # workspace header: sticky device error word first


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {kvq_status_string(status)} (status {status})")


class kvq_oaken(ctypes.Structure):
    _fields_ = [("inner_scale", ctypes.c_float), ("inner_zero", ctypes.c_int32),
                ("outer_scale", ctypes.c_float), ("outer_bits", ctypes.c_int32)]


class kvq_plane(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("fmt", ctypes.c_int32),
                ("axis", ctypes.c_int32), ("oaken", kvq_oaken)]


class kvq_cache(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("max_tokens", ctypes.c_int32),
                ("k", kvq_plane), ("v", kvq_plane), ("seq_lens", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so not built ({LIB_PATH}); run "
                          "`python -m quantized_kv_cache_12_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, f32, f64, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_double,
                            ctypes.c_size_t)
    cp = ctypes.POINTER(kvq_cache)
    lib.kvq_status_string.argtypes = [ctypes.c_int]
    lib.kvq_status_string.restype = ctypes.c_char_p
    lib.kvq_version.restype = ctypes.c_char_p
    lib.kvq_plane_bytes.argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(sz),
                                    ctypes.POINTER(sz)]
    lib.kvq_kv_elements.argtypes = [ctypes.c_uint64] * 5
    lib.kvq_kv_elements.restype = ctypes.c_uint64
    lib.kvq_quantize_append.argtypes = [cp, P, P, i32, i32, i32, P]
    lib.kvq_decode_workspace_bytes.argtypes = [cp, i32, i32, i32, ctypes.POINTER(sz)]
    for name in ("kvq_decode_attention", "kvq_decode_partials", "kvq_decode_merge"):
        getattr(lib, name).argtypes = [cp, i32, P, ctypes.c_int, i32, f32, P, P, i32, P, sz, P]
    for name in ("kvq_decode_step", "kvq_decode_step_partials"):
        getattr(lib, name).argtypes = [cp, P, P, P, ctypes.c_int, i32, f32, P, P, i32, P, sz, P]
    lib.kvq_decode_attention_noalloc.argtypes = [cp, i32, P, ctypes.c_int, i32, f32, P, P,
                                                 i32, P]
    lib.kvq_decode_attention_noalloc.restype = ctypes.c_int
    lib.kvq_chunk_assign.argtypes = [P, P, i32, i32, i32, f64, f64, P, P, P]
    lib.kvq_chunk_reorder.argtypes = [cp, P, P, i32, i32, P, P, P]
    for name in ("kvq_plane_bytes", "kvq_quantize_append", "kvq_decode_workspace_bytes",
                 "kvq_decode_attention", "kvq_decode_partials", "kvq_decode_merge",
                 "kvq_decode_step", "kvq_decode_step_partials", "kvq_chunk_assign",
                 "kvq_chunk_reorder"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


lib = _load()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        if torch.cuda.is_available():
            return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        return ctypes.c_void_p(0)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(status: int, where: str):
    if status != KVQ_OK:
        raise KvqError(status, where)


def _caches(segs) -> ctypes.Array:
    if isinstance(segs, QuantizedKVCache):
        return segs.struct_array()
    if isinstance(segs, kvq_cache):
        segs = [segs]
    arr = (kvq_cache * len(segs))()
    for i, s in enumerate(segs):
        arr[i] = s.struct() if isinstance(s, QuantizedKVCache) else s
    return arr


# ---------------------------------------------------------------- C entry points

def kvq_status_string(status: int) -> str:
    return lib.kvq_status_string(int(status)).decode()


def kvq_version() -> str:
    return lib.kvq_version().decode()


def kvq_plane_bytes(batch, kv_heads, head_dim, max_tokens, bits, group_size):
    """-> (codes_bytes, meta_bytes)."""
    c, m = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.kvq_plane_bytes(batch, kv_heads, head_dim, max_tokens, bits, group_size,
                               ctypes.byref(c), ctypes.byref(m)), "kvq_plane_bytes")
    return c.value, m.value


def kvq_kv_elements(layers, kv_heads, head_dim, seq_len, batch) -> int:
    return int(lib.kvq_kv_elements(layers, kv_heads, head_dim, seq_len, batch))


def kvq_quantize_append(cache, k_new: torch.Tensor, v_new: torch.Tensor, n_new: int,
                        advance_seq_lens: bool = True, stream=None):
    """k_new and v_new are fp16 or bf16 (both the same); the dtype is passed
    as kvq_dtype."""
    if k_new.dtype != v_new.dtype or k_new.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("kvq_quantize_append: k_new and v_new must both be float16 or bfloat16")
    dt = KVQ_BF16 if k_new.dtype == torch.bfloat16 else KVQ_F16
    arr = _caches(cache)
    _check(lib.kvq_quantize_append(arr, _ptr(k_new), _ptr(v_new), dt, int(n_new),
                                   int(bool(advance_seq_lens)), _stream(stream)),
           "kvq_quantize_append")


def kvq_decode_workspace_bytes(segs, q_heads: int, max_len_hint: int = 0) -> int:
    arr = _caches(segs)
    n = ctypes.c_size_t()
    _check(lib.kvq_decode_workspace_bytes(arr, len(arr), int(q_heads), int(max_len_hint),
                                          ctypes.byref(n)), "kvq_decode_workspace_bytes")
    return n.value


def _decode_call(fn, name, segs, q, out, lse, workspace, softmax_scale, max_len_hint, stream):
    arr = _caches(segs)
    q_heads = q.shape[1]
    head_dim = q.shape[2]
    dt = KVQ_BF16 if q.dtype == torch.bfloat16 else KVQ_F16
    scale = softmax_scale if softmax_scale is not None else head_dim ** -0.5
    _check(fn(arr, len(arr), _ptr(q), dt, int(q_heads), float(scale), _ptr(out), _ptr(lse),
              int(max_len_hint), _ptr(workspace), workspace.numel() * workspace.element_size(),
              _stream(stream)), name)


def kvq_decode_attention(segs, q: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor],
                         workspace: torch.Tensor, softmax_scale: Optional[float] = None,
                         max_len_hint: int = 0, stream=None):
    _decode_call(lib.kvq_decode_attention, "kvq_decode_attention", segs, q, out, lse, workspace,
                 softmax_scale, max_len_hint, stream)


def kvq_decode_partials(segs, q: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor],
                        workspace: torch.Tensor, softmax_scale: Optional[float] = None,
                        max_len_hint: int = 0, stream=None):
    _decode_call(lib.kvq_decode_partials, "kvq_decode_partials", segs, q, out, lse, workspace,
                 softmax_scale, max_len_hint, stream)


def kvq_decode_merge(segs, q: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor],
                     workspace: torch.Tensor, softmax_scale: Optional[float] = None,
                     max_len_hint: int = 0, stream=None):
    _decode_call(lib.kvq_decode_merge, "kvq_decode_merge", segs, q, out, lse, workspace,
                 softmax_scale, max_len_hint, stream)


def _step_call(fn, name, cache, k_new, v_new, q, out, lse, workspace, softmax_scale,
               max_len_hint, stream):
    arr = _caches(cache)
    dt = KVQ_BF16 if q.dtype == torch.bfloat16 else KVQ_F16
    scale = softmax_scale if softmax_scale is not None else q.shape[2] ** -0.5
    _check(fn(arr, _ptr(k_new), _ptr(v_new), _ptr(q), dt, int(q.shape[1]), float(scale),
              _ptr(out), _ptr(lse), int(max_len_hint), _ptr(workspace),
              workspace.numel() * workspace.element_size(), _stream(stream)), name)


def kvq_decode_step(cache, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                    out: torch.Tensor, lse: Optional[torch.Tensor], workspace: torch.Tensor,
                    softmax_scale: Optional[float] = None, max_len_hint: int = 0, stream=None):
    """Append one token per (sequence, KV head) -- quantized into the cache --
    and attend over the cache including it; advances cache.seq_lens."""
    _step_call(lib.kvq_decode_step, "kvq_decode_step", cache, k_new, v_new, q, out, lse,
               workspace, softmax_scale, max_len_hint, stream)


def kvq_decode_step_partials(cache, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor,
                             out: torch.Tensor, lse: Optional[torch.Tensor],
                             workspace: torch.Tensor, softmax_scale: Optional[float] = None,
                             max_len_hint: int = 0, stream=None):
    """The append and the split-K partials of kvq_decode_step; follow with
    kvq_decode_merge."""
    _step_call(lib.kvq_decode_step_partials, "kvq_decode_step_partials", cache, k_new, v_new,
               q, out, lse, workspace, softmax_scale, max_len_hint, stream)


def kvq_decode_attention_noalloc(segs, q: torch.Tensor, out: torch.Tensor,
                                 lse: Optional[torch.Tensor], softmax_scale: Optional[float] = None,
                                 max_len_hint: int = 0, stream=None):
    """kvq_decode_attention with the library's own fixed scratch array instead
    of a caller workspace (for callers that cannot allocate device memory)."""
    arr = _caches(segs)
    dt = KVQ_BF16 if q.dtype == torch.bfloat16 else KVQ_F16
    scale = softmax_scale if softmax_scale is not None else q.shape[2] ** -0.5
    _check(lib.kvq_decode_attention_noalloc(arr, len(arr), _ptr(q), dt, int(q.shape[1]),
                                            float(scale), _ptr(out), _ptr(lse),
                                            int(max_len_hint), _stream(stream)),
           "kvq_decode_attention_noalloc")


def kvq_chunk_assign(chunk_emb: torch.Tensor, query_emb: torch.Tensor, alpha: float,
                     beta: float, chunk_bits_out: torch.Tensor,
                     sim_out: Optional[torch.Tensor] = None, stream=None):
    B, n, E = chunk_emb.shape
    _check(lib.kvq_chunk_assign(_ptr(chunk_emb), _ptr(query_emb), B, n, E, float(alpha),
                                float(beta), _ptr(sim_out), _ptr(chunk_bits_out),
                                _stream(stream)), "kvq_chunk_assign")


def kvq_chunk_reorder(segs, k_src: torch.Tensor, v_src: torch.Tensor, chunk_tokens: int,
                      chunk_bits: torch.Tensor, perm_out: torch.Tensor, stream=None):
    arr = _caches(segs)
    _check(lib.kvq_chunk_reorder(arr, _ptr(k_src), _ptr(v_src), int(k_src.shape[2]),
                                 int(chunk_tokens), _ptr(chunk_bits), _ptr(perm_out),
                                 _stream(stream)), "kvq_chunk_reorder")


# ---------------------------------------------------------------- torch-owned cache

@dataclass
class QuantizedKVCache:
    """Packed K/V planes of one cache (or one segment), owned by torch.

    codes: uint8 [B, H_kv, max_tokens, head_dim*bits/8];
    meta: fp16 [B, H_kv, max_tokens, head_dim/G, 2] (scale, zero), None for bits 16;
    seq_lens: int32 [B] on the device; fmt: KVQ_FMT_INT, KVQ_FMT_FP8_E4M3
    (bits 8: E4M3 codes, zero points 0), KVQ_FMT_FP8_E5M2 (bits 8: E5M2 codes,
    zero points 0) or KVQ_FMT_INT8_SYM (bits 8: two's complement codes, zero
    points 0).
    k_axis: KVQ_AXIS_TOKEN, or KVQ_AXIS_CHANNEL (K grouped per channel over
    blocks of KVQ_CHANNEL_BLOCK tokens: k_meta fp16 [B, H_kv,
    max_tokens / KVQ_CHANNEL_BLOCK, head_dim, 2]; group_size is V's).
    fmt KVQ_FMT_OAKEN (bits 4, group_size = head_dim): meta holds the outlier
    slots, int16 [B, H_kv, max_tokens, KVQ_OAKEN_SLOTS] (16-bit words), and
    k_oaken / v_oaken the planes' offline (inner_scale, inner_zero,
    outer_scale, outer_bits).
    """
    batch: int
    kv_heads: int
    head_dim: int
    max_tokens: int
    bits: int
    group_size: int
    k_codes: torch.Tensor
    v_codes: torch.Tensor
    k_meta: Optional[torch.Tensor]
    v_meta: Optional[torch.Tensor]
    seq_lens: torch.Tensor
    fmt: int = KVQ_FMT_INT
    k_axis: int = KVQ_AXIS_TOKEN
    k_oaken: Optional[tuple] = None
    v_oaken: Optional[tuple] = None

    @classmethod
    def allocate(cls, batch, kv_heads, head_dim, max_tokens, bits, group_size, device="cuda",
                 fmt: int = KVQ_FMT_INT, k_axis: int = KVQ_AXIS_TOKEN, k_oaken=None,
                 v_oaken=None):
        rb = head_dim * bits // 8
        shape = (batch, kv_heads, max_tokens, rb)
        k = torch.empty(shape, dtype=torch.uint8, device=device)
        v = torch.empty(shape, dtype=torch.uint8, device=device)
        km = vm = None
        if fmt == KVQ_FMT_OAKEN:
            sshape = (batch, kv_heads, max_tokens, KVQ_OAKEN_SLOTS)
            km = torch.empty(sshape, dtype=torch.int16, device=device)
            vm = torch.empty(sshape, dtype=torch.int16, device=device)
        elif bits != 16:
            mshape = (batch, kv_heads, max_tokens, head_dim // group_size, 2)
            kshape = ((batch, kv_heads, max_tokens // KVQ_CHANNEL_BLOCK, head_dim, 2)
                      if k_axis == KVQ_AXIS_CHANNEL else mshape)
            km = torch.empty(kshape, dtype=torch.float16, device=device)
            vm = torch.empty(mshape, dtype=torch.float16, device=device)
        lens = torch.zeros(batch, dtype=torch.int32, device=device)
        return cls(batch, kv_heads, head_dim, max_tokens, bits, group_size, k, v, km, vm, lens,
                   fmt, k_axis, k_oaken, v_oaken)

    def struct_array(self) -> ctypes.Array:
        """A one-element kvq_cache array for this cache, built on first use
        (the planes' tensors are allocated once and never replaced)."""
        arr = self.__dict__.get("_struct_array")
        if arr is None:
            arr = (kvq_cache * 1)(self.struct())
            self.__dict__["_struct_array"] = arr
        return arr

    def struct(self) -> kvq_cache:
        c = kvq_cache()
        c.batch, c.kv_heads, c.head_dim, c.max_tokens = (self.batch, self.kv_heads,
                                                         self.head_dim, self.max_tokens)
        c.k = kvq_plane(self.bits, self.group_size, self.k_codes.data_ptr(),
                        self.k_meta.data_ptr() if self.k_meta is not None else None, self.fmt,
                        self.k_axis, kvq_oaken(*(self.k_oaken or (0.0, 0, 0.0, 0))))
        c.v = kvq_plane(self.bits, self.group_size, self.v_codes.data_ptr(),
                        self.v_meta.data_ptr() if self.v_meta is not None else None, self.fmt,
                        KVQ_AXIS_TOKEN, kvq_oaken(*(self.v_oaken or (0.0, 0, 0.0, 0))))
        c.seq_lens = self.seq_lens.data_ptr()
        return c


def alloc_workspace(segs, q_heads: int, max_len_hint: int = 0, device="cuda") -> torch.Tensor:
    """A zeroed workspace tensor for kvq_decode_attention (256-byte aligned)."""
    n = kvq_decode_workspace_bytes(segs, q_heads, max_len_hint)
    return torch.zeros((n + 255) // 256 * 64, dtype=torch.float32, device=device)


def workspace_error_word(workspace: torch.Tensor) -> int:
    """The sticky device error word at the start of a decode workspace."""
    return int(workspace[:1].view(torch.int32).item())
