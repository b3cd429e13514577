"""CPU oracle for the quantized-KV-cache hot path (test infrastructure).

TEST INFRASTRUCTURE ONLY.  The test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers allowed; the product
library never imports, links or runs anything here, and this package never
imports the product library.  The arithmetic lives in ``kvq_oracle.c`` (plain
C, built with ``-ffp-contract=off`` and no fast-math); this module only
marshals numpy arrays and loops over (sequence, KV head) pairs.

Every function cites the page passage it follows; the readings taken where
the pages are silent are listed at the top of ``kvq_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-fPIC", "-shared"]

_lib = None


def build(force: bool = False) -> str:
    """Compile ``kvq_oracle.c`` into ``libkvq_oracle.so`` with gcc."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, u64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
        lib.kvqo_f32_to_f16.argtypes = [ctypes.c_float]
        lib.kvqo_f32_to_f16.restype = ctypes.c_uint16
        lib.kvqo_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.kvqo_f16_to_f32.restype = ctypes.c_float
        lib.kvqo_f32_to_f16_up.argtypes = [ctypes.c_float]
        lib.kvqo_f32_to_f16_up.restype = ctypes.c_uint16
        lib.kvqo_f32_to_f16_array.argtypes = [P, i64, P]
        lib.kvqo_f16_to_f32_array.argtypes = [P, i64, P]
        lib.kvqo_quantize_group.argtypes = [P, i32, i32, P, P, P]
        lib.kvqo_quantize_rows.argtypes = [P, i64, i32, i32, i32, P, P]
        lib.kvqo_quantize_rows_any.argtypes = [P, i32, i64, i32, i32, i32, i32, P, P]
        lib.kvqo_dequantize_rows.argtypes = [P, P, i64, i32, i32, i32, P]
        lib.kvqo_attention.argtypes = [P, i32, P, P, i64, i32, f64, P, P]
        lib.kvqo_attention_blocks.argtypes = [P, i32, P, P, i32, f64, P, i32, P, P]
        lib.kvqo_attention_packed.argtypes = [P, i32, i32, P, P, i32, P, P, i32, i32,
                                              i64, i32, f64, P, P]
        lib.kvqo_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.kvqo_e4m3_to_f64.restype = f64
        lib.kvqo_f32_to_e4m3.argtypes = [ctypes.c_float]
        lib.kvqo_f32_to_e4m3.restype = ctypes.c_uint8
        lib.kvqo_quantize_group_fp8.argtypes = [P, i32, P, P]
        lib.kvqo_quantize_rows_fp8.argtypes = [P, i64, i32, i32, P, P]
        lib.kvqo_quantize_group_sym8.argtypes = [P, i32, P, P]
        lib.kvqo_e5m2_to_f64.restype = ctypes.c_double
        lib.kvqo_e5m2_to_f64.argtypes = [ctypes.c_uint8]
        lib.kvqo_f32_to_e5m2.restype = ctypes.c_uint8
        lib.kvqo_f32_to_e5m2.argtypes = [ctypes.c_float]
        lib.kvqo_quantize_group_e5m2.argtypes = [P, i32, P, P]
        lib.kvqo_quantize_rows_e5m2.argtypes = [P, i64, i32, i32, P, P]
        lib.kvqo_quantize_block_channels.argtypes = [P, i32, i32, i32, P, P]
        lib.kvqo_quantize_block_channels_in.argtypes = [P, i32, i32, i32, i32, P, P]
        lib.kvqo_dequantize_block_channels.argtypes = [P, P, i32, i32, i32, P]
        lib.kvqo_quantize_rows_sym8.argtypes = [P, i64, i32, i32, P, P]
        lib.kvqo_dequantize_rows_fmt.argtypes = [P, P, i64, i32, i32, i32, i32, P]
        lib.kvqo_attention_packed_fmt.argtypes = [P, i32, i32, P, P, i32, P, P, i32, i32, i32,
                                                  i64, i32, f64, P, P]
        lib.kvqo_chunk_assign.argtypes = [P, P, i32, i32, f64, f64, P, P]
        lib.kvqo_chunk_partition.argtypes = [P, i32, P, P]
        f32 = ctypes.c_float
        lib.kvqo_oaken_quantize_rows.argtypes = [P, i64, i32, f32, i32, f32, i32, P, P]
        lib.kvqo_oaken_quantize_rows_in.argtypes = [P, i32, i64, i32, f32, i32, f32, i32, P,
                                                    P]
        lib.kvqo_oaken_dequantize_rows.argtypes = [P, P, i64, i32, f32, i32, f32, P]
        lib.kvqo_kv_elements.argtypes = [u64, u64, u64, u64, u64]
        lib.kvqo_kv_elements.restype = u64
        _lib = lib
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------
# binary16 codec (IEEE 754 binary16, round to nearest even)
# --------------------------------------------------------------------------

def f32_to_f16_bits(x) -> np.ndarray:
    """fp32 values -> binary16 bit patterns (uint16), ties to even."""
    lib = _load()
    x = _c(x, np.float32)
    out = np.zeros(x.shape, np.uint16)
    lib.kvqo_f32_to_f16_array(_p(x), x.size, _p(out))
    return out


def f32_to_f16_bits_up(x) -> np.ndarray:
    """positive fp32 values -> smallest binary16 value not below them."""
    lib = _load()
    x = _c(x, np.float32).ravel()
    return np.array([lib.kvqo_f32_to_f16_up(float(v)) for v in x], np.uint16)


def f16_bits_to_f32(h) -> np.ndarray:
    lib = _load()
    h = _c(h, np.uint16)
    out = np.zeros(h.shape, np.float32)
    lib.kvqo_f16_to_f32_array(_p(h), h.size, _p(out))
    return out


# --------------------------------------------------------------------------
# group quantization (Cocktail page 3.2.2; static-quantization page 2.1)
# --------------------------------------------------------------------------

def quantize_group(x16, bits: int):
    """One group of fp16 bit patterns -> (codes uint8[G], s16, z16)."""
    lib = _load()
    x16 = _c(x16, np.uint16)
    G = x16.size
    code = np.zeros(G, np.uint8)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    lib.kvqo_quantize_group(_p(x16), G, bits, _p(code), _p(s), _p(z))
    return code, int(s[0]), int(z[0])


# code formats of the C functions' `fmt` argument
FMT_CODES = {"int": 0, "fp8": 1, "sym8": 2, "e5m2": 3}


def quantize_rows(x16, group: int, bits: int, fmt: str = "int", in_dtype: str = "f16"):
    """Token rows [N, D] of fp16 bit patterns -> (codes [N, D*bits/8] uint8,
    meta [N, D/G, 2] uint16 holding the (scale, zero) fp16 patterns).
    fmt "fp8": E4M3 codes (bits 8) with zero point 0 (KV-cache page, FP8);
    fmt "sym8": symmetric INT8, two's complement codes (bits 8) with zero
    point 0 (KV-cache page, INT8 item); fmt "e5m2": E5M2 codes (bits 8) with
    zero point 0 (KV-cache page, FP8).  in_dtype "bf16": the rows are
    bfloat16 bit patterns, read exactly into fp32 like the fp16 ones (the
    same arithmetic follows)."""
    lib = _load()
    x16 = _c(x16, np.uint16)
    N, D = x16.shape
    codes = np.zeros((N, D * bits // 8), np.uint8)
    ng = D // group if bits != 16 else 1
    meta = np.zeros((N, ng, 2), np.uint16)
    if in_dtype == "bf16":
        assert bits != 16, "raw rows hold fp16 values"
        lib.kvqo_quantize_rows_any(_p(x16), 1, N, D, group, bits, FMT_CODES[fmt], _p(codes),
                                   _p(meta))
        return codes, meta
    assert in_dtype == "f16", in_dtype
    if fmt == "fp8":
        assert bits == 8
        lib.kvqo_quantize_rows_fp8(_p(x16), N, D, group, _p(codes), _p(meta))
    elif fmt == "sym8":
        assert bits == 8
        lib.kvqo_quantize_rows_sym8(_p(x16), N, D, group, _p(codes), _p(meta))
    elif fmt == "e5m2":
        assert bits == 8
        lib.kvqo_quantize_rows_e5m2(_p(x16), N, D, group, _p(codes), _p(meta))
    else:
        assert fmt == "int", fmt
        lib.kvqo_quantize_rows(_p(x16), N, D, group, bits, _p(codes), _p(meta))
    return codes, meta


def dequantize_rows(codes, meta, D: int, group: int, bits: int, fmt: str = "int") -> np.ndarray:
    """Packed rows -> fp64 [N, D]: x_hat = (c - z) * s, e4m3(c) * s for
    fmt "fp8", int8(c) * s for fmt "sym8", e5m2(c) * s for fmt "e5m2" (all
    exact in fp64)."""
    lib = _load()
    codes = _c(codes, np.uint8)
    N = codes.shape[0]
    meta = _c(meta if meta is not None else np.zeros((N, 1, 2), np.uint16), np.uint16)
    out = np.zeros((N, D), np.float64)
    lib.kvqo_dequantize_rows_fmt(_p(codes), _p(meta), N, D, group if bits != 16 else D, bits,
                                 FMT_CODES[fmt], _p(out))
    return out


# --------------------------------------------------------------------------
# FP8 E4M3 (KV-cache page, FP8 KV cache; reading R14 in kvq_oracle.c)
# --------------------------------------------------------------------------

def e4m3_to_f64(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> fp64 values (NaN for S.1111.111)."""
    lib = _load()
    c = _c(codes, np.uint8).ravel()
    return np.array([lib.kvqo_e4m3_to_f64(int(v)) for v in c], np.float64).reshape(
        np.shape(codes))


def f32_to_e4m3(x) -> np.ndarray:
    """fp32 values -> nearest E4M3 codes, ties to even, saturating at 448."""
    lib = _load()
    x = _c(x, np.float32)
    return np.array([lib.kvqo_f32_to_e4m3(float(v)) for v in x.ravel()], np.uint8).reshape(
        x.shape)


def quantize_group_fp8(x16):
    """One group of fp16 bit patterns -> (E4M3 codes uint8[G], s16)."""
    lib = _load()
    x16 = _c(x16, np.uint16)
    code = np.zeros(x16.size, np.uint8)
    s = np.zeros(1, np.uint16)
    lib.kvqo_quantize_group_fp8(_p(x16), x16.size, _p(code), _p(s))
    return code, int(s[0])


def e5m2_to_f64(codes) -> np.ndarray:
    """E5M2 codes (uint8) -> fp64 values (infinities and NaN in E = 31)."""
    lib = _load()
    c = _c(codes, np.uint8).ravel()
    return np.array([lib.kvqo_e5m2_to_f64(int(v)) for v in c], np.float64).reshape(
        np.shape(codes))


def f32_to_e5m2(x) -> np.ndarray:
    """fp32 values -> nearest E5M2 codes, ties to even, saturating at 57344."""
    lib = _load()
    x = _c(x, np.float32)
    return np.array([lib.kvqo_f32_to_e5m2(float(v)) for v in x.ravel()], np.uint8).reshape(
        x.shape)


def quantize_group_e5m2(x16):
    """One group of fp16 bit patterns -> (E5M2 codes uint8[G], s16)."""
    lib = _load()
    x16 = _c(x16, np.uint16)
    code = np.zeros(x16.size, np.uint8)
    s = np.zeros(1, np.uint16)
    lib.kvqo_quantize_group_e5m2(_p(x16), x16.size, _p(code), _p(s))
    return code, int(s[0])


# --------------------------------------------------------------------------
# Symmetric INT8 (KV-cache page, INT8 item; reading R15 in kvq_oracle.c)
# --------------------------------------------------------------------------

def quantize_group_sym8(x16):
    """One group of fp16 bit patterns -> (int8 codes as uint8[G] two's
    complement bytes, s16)."""
    lib = _load()
    x16 = _c(x16, np.uint16)
    code = np.zeros(x16.size, np.uint8)
    s = np.zeros(1, np.uint16)
    lib.kvqo_quantize_group_sym8(_p(x16), x16.size, _p(code), _p(s))
    return code, int(s[0])


# --------------------------------------------------------------------------
# Per-channel K (KV-cache page, INT8 item: the Key quantized per channel;
# reading R16 in kvq_oracle.c): blocks of KPC_BLOCK tokens, one (s, z) per
# channel and block
# --------------------------------------------------------------------------

KPC_BLOCK = 32


def quantize_block_channels(x16, bits: int, in_dtype: str = "f16"):
    """One block of token rows [T, D] (fp16 patterns, or bfloat16 ones with
    in_dtype "bf16", read exactly into fp32 like the fp16 ones) ->
    (codes [T, D*bits/8], meta [D, 2] uint16 (s, z) per channel)."""
    assert in_dtype in ("f16", "bf16"), in_dtype
    lib = _load()
    x16 = _c(x16, np.uint16)
    T, D = x16.shape
    codes = np.zeros((T, D * bits // 8), np.uint8)
    meta = np.zeros((D, 2), np.uint16)
    lib.kvqo_quantize_block_channels_in(_p(x16), int(in_dtype == "bf16"), T, D, bits, _p(codes),
                                        _p(meta))
    return codes, meta


def dequantize_block_channels(codes, meta, D: int, bits: int) -> np.ndarray:
    """One block's codes [T, D*bits/8] and meta [D, 2] -> fp64 [T, D]."""
    lib = _load()
    codes = _c(codes, np.uint8)
    meta = _c(meta, np.uint16)
    T = codes.shape[0]
    out = np.zeros((T, D), np.float64)
    lib.kvqo_dequantize_block_channels(_p(codes), _p(meta), T, D, bits, _p(out))
    return out


def quantize_cache_channels(x16, bits: int, in_dtype: str = "f16"):
    """x16 [..., T, D] (fp16, or with in_dtype "bf16" bfloat16, patterns) with
    T a multiple of KPC_BLOCK -> codes [..., T, D*bits/8], meta
    [..., T / KPC_BLOCK, D, 2]."""
    x16 = _c(x16, np.uint16)
    lead, (T, D) = x16.shape[:-2], x16.shape[-2:]
    assert T % KPC_BLOCK == 0, T
    flat = x16.reshape(-1, T // KPC_BLOCK, KPC_BLOCK, D)
    codes = np.zeros((flat.shape[0], T, D * bits // 8), np.uint8)
    meta = np.zeros((flat.shape[0], T // KPC_BLOCK, D, 2), np.uint16)
    for i in range(flat.shape[0]):
        for blk in range(T // KPC_BLOCK):
            c, m = quantize_block_channels(flat[i, blk], bits, in_dtype)
            codes[i, blk * KPC_BLOCK:(blk + 1) * KPC_BLOCK] = c
            meta[i, blk] = m
    return (codes.reshape(*lead, T, D * bits // 8),
            meta.reshape(*lead, T // KPC_BLOCK, D, 2))


def dequantize_channels(codes, meta, L: int, D: int, bits: int) -> np.ndarray:
    """The first L tokens (L a multiple of KPC_BLOCK) of one (sequence, KV
    head) of a per-channel K plane -> fp64 [L, D]."""
    assert L % KPC_BLOCK == 0, L
    out = np.zeros((L, D), np.float64)
    for blk in range(L // KPC_BLOCK):
        r = slice(blk * KPC_BLOCK, (blk + 1) * KPC_BLOCK)
        out[r] = dequantize_block_channels(codes[r], meta[blk], D, bits)
    return out


# --------------------------------------------------------------------------
# Oaken group-shift codec ("大模型KV缓存量化技术：原理、优化与实践" page,
# sections 3.1, 3.2.1, 3.2.2; reading R18 in kvq_oracle.c)
# --------------------------------------------------------------------------

OAKEN_SLOTS = 16


def oaken_quantize_rows(x16, s_in: float, z_in: int, s_out: float, outer_bits: int,
                        in_dtype: str = "f16"):
    """Token rows [N, D] (fp16 patterns, or bfloat16 ones with in_dtype "bf16",
    read exactly into fp32) -> (codes [N, D/2] uint8, slots [N, OAKEN_SLOTS]
    uint16) with the plane's offline parameters."""
    assert in_dtype in ("f16", "bf16"), in_dtype
    lib = _load()
    x16 = _c(x16, np.uint16)
    N, D = x16.shape
    codes = np.zeros((N, D // 2), np.uint8)
    slots = np.zeros((N, OAKEN_SLOTS), np.uint16)
    lib.kvqo_oaken_quantize_rows_in(_p(x16), int(in_dtype == "bf16"), N, D, float(s_in),
                                    int(z_in), float(s_out), int(outer_bits), _p(codes),
                                    _p(slots))
    return codes, slots


def oaken_dequantize_rows(codes, slots, D: int, s_in: float, z_in: int, s_out: float):
    """codes [N, D/2], slots [N, OAKEN_SLOTS] -> fp64 [N, D]."""
    lib = _load()
    codes = _c(codes, np.uint8)
    slots = _c(slots, np.uint16)
    N = codes.shape[0]
    out = np.zeros((N, D), np.float64)
    lib.kvqo_oaken_dequantize_rows(_p(codes), _p(slots), N, D, float(s_in), int(z_in),
                                   float(s_out), _p(out))
    return out


def oaken_quantize_cache(x16, params, in_dtype: str = "f16"):
    """x16 [..., T, D] (fp16, or with in_dtype "bf16" bfloat16, patterns) ->
    codes [..., T, D/2], slots [..., T, OAKEN_SLOTS]; params = (s_in, z_in,
    s_out, outer_bits)."""
    x16 = _c(x16, np.uint16)
    lead, D = x16.shape[:-1], x16.shape[-1]
    codes, slots = oaken_quantize_rows(x16.reshape(-1, D), *params, in_dtype=in_dtype)
    return codes.reshape(*lead, D // 2), slots.reshape(*lead, OAKEN_SLOTS)


# --------------------------------------------------------------------------
# fp64 attention (score definition: KVO-LLM page 3.2; chunked + merge:
# Cocktail page 3.2.3)
# --------------------------------------------------------------------------

def attention(q, K, V, scale: float):
    """q [g, D], K/V [L, D] fp64 -> (o [g, D], lse [g]) in fp64."""
    lib = _load()
    q = _c(q, np.float64)
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    g, D = q.shape
    L = K.shape[0]
    o = np.zeros((g, D), np.float64)
    lse = np.zeros(g, np.float64)
    lib.kvqo_attention(_p(q), g, _p(K), _p(V), L, D, float(scale), _p(o), _p(lse))
    return o, lse


def attention_blocks(q, K, V, scale: float, bounds: Sequence[int]):
    """Block-wise attention merged by log-sum-exp; bounds = [0, ..., L]."""
    lib = _load()
    q = _c(q, np.float64)
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    g, D = q.shape
    b = _c(bounds, np.int64)
    o = np.zeros((g, D), np.float64)
    lse = np.zeros(g, np.float64)
    lib.kvqo_attention_blocks(_p(q), g, _p(K), _p(V), D, float(scale), _p(b), b.size - 1,
                              _p(o), _p(lse))
    return o, lse


def attention_packed(q16, q_is_bf16: bool, k_codes, k_meta, k_bits: int, v_codes, v_meta,
                     v_bits: int, group: int, L: int, scale: float, fmt: str = "int"):
    """Attention of g query heads over one packed (sequence, KV head) cache
    (fmt "fp8": E4M3 codes for K and V; "sym8": symmetric INT8; "e5m2": E5M2)."""
    lib = _load()
    q16 = _c(q16, np.uint16)
    g, D = q16.shape
    kc = _c(k_codes, np.uint8)
    vc = _c(v_codes, np.uint8)
    km = _c(k_meta, np.uint16) if k_bits != 16 else np.zeros(1, np.uint16)
    vm = _c(v_meta, np.uint16) if v_bits != 16 else np.zeros(1, np.uint16)
    o = np.zeros((g, D), np.float64)
    lse = np.zeros(g, np.float64)
    lib.kvqo_attention_packed_fmt(_p(q16), int(bool(q_is_bf16)), g, _p(kc), _p(km), k_bits,
                                  _p(vc), _p(vm), v_bits, FMT_CODES[fmt], group, L, D,
                                  float(scale), _p(o), _p(lse))
    return o, lse


# --------------------------------------------------------------------------
# Cocktail chunk search and reorder (Cocktail page 3.1.1, 3.1.2)
# --------------------------------------------------------------------------

def chunk_assign(emb, qemb, alpha: float, beta: float):
    """emb [n, E] fp32, qemb [E] fp32 -> (sim fp64 [n], class uint8 [n])."""
    lib = _load()
    emb = _c(emb, np.float32)
    qemb = _c(qemb, np.float32)
    n, E = emb.shape
    sim = np.zeros(n, np.float64)
    bits = np.zeros(n, np.uint8)
    lib.kvqo_chunk_assign(_p(emb), _p(qemb), n, E, float(alpha), float(beta), _p(sim),
                          _p(bits))
    return sim, bits


def chunk_partition(bits):
    """class per chunk -> (perm int32 [n], counts int32 [3] for FP16/INT4/INT2)."""
    lib = _load()
    bits = _c(bits, np.uint8)
    perm = np.zeros(bits.size, np.int32)
    counts = np.zeros(3, np.int32)
    lib.kvqo_chunk_partition(_p(bits), bits.size, _p(perm), _p(counts))
    return perm, counts


def kv_elements(layers: int, kv_heads: int, head_dim: int, seq_len: int, batch: int) -> int:
    """2 * layers * kv_heads * head_dim * seq_len * batch (KV-cache size page)."""
    return int(_load().kvqo_kv_elements(layers, kv_heads, head_dim, seq_len, batch))


# --------------------------------------------------------------------------
# Whole-cache helpers built from the functions above
# --------------------------------------------------------------------------

def quantize_cache(x16, group: int, bits: int, fmt: str = "int", in_dtype: str = "f16"):
    """x16 [..., T, D] fp16 (or, with in_dtype "bf16", bfloat16) patterns ->
    codes [..., T, D*bits/8], meta [..., T, D/G, 2]."""
    x16 = _c(x16, np.uint16)
    lead = x16.shape[:-1]
    D = x16.shape[-1]
    codes, meta = quantize_rows(x16.reshape(-1, D), group, bits, fmt, in_dtype)
    return (codes.reshape(*lead, D * bits // 8),
            meta.reshape(*lead, meta.shape[-2], 2))


def decode_attention(q16, q_is_bf16: bool, segments, seq_lens_per_seg, scale: float,
                     pairs=None):
    """Decode attention of every query head over one or more packed segments.

    q16: [B, Hq, D] fp16/bf16 patterns.  segments: list of dicts with numpy
    arrays ``k_codes``/``v_codes`` [B, Hkv, T, row_bytes], ``k_meta``/``v_meta``
    [B, Hkv, T, D/G, 2] (None for bits 16), ``bits``, ``group`` and optionally
    ``fmt`` ("int", the default, "fp8", "sym8", "e5m2" or "oaken") and ``k_channels``
    (True: K is per-channel, ``k_meta`` [B, Hkv, T / KPC_BLOCK, D, 2], lengths
    multiples of KPC_BLOCK).  An "oaken" segment holds the outlier slots
    [B, Hkv, T, OAKEN_SLOTS] in ``k_meta``/``v_meta`` and the planes' offline
    parameters (s_in, z_in, s_out, outer_bits) in ``k_oaken``/``v_oaken``.
    seq_lens_per_seg: list of int arrays [B].  The segments of a sequence are
    concatenated in token order (attention does not depend on the order).
    pairs: optional list of (b, kv_head) to evaluate; others stay NaN.
    Returns (o [B, Hq, D] fp64, lse [B, Hq] fp64).
    """
    q16 = _c(q16, np.uint16)
    B, Hq, D = q16.shape
    Hkv = segments[0]["k_codes"].shape[1]
    g = Hq // Hkv
    o = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in pairs:
        Ks, Vs = [], []
        for seg, lens in zip(segments, seq_lens_per_seg):
            L = int(lens[b])
            bits, G = seg["bits"], seg["group"]
            vm = seg["v_meta"][b, h, :L] if bits != 16 else None
            fmt = seg.get("fmt", "int")
            if fmt == "oaken":
                kp, vp = seg["k_oaken"], seg["v_oaken"]
                Ks.append(oaken_dequantize_rows(seg["k_codes"][b, h, :L], seg["k_meta"][b, h, :L],
                                                D, kp[0], kp[1], kp[2]))
                Vs.append(oaken_dequantize_rows(seg["v_codes"][b, h, :L], seg["v_meta"][b, h, :L],
                                                D, vp[0], vp[1], vp[2]))
                continue
            if seg.get("k_channels", False):
                Ks.append(dequantize_channels(seg["k_codes"][b, h, :L], seg["k_meta"][b, h], L,
                                              D, bits))
            else:
                km = seg["k_meta"][b, h, :L] if bits != 16 else None
                Ks.append(dequantize_rows(seg["k_codes"][b, h, :L], km, D, G, bits, fmt))
            Vs.append(dequantize_rows(seg["v_codes"][b, h, :L], vm, D, G, bits, fmt))
        K = np.concatenate(Ks, 0)
        V = np.concatenate(Vs, 0)
        qh = q16[b, h * g:(h + 1) * g]
        qd = (bf16_bits_to_f64(qh) if q_is_bf16 else f16_bits_to_f32(qh).astype(np.float64)
              ).reshape(g, D)
        ob, lb = attention(qd, K, V, scale)
        o[b, h * g:(h + 1) * g] = ob
        lse[b, h * g:(h + 1) * g] = lb
    return o, lse


def bf16_bits_to_f64(h) -> np.ndarray:
    """bfloat16 bit patterns -> fp64 (exact: the pattern is the top half of fp32)."""
    h = _c(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
