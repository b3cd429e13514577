"""Host-only checks of the C ABI (no GPU needed): the library loads, exports
every entry point declared in include/kvq.h, sizes its buffers by the
pages' KV-size formula, and rejects bad arguments before touching CUDA."""
import ctypes
import json
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kvq():
    from quantized_kv_cache_12_b200 import build
    build.build()
    from quantized_kv_cache_12_b200 import kvq as m
    return m


def declared_functions():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_header_declares_the_three_hot_path_entry_points():
    names = declared_functions()
    for n in ("kvq_quantize_append", "kvq_decode_attention", "kvq_chunk_reorder"):
        assert n in names


def test_library_exports_every_declared_symbol(kvq):
    lib = ctypes.CDLL(kvq.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_binding_has_a_function_per_entry_point(kvq):
    for n in declared_functions():
        assert callable(getattr(kvq, n)), n


def test_version_and_status_strings(kvq):
    assert "sm_100a" in kvq.kvq_version()
    assert kvq.kvq_status_string(0) == "ok"
    assert "workspace" in kvq.kvq_status_string(4)


def test_kv_elements_matches_worked_example(kvq):
    ex = json.load(open(os.path.join(ROOT, "tests", "golden", "kv_size_worked_example.json")))
    n = kvq.kvq_kv_elements(ex["layers"], ex["kv_heads"], ex["head_dim"], ex["seq_len"],
                            ex["batch"])
    assert n == ex["elements"]
    assert kvq.kvq_kv_elements(2**40, 2**40, 1, 1, 1) == 0  # overflow reported as 0


def test_plane_bytes(kvq):
    # per plane: rows * head_dim * bits/8 code bytes + rows * (head_dim/G) * 4 meta bytes
    assert kvq.kvq_plane_bytes(16, 32, 128, 4224, 8, 128) == (16 * 32 * 4224 * 128,
                                                             16 * 32 * 4224 * 4)
    assert kvq.kvq_plane_bytes(1, 8, 128, 131072, 4, 64) == (8 * 131072 * 64, 8 * 131072 * 8)
    assert kvq.kvq_plane_bytes(2, 3, 128, 64, 2, 32) == (2 * 3 * 64 * 32, 2 * 3 * 64 * 16)
    assert kvq.kvq_plane_bytes(1, 1, 128, 64, 16, 0) == (64 * 256, 0)
    # per (sequence, head, token), K plus V: 144 bytes for INT4 G64, 264 for INT8 G128
    c, m = kvq.kvq_plane_bytes(1, 1, 128, 1, 4, 64)
    assert 2 * (c + m) == 144
    c, m = kvq.kvq_plane_bytes(1, 1, 128, 1, 8, 128)
    assert 2 * (c + m) == 264
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_plane_bytes(1, 1, 128, 64, 3, 64)
    assert e.value.status == kvq.KVQ_ERR_UNSUPPORTED
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_plane_bytes(0, 1, 128, 64, 4, 64)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG


def _fake_cache(kvq, bits=4, group=64, max_tokens=256, batch=2, kv_heads=2, head_dim=128):
    c = kvq.kvq_cache()
    c.batch, c.kv_heads, c.head_dim, c.max_tokens = batch, kv_heads, head_dim, max_tokens
    # fake, never-dereferenced 256-aligned addresses: validation must reject
    # or accept without touching memory
    c.k = kvq.kvq_plane(bits, group, 0x10000, 0x20000)
    c.v = kvq.kvq_plane(bits, group, 0x30000, 0x40000)
    c.seq_lens = 0x50000
    return c


def _status(fn, *args):
    try:
        fn(*args)
    except Exception as e:  # KvqError
        return getattr(e, "status", None)
    return 0


def test_quantize_append_rejects_bad_arguments(kvq):
    S = kvq.kvq_quantize_append
    ok_ptr = 0x60000

    import torch

    class T:  # minimal tensor stand-in: only data_ptr() and dtype are used
        dtype = torch.float16

        def __init__(self, p):
            self.p = p

        def data_ptr(self):
            return self.p

    c = _fake_cache(kvq)
    assert _status(S, c, T(0), T(ok_ptr), 1) == kvq.KVQ_ERR_INVALID_ARG       # null k_new
    assert _status(S, c, T(ok_ptr + 4), T(ok_ptr), 1) == kvq.KVQ_ERR_INVALID_ARG  # misaligned
    assert _status(S, c, T(ok_ptr), T(ok_ptr), 0) == kvq.KVQ_ERR_INVALID_ARG  # n_new < 1
    assert _status(S, c, T(ok_ptr), T(ok_ptr), 257) == kvq.KVQ_ERR_CAPACITY
    assert _status(S, _fake_cache(kvq, bits=3), T(ok_ptr), T(ok_ptr), 1) == kvq.KVQ_ERR_UNSUPPORTED
    assert _status(S, _fake_cache(kvq, group=48), T(ok_ptr), T(ok_ptr), 1) == \
        kvq.KVQ_ERR_UNSUPPORTED
    assert _status(S, _fake_cache(kvq, head_dim=64), T(ok_ptr), T(ok_ptr), 1) == \
        kvq.KVQ_ERR_UNSUPPORTED
    assert _status(S, _fake_cache(kvq, max_tokens=100), T(ok_ptr), T(ok_ptr), 1) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert _status(S, _fake_cache(kvq, bits=16), T(ok_ptr), T(ok_ptr), 1) == \
        kvq.KVQ_ERR_UNSUPPORTED  # FP16 planes are written by the reorder, not quantized
    c2 = _fake_cache(kvq)
    c2.v.group_size = 32
    assert _status(S, c2, T(ok_ptr), T(ok_ptr), 1) == kvq.KVQ_ERR_UNSUPPORTED


def test_quantize_append_kv_dtype(kvq):
    """kv_dtype is KVQ_F16 or KVQ_BF16, taken by every format (a per-channel K
    plane goes on to its block check, an Oaken plane to its capacity check
    exactly as with fp16); the binding passes the tensors' dtype and refuses
    mixed or other dtypes before calling.  No call here reaches a launch."""
    import torch
    fake = ctypes.c_void_p(0x60000)

    def st(c, dt, n=1):
        return kvq.lib.kvq_quantize_append((kvq.kvq_cache * 1)(c), fake, fake, dt, n, 1, None)
    assert st(_fake_cache(kvq), 2) == kvq.KVQ_ERR_INVALID_ARG
    assert st(_fake_cache(kvq), -1) == kvq.KVQ_ERR_INVALID_ARG
    assert st(_fake_cache(kvq), kvq.KVQ_BF16, n=0) == kvq.KVQ_ERR_INVALID_ARG
    assert st(_fake_cache(kvq, bits=3), kvq.KVQ_BF16) == kvq.KVQ_ERR_UNSUPPORTED
    c = _fake_cache(kvq, bits=4)
    c.k.axis = kvq.KVQ_AXIS_CHANNEL
    assert st(c, kvq.KVQ_BF16, n=31) == kvq.KVQ_ERR_INVALID_ARG  # off a block boundary
    c = _fake_cache(kvq, bits=4, group=128)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_OAKEN
    c.k.oaken = kvq.kvq_oaken(0.25, 8, 0.5, 5)
    c.v.oaken = kvq.kvq_oaken(0.125, 3, 0.05, 7)
    big = c.max_tokens + 1
    assert st(c, kvq.KVQ_BF16, n=big) == st(c, kvq.KVQ_F16, n=big) == kvq.KVQ_ERR_CAPACITY

    class T:
        def __init__(self, dtype):
            self.dtype = dtype

        def data_ptr(self):
            return 0x60000
    for a, b in ((torch.float16, torch.bfloat16), (torch.float32, torch.float32)):
        with pytest.raises(TypeError):
            kvq.kvq_quantize_append(_fake_cache(kvq), T(a), T(b), 1)


def test_decode_workspace_and_argument_checks(kvq):
    c = _fake_cache(kvq, batch=4, kv_heads=8, max_tokens=8192)
    n1 = kvq.kvq_decode_workspace_bytes(c, 32)
    n2 = kvq.kvq_decode_workspace_bytes(c, 32, max_len_hint=300)
    assert n1 > n2 > 256
    assert (n1 - 256) % 4 == 0
    # q_heads not a multiple of kv_heads; unsupported group ratio; too many rows
    assert _status(kvq.kvq_decode_workspace_bytes, c, 12) == kvq.KVQ_ERR_INVALID_ARG
    assert _status(kvq.kvq_decode_workspace_bytes, c, 24) == kvq.KVQ_ERR_UNSUPPORTED
    c32 = _fake_cache(kvq, group=32, kv_heads=4)
    assert _status(kvq.kvq_decode_workspace_bytes, c32, 32) == kvq.KVQ_ERR_UNSUPPORTED
    assert kvq.kvq_decode_workspace_bytes(c32, 16) > 0

    lib = kvq.lib
    arr = (kvq.kvq_cache * 1)(c)
    fake = ctypes.c_void_p(0x70000)
    st = lib.kvq_decode_attention(arr, 1, fake, 0, 32, ctypes.c_float(0.088), fake, None, 0,
                                  ctypes.c_void_p(0x80000), 16, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
    st = lib.kvq_decode_attention(arr, 1, None, 0, 32, ctypes.c_float(0.088), fake, None, 0,
                                  ctypes.c_void_p(0x80000), n1, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG
    st = lib.kvq_decode_attention(arr, 1, fake, 0, 32, ctypes.c_float(-1.0), fake, None, 0,
                                  ctypes.c_void_p(0x80000), n1, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG
    st = lib.kvq_decode_attention(arr, 1, fake, 0, 32, ctypes.c_float(0.088), fake, None, 0,
                                  ctypes.c_void_p(0x80010), n1, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG  # workspace not 256-byte aligned
    c16 = _fake_cache(kvq, bits=16, batch=4, kv_heads=8, max_tokens=8192)
    arr16 = (kvq.kvq_cache * 1)(c16)
    n16 = kvq.kvq_decode_workspace_bytes(c16, 32)
    st = lib.kvq_decode_attention(arr16, 1, fake, kvq.KVQ_BF16, 32, ctypes.c_float(0.088), fake,
                                  None, 0, ctypes.c_void_p(0x80000), n16, None)
    assert st == kvq.KVQ_ERR_UNSUPPORTED  # bf16 queries with raw fp16 keys


def test_decode_step_rejects_bad_arguments(kvq):
    """kvq_decode_step checks everything on the host before its first launch,
    on both of its paths (one fused launch, or append then attention)."""
    lib = kvq.lib
    fake = ctypes.c_void_p(0x70000)
    ws = ctypes.c_void_p(0x80000)
    for kv_heads, q_heads in ((8, 32), (2, 16)):  # g = 4 (fused), g = 8 with G64 (two launches)
        c = _fake_cache(kvq, batch=4, kv_heads=kv_heads, max_tokens=8192)
        arr = (kvq.kvq_cache * 1)(c)
        n = kvq.kvq_decode_workspace_bytes(c, q_heads)

        def step(k_new, v_new, q, ws_bytes, scale=0.088):
            return lib.kvq_decode_step(arr, k_new, v_new, q, 0, q_heads, ctypes.c_float(scale),
                                       fake, None, 0, ws, ws_bytes, None)
        assert step(None, fake, fake, n) == kvq.KVQ_ERR_INVALID_ARG
        assert step(fake, ctypes.c_void_p(0x70004), fake, n) == kvq.KVQ_ERR_INVALID_ARG
        assert step(fake, fake, None, n) == kvq.KVQ_ERR_INVALID_ARG
        assert step(fake, fake, fake, n, scale=-1.0) == kvq.KVQ_ERR_INVALID_ARG
        assert step(fake, fake, fake, 64) == kvq.KVQ_ERR_WORKSPACE
    c16 = _fake_cache(kvq, bits=16, batch=4, kv_heads=8, max_tokens=8192)
    arr16 = (kvq.kvq_cache * 1)(c16)
    st = lib.kvq_decode_step(arr16, fake, fake, fake, 0, 32, ctypes.c_float(0.088), fake, None, 0,
                             ws, 1 << 30, None)
    assert st == kvq.KVQ_ERR_UNSUPPORTED  # raw fp16 caches take no quantized append


def test_fp8_planes_validated(kvq):
    """KVQ_FMT_FP8_E4M3 needs bits 8 and the same format on K and V; unknown
    formats are rejected; FP8 decode is built for (head_dim / G) * g <= 8."""
    fake = ctypes.c_void_p(0x60000)

    def append_status(c):
        return kvq.lib.kvq_quantize_append((kvq.kvq_cache * 1)(c), fake, fake, kvq.KVQ_F16, 1, 1, None)
    c = _fake_cache(kvq, bits=4)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_FP8_E4M3
    assert append_status(c) == kvq.KVQ_ERR_UNSUPPORTED
    c = _fake_cache(kvq, bits=8)
    c.k.fmt = c.v.fmt = 7
    assert append_status(c) == kvq.KVQ_ERR_INVALID_ARG
    c = _fake_cache(kvq, bits=8)
    c.k.fmt = kvq.KVQ_FMT_FP8_E4M3
    assert append_status(c) == kvq.KVQ_ERR_UNSUPPORTED
    c = _fake_cache(kvq, bits=8, group=64, kv_heads=2)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_FP8_E4M3
    assert kvq.kvq_decode_workspace_bytes(c, 8) > 0   # g = 4: tokens-on-M kernel
    assert _status(kvq.kvq_decode_workspace_bytes, c, 16) == kvq.KVQ_ERR_UNSUPPORTED  # g = 8


def test_e5m2_planes_validated(kvq):
    """KVQ_FMT_FP8_E5M2 needs bits 8 and the same format on K and V; its decode
    is built for the same (G, g) as E4M3."""
    fake = ctypes.c_void_p(0x60000)

    def append_status(c):
        return kvq.lib.kvq_quantize_append((kvq.kvq_cache * 1)(c), fake, fake, kvq.KVQ_F16, 1, 1, None)
    c = _fake_cache(kvq, bits=4)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_FP8_E5M2
    assert append_status(c) == kvq.KVQ_ERR_UNSUPPORTED
    c = _fake_cache(kvq, bits=8)
    c.k.fmt = kvq.KVQ_FMT_FP8_E5M2
    c.v.fmt = kvq.KVQ_FMT_FP8_E4M3
    assert append_status(c) == kvq.KVQ_ERR_UNSUPPORTED
    c = _fake_cache(kvq, bits=8, group=64, kv_heads=2)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_FP8_E5M2
    assert kvq.kvq_decode_workspace_bytes(c, 8) > 0   # g = 4
    assert _status(kvq.kvq_decode_workspace_bytes, c, 16) == kvq.KVQ_ERR_UNSUPPORTED  # g = 8


def test_sym8_planes_validated(kvq):
    """KVQ_FMT_INT8_SYM needs bits 8 and the same format on K and V; its
    decode is built for the same (G, g) as FP8."""
    fake = ctypes.c_void_p(0x60000)

    def append_status(c):
        return kvq.lib.kvq_quantize_append((kvq.kvq_cache * 1)(c), fake, fake, kvq.KVQ_F16, 1, 1, None)
    c = _fake_cache(kvq, bits=2)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_INT8_SYM
    assert append_status(c) == kvq.KVQ_ERR_UNSUPPORTED
    c = _fake_cache(kvq, bits=8)
    c.k.fmt = kvq.KVQ_FMT_INT8_SYM
    c.v.fmt = kvq.KVQ_FMT_INT
    assert append_status(c) == kvq.KVQ_ERR_UNSUPPORTED
    c = _fake_cache(kvq, bits=8, group=128, kv_heads=2)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_INT8_SYM
    assert kvq.kvq_decode_workspace_bytes(c, 16) > 0   # g = 8, G = 128
    c = _fake_cache(kvq, bits=8, group=32, kv_heads=2)
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_INT8_SYM
    assert _status(kvq.kvq_decode_workspace_bytes, c, 8) == kvq.KVQ_ERR_UNSUPPORTED  # 4 x 4


def test_channel_axis_validated(kvq):
    """KVQ_AXIS_CHANNEL is for the K plane of an integer-code cache only; an
    append to it must be whole 32-token blocks; the one-call decode step does
    not take it (single tokens go to an fp16 segment); unknown axes are
    rejected."""
    fake = ctypes.c_void_p(0x60000)

    def append_status(c, n):
        return kvq.lib.kvq_quantize_append((kvq.kvq_cache * 1)(c), fake, fake, kvq.KVQ_F16, n, 1, None)
    c = _fake_cache(kvq, bits=4)
    c.k.axis = kvq.KVQ_AXIS_CHANNEL
    assert append_status(c, 5) == kvq.KVQ_ERR_INVALID_ARG      # not a whole block
    c.k.group_size = 7                                          # not used on that plane
    assert append_status(c, 33) == kvq.KVQ_ERR_INVALID_ARG
    c = _fake_cache(kvq, bits=4)
    c.v.axis = kvq.KVQ_AXIS_CHANNEL
    assert append_status(c, 32) == kvq.KVQ_ERR_UNSUPPORTED     # V stays per token
    c = _fake_cache(kvq, bits=8)
    c.k.axis = kvq.KVQ_AXIS_CHANNEL
    c.k.fmt = c.v.fmt = kvq.KVQ_FMT_FP8_E4M3
    assert append_status(c, 32) == kvq.KVQ_ERR_UNSUPPORTED     # integer codes only
    c = _fake_cache(kvq, bits=4)
    c.k.axis = 3
    assert append_status(c, 32) == kvq.KVQ_ERR_INVALID_ARG
    c = _fake_cache(kvq, bits=4, group=64, kv_heads=2)
    c.k.axis = kvq.KVQ_AXIS_CHANNEL
    ws = ctypes.c_void_p(0x80000)
    st = kvq.lib.kvq_decode_step((kvq.kvq_cache * 1)(c), fake, fake, fake, kvq.KVQ_F16, 8,
                                 ctypes.c_float(0.08), fake, None, 0, ws, 1 << 30, None)
    assert st == kvq.KVQ_ERR_UNSUPPORTED


def test_chunk_entry_points_reject_bad_arguments(kvq):
    lib = kvq.lib
    fake = ctypes.c_void_p(0x10000)
    assert lib.kvq_chunk_assign(None, fake, 8, 1024, 768, 0.6, 0.1, None, fake, None) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_chunk_assign(fake, fake, 8, 5000, 768, 0.6, 0.1, None, fake, None) == \
        kvq.KVQ_ERR_INVALID_ARG
    # the staged embedding copies need 16-byte rows and fit emb_dim <= 4096
    assert lib.kvq_chunk_assign(fake, fake, 8, 1024, 770, 0.6, 0.1, None, fake, None) == \
        kvq.KVQ_ERR_UNSUPPORTED
    assert lib.kvq_chunk_assign(fake, fake, 8, 1024, 4100, 0.6, 0.1, None, fake, None) == \
        kvq.KVQ_ERR_UNSUPPORTED
    assert lib.kvq_chunk_assign(ctypes.c_void_p(0x10004), fake, 8, 1024, 768, 0.6, 0.1, None,
                                fake, None) == kvq.KVQ_ERR_INVALID_ARG
    segs = (kvq.kvq_cache * 3)(_fake_cache(kvq, bits=16, max_tokens=1024),
                               _fake_cache(kvq, bits=4, group=32, max_tokens=1024),
                               _fake_cache(kvq, bits=2, group=32, max_tokens=1024))
    # chunk size not a multiple of 16; context not a multiple of the chunk size
    assert lib.kvq_chunk_reorder(segs, fake, fake, 1024, 24, fake, fake, None) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_chunk_reorder(segs, fake, fake, 1000, 32, fake, fake, None) == \
        kvq.KVQ_ERR_INVALID_ARG
    assert lib.kvq_chunk_reorder(segs, fake, fake, 2048, 32, fake, fake, None) == \
        kvq.KVQ_ERR_CAPACITY
    wrong = (kvq.kvq_cache * 3)(segs[1], segs[0], segs[2])
    assert lib.kvq_chunk_reorder(wrong, fake, fake, 1024, 32, fake, fake, None) == \
        kvq.KVQ_ERR_INVALID_ARG


def test_oaken_planes_validated(kvq):
    """KVQ_FMT_OAKEN needs bits 4, group_size = head_dim, the token axis, the
    same format on K and V, and offline parameters in range (inner_scale a
    positive fp16 value, inner_zero in [0, 15], outer_scale positive and
    finite, outer_bits 5 to 7); its decode is built for g = 1, 2, 4, 8."""
    fake = ctypes.c_void_p(0x60000)

    def oaken_cache(kp=(0.25, 8, 0.5, 5), vp=(0.125, 3, 0.05, 7), bits=4, group=128, kv_heads=2):
        c = _fake_cache(kvq, bits=bits, group=group, kv_heads=kv_heads)
        c.k.fmt = c.v.fmt = kvq.KVQ_FMT_OAKEN
        c.k.oaken = kvq.kvq_oaken(*kp)
        c.v.oaken = kvq.kvq_oaken(*vp)
        return c

    def append_status(c):
        return kvq.lib.kvq_quantize_append((kvq.kvq_cache * 1)(c), fake, fake, kvq.KVQ_F16, 1, 1, None)

    for g in (1, 2, 4, 8):
        assert kvq.kvq_decode_workspace_bytes(oaken_cache(), 2 * g) > 0
    assert _status(kvq.kvq_decode_workspace_bytes, oaken_cache(), 6) == kvq.KVQ_ERR_UNSUPPORTED
    assert append_status(oaken_cache(bits=8)) == kvq.KVQ_ERR_UNSUPPORTED
    assert append_status(oaken_cache(group=64)) == kvq.KVQ_ERR_UNSUPPORTED
    for bad in [(0.3, 8, 0.5, 5),            # not an fp16 value
                (0.0, 8, 0.5, 5), (float("nan"), 8, 0.5, 5),
                (0.25, -1, 0.5, 5), (0.25, 16, 0.5, 5),
                (0.25, 8, 0.0, 5), (0.25, 8, float("inf"), 5),
                (0.25, 8, 0.5, 4), (0.25, 8, 0.5, 8)]:
        assert append_status(oaken_cache(kp=bad)) == kvq.KVQ_ERR_INVALID_ARG, bad
        assert append_status(oaken_cache(vp=bad)) == kvq.KVQ_ERR_INVALID_ARG, bad
    c = oaken_cache()
    c.k.meta = None
    assert append_status(c) == kvq.KVQ_ERR_INVALID_ARG
    c = oaken_cache()
    c.v.fmt = kvq.KVQ_FMT_INT
    c.v.bits = 4
    assert append_status(c) in (kvq.KVQ_ERR_UNSUPPORTED, kvq.KVQ_ERR_INVALID_ARG)
    c = oaken_cache()
    c.k.axis = kvq.KVQ_AXIS_CHANNEL
    assert append_status(c) == kvq.KVQ_ERR_UNSUPPORTED


def test_struct_layout_matches_the_header(kvq, tmp_path):
    """The binding's ctypes structs have the header's sizes and offsets (a C
    program built from include/kvq.h prints them)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    src = tmp_path / "layout.c"
    src.write_text('#include <stdio.h>\n#include "kvq.h"\nint main(void) {\n'
                   ' printf("%zu %zu %zu %zu %zu\\n", sizeof(kvq_plane), sizeof(kvq_cache),'
                   ' offsetof(kvq_plane, oaken), offsetof(kvq_cache, v),'
                   ' offsetof(kvq_cache, seq_lens));\n return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                   check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    want = [ctypes.sizeof(kvq.kvq_plane), ctypes.sizeof(kvq.kvq_cache),
            kvq.kvq_plane.oaken.offset, kvq.kvq_cache.v.offset, kvq.kvq_cache.seq_lens.offset]
    assert got == want


def _plan_parts(kvq, B, H, Hq, max_tokens, hint, bits=4, group=64, fmt=0):
    """Partials per (sequence, query head) of a split plan, read back through
    the workspace size: header, per-sequence counters, then (m, l) and o of
    every partial."""
    c = _fake_cache(kvq, bits=bits, group=group, max_tokens=max_tokens, batch=B, kv_heads=H)
    c.k.fmt = c.v.fmt = fmt
    if fmt == kvq.KVQ_FMT_OAKEN:
        c.k.oaken = c.v.oaken = kvq.kvq_oaken(0.25, 8, 0.5, 5)
    ws = kvq.kvq_decode_workspace_bytes(c, Hq, hint)
    r256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    return next(p for p in range(1, 4096)
                if 256 + r256(B * 4) + r256(B * Hq * p * 8) + r256(B * Hq * p * 128 * 4) == ws)


def test_split_plan_per_workload(kvq):
    """The host split plan at the benchmark's shapes (148 SMs on a host
    without a device), as partials per (sequence, query head).  The plan
    minimises the busiest SM's time: u = ceil(units / SMs) units in rounds of
    up to C (the format's CTAs per SM), a round of c < 3 units at c/3 of the
    SM's rate, each unit (tokens rounded up to 32) + 300 tokens of fixed cost,
    plus 600 for the merge kernel when there is more than one split (the
    costs below leave it out: it is the same for every n > 1):
      Llama-3 GQA INT4 (256 pairs, L 8292, C 4): 4 splits, u = 7, rounds 4 + 3,
        7 x (2080 + 300) = 16660; 2 splits cost 4 x 4460 = 17840, 6 splits
        11 x 1708 = 18788, 5 splits (4 + 4 + a lone unit) 11 x 1964 = 21604.
      half that batch (128 pairs): 3 splits, u = 3, 3 x 3084 = 9252 against
        4 x 2380 = 9520 for 4.
      long context (8 pairs, L 131328): 55 splits, u = 3, 3 x (2400 + 300) =
        8100 against 4 x (1792 + 300) = 8368 for 74.
      Llama-2 MHA INT8 (512 pairs, L 4196, C 3): 4 splits, u = 14, rounds
        3 + 3 + 3 + 3 + 2 (at 2/3 rate), 15 x 1356 = 20340 against
        12 x 1708 = 20496 for 3.
      Oaken codec (256 pairs, L 8192, C 3): 5 splits, u = 9, 9 x 1964 =
        17676 against 6 x 3052 = 18312 for 3."""
    parts = lambda *a, **k: _plan_parts(kvq, *a, **k)  # noqa: E731
    assert parts(32, 8, 32, 8320, 8292) == 4
    assert parts(16, 8, 32, 8320, 8292) == 3
    assert parts(1, 8, 32, 131392, 131328) == 55
    assert parts(16, 32, 32, 4224, 4196, bits=8, group=128) == 4
    assert parts(32, 8, 32, 8320, 8192, group=128, fmt=kvq.KVQ_FMT_OAKEN) == 5
    # Tiny (1 pair, 256 tokens): one split, 3 x (256 + 300) = 1668 with the
    # lone unit at a third of the SM's rate, against 3 x (128 + 300) + 600 =
    # 1884 for two splits and their merge
    assert parts(1, 1, 1, 256, 256) == 1


def test_split_plan_follows_the_sm_count(tmp_path):
    """The plan reads the device's SM count; KVQ_NUM_SMS overrides it (read
    once per process, so the check runs in a child process).  With 74 SMs,
    worked by hand from the same cost: Llama-3 GQA INT4 (256 pairs, 4 CTAs
    per SM) takes 2 splits -- u = 7, rounds 4 + 3, 7 x 4460 = 31220, against
    4 x 8620 = 34480 for one split and (12 + 3) x 2380 = 35700 for four --
    and the long context (8 pairs) takes 37 splits -- u = 4, 4 x 3852 =
    15408, against (4 + 3) x 2700 = 18900 for 55."""
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from quantized_kv_cache_12_b200 import kvq\n"
        "import tests.test_abi_host as t\n"
        "print(t._plan_parts(kvq, 32, 8, 32, 8320, 8292), "
        "t._plan_parts(kvq, 1, 8, 32, 131392, 131328))\n" % ROOT)
    env = dict(os.environ, KVQ_NUM_SMS="74")
    out = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, check=True,
                         capture_output=True, text=True).stdout.split()
    assert out == ["2", "37"]
