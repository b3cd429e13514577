"""Host-side pieces of bench.py (no GPU): the algorithmic bytes behind the
roofline's `achieved` figure, checked against the per-head-token byte counts
of the layout (4-bit codes of 128 dims are 64 bytes, a (scale, zero) pair is
4 bytes, an Oaken row adds 16 two-byte slots), and the kernel-source hash
that invalidates recorded traffic."""
import os

import bench


def test_bytes_per_head_token():
    f = bench.bytes_per_head_token
    assert f(8, 128) == 2 * (128 + 4)            # INT8 G128
    assert f(4, 64) == 2 * (64 + 8)              # INT4 G64
    assert f(4, 32) == 2 * (64 + 16)             # INT4 G32
    assert f(2, 32) == 2 * (32 + 16)             # INT2 G32
    assert f(16, 128) == 2 * 256                 # FP16 rows, no meta
    assert f(8, 64) == 2 * (128 + 8)             # 8-bit codes G64 (FP8, symmetric INT8)
    # per-channel K: 128 (s, z) pairs per 32-token block = 16 bytes a token
    assert f(4, 64, k_channels=True) == 64 + 64 + 8 + 16
    assert f(4, 128, fmt="oaken") == 2 * (64 + 32)


def test_kernel_hash_covers_every_decode_source():
    csrc = os.path.join(bench.ROOT, "quantized_kv_cache_12_b200", "csrc")
    h0 = bench.kernel_source_hash()
    assert len(h0) == 16 and h0 == bench.kernel_source_hash()
    # every file whose code a decode launch runs or whose plan picks it
    decode_files = {"kvq_decode.cu", "kvq_decode_tm.cu", "kvq_decode_common.cuh",
                    "kvq_device.cuh", "kvq_quant_core.cuh", "kvq_internal.h", "kvq_abi.cu",
                    "kvq_oaken.cu"}
    assert decode_files <= set(os.listdir(csrc))
    import inspect
    src = inspect.getsource(bench.kernel_source_hash)
    for f in decode_files:
        assert f'"{f}"' in src, f
