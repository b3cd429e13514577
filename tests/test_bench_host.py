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


def test_oaken_outlier_stats():
    """Rows with more outliers than the 16 slots: s_in = 1, z_in = 8 puts the
    thresholds at -8 and 7; values equal to a threshold are inner."""
    import torch
    x = torch.zeros((1, 1, 3, 128), dtype=torch.float16)
    x[0, 0, 0, :20] = 7.5          # 20 outliers above T_hi: 4 dropped
    x[0, 0, 1, :3] = -9.0          # 3 below T_lo
    x[0, 0, 1, 3:5] = 7.0          # on T_hi: inner
    x[0, 0, 2, 0] = -8.0           # on T_lo: inner
    st = bench.oaken_outlier_stats(x, (1.0, 8, 0.5, 5))
    assert st["rows"] == 3 and st["rows_over_16"] == 1 and st["max_outliers_per_row"] == 20
    assert st["outliers_dropped"] == 4 and abs(st["mean_outliers_per_row"] - 23 / 3) < 1e-12
