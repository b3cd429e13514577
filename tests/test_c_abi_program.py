"""The C ABI from plain C: tests/c_abi_roundtrip.c includes include/kvq.h,
allocates with cudaMalloc, sizes its buffers with kvq_plane_bytes and
kvq_decode_workspace_bytes, prefills an INT4 G64 cache with
kvq_quantize_append and runs kvq_decode_attention, with no PyTorch in the
process.  On the CPU the program is compiled and linked against libkvq.so;
on a GPU it runs, and its codes and (s, z) must equal the oracle's byte for
byte and its attention output must be within the attention tolerance of the
oracle's fp64 result on the same inputs (which the program writes out)."""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi_roundtrip.c")
PKG = os.path.join(ROOT, "quantized_kv_cache_12_b200")
B, H, G_RATIO, D, L, MAX_TOKENS, BITS, GROUP = 2, 2, 4, 128, 300, 320, 4, 64
LENS = [L, 123]


def _cuda_home():
    nvcc = shutil.which("nvcc")
    return os.environ.get("CUDA_HOME") or (os.path.dirname(os.path.dirname(nvcc)) if nvcc
                                           else "/usr/local/cuda")


def _build(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    lib = os.path.join(PKG, "libkvq.so")
    assert os.path.exists(lib), "libkvq.so not built"
    cuda = _cuda_home()
    exe = tmp_path / "c_abi_roundtrip"
    subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Werror",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
                    SRC, "-o", str(exe), "-L", PKG, "-lkvq",
                    "-L", os.path.join(cuda, "lib64"), "-lcudart", "-lm",
                    f"-Wl,-rpath,{PKG}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}"],
                   check=True, capture_output=True, text=True)
    return exe


def test_c_program_compiles_and_links(tmp_path):
    assert os.path.exists(_build(tmp_path))


@pytest.mark.gpu
def test_c_program_matches_the_oracle(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    exe = _build(tmp_path)
    run = subprocess.run([str(exe), str(tmp_path)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    Hq = H * G_RATIO

    def rd(name, dtype, shape):
        return np.fromfile(tmp_path / name, dtype=dtype).reshape(shape)
    k = rd("k.bin", np.uint16, (B, H, L, D))
    v = rd("v.bin", np.uint16, (B, H, L, D))
    q = rd("q.bin", np.uint16, (B, Hq, D))
    rb = D * BITS // 8
    kc = rd("k_codes.bin", np.uint8, (B, H, MAX_TOKENS, rb))
    vc = rd("v_codes.bin", np.uint8, (B, H, MAX_TOKENS, rb))
    km = rd("k_meta.bin", np.uint16, (B, H, MAX_TOKENS, D // GROUP, 2))
    vm = rd("v_meta.bin", np.uint16, (B, H, MAX_TOKENS, D // GROUP, 2))
    okc, okm = oracle.quantize_cache(k, GROUP, BITS)
    ovc, ovm = oracle.quantize_cache(v, GROUP, BITS)
    assert np.array_equal(kc[:, :, :L], okc) and np.array_equal(km[:, :, :L], okm)
    assert np.array_equal(vc[:, :, :L], ovc) and np.array_equal(vm[:, :, :L], ovm)
    seg = dict(k_codes=okc, k_meta=okm, v_codes=ovc, v_meta=ovm, bits=BITS, group=GROUP)
    o_ref, l_ref = oracle.decode_attention(q, False, [seg], [np.asarray(LENS)], D ** -0.5)
    out = torch.from_numpy(rd("out.bin", np.float32, (B, Hq, D)).copy())
    lse = rd("lse.bin", np.float32, (B, Hq))
    assert_close(out, o_ref, lse, l_ref, what="plain-C caller vs oracle")
