"""Host logic of the multi-GPU path, run as world-size-2 process groups on the
CPU (gloo): the path shards whole sequences across ranks (weak scaling), so
the only collectives are the timing reductions, and the reference arm runs on
rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))


def _max_worker(rank, world, port, out):
    _init(rank, world, port)
    try:
        out[rank] = bench.max_over_ranks(1.5 + 3.0 * rank, "cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    """Every rank gets the slowest rank's time."""
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_max_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    assert dict(out) == {0: 4.5, 1: 4.5}


def _shard_worker(rank, world, port, out):
    """Each rank attends its own sequences with the oracle (standing in for
    the kernel on CPU), then the results are gathered for the check."""
    _init(rank, world, port)
    try:
        wl = bench.rank_workload(workloads.WORKLOADS["tiny"].scaled(batch=2, kv_heads=2,
                                                                    q_heads=4), rank)
        k, v = workloads.kv_tokens(wl, 64, "cpu")
        q = workloads.queries(wl, "cpu")
        segs = []
        for plane in (k, v):
            c, m = oracle.quantize_cache(plane.numpy().view(np.uint16), wl.group, wl.bits)
            segs.append((c, m))
        seg = dict(k_codes=segs[0][0], k_meta=segs[0][1], v_codes=segs[1][0],
                   v_meta=segs[1][1], bits=wl.bits, group=wl.group)
        qb = q.contiguous().view(torch.int16).numpy().view(np.uint16)
        o, lse = oracle.decode_attention(qb, False, [seg], [[64, 40]], 128 ** -0.5)
        ko = torch.from_numpy(k.numpy().astype(np.float32))
        gathered = [torch.zeros_like(ko) for _ in range(world)]
        dist.all_gather(gathered, ko)
        og = [torch.zeros(o.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(og, torch.from_numpy(o))
        if rank == 0:
            out["k"] = [g.numpy() for g in gathered]
            out["o"] = [g.numpy() for g in og]
    finally:
        dist.destroy_process_group()


def test_ranks_attend_disjoint_sequences_gloo():
    """Weak scaling shards by sequence: the ranks' inputs differ, and each
    rank's output is exactly what one process computes for those sequences."""
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_shard_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    k0, k1 = out["k"]
    assert not np.array_equal(k0, k1)
    # rank 1's sequences recomputed in this process
    wl = bench.rank_workload(workloads.WORKLOADS["tiny"].scaled(batch=2, kv_heads=2, q_heads=4),
                             1)
    k, v = workloads.kv_tokens(wl, 64, "cpu")
    q = workloads.queries(wl, "cpu")
    kc, km = oracle.quantize_cache(k.numpy().view(np.uint16), wl.group, wl.bits)
    vc, vm = oracle.quantize_cache(v.numpy().view(np.uint16), wl.group, wl.bits)
    seg = dict(k_codes=kc, k_meta=km, v_codes=vc, v_meta=vm, bits=wl.bits, group=wl.group)
    o, _ = oracle.decode_attention(q.contiguous().view(torch.int16).numpy().view(np.uint16),
                                   False, [seg], [[64, 40]], 128 ** -0.5)
    np.testing.assert_array_equal(out["o"][1], o)


def test_reference_arm_runs_on_rank0_only():
    """Under torchrun the reference arm prints one line from rank 0; the other
    rank exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "1",
           "--workload", "tiny"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
