#!/usr/bin/env python
"""Decode-step benchmark of the quantized KV cache on B200.

One step = quantize-on-write of one new token per sequence + decode
attention of one query per sequence over the whole packed cache
(kvq_decode_step: the split-K kernel with the append inside it, then the
log-sum-exp merge kernel).  Default workload: the Llama-3-8B-shaped GQA layer (batch 32,
32 query / 8 KV heads, head_dim 128, context 8192, INT4 group 64, fp16
queries); the cache length runs through the workload's 100-step episode
(8193 .. 8292 tokens) and restarts, so any --steps keeps the same shape.

Prints one JSON line (rank 0): tokens/s over all ranks (device-timed, max
over ranks), the roofline of the split-K attention kernel against the
measured HBM copy bandwidth, end-to-end tokens/s through the public API with
host buffers, the oracle's CPU throughput, and clocks sampled during the
timed region.  `--impl reference` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attention tokens/s; KV-read GB/s as % of B200 HBM peak"
DTYPE = {2: "u2", 4: "u4", 8: "u8", 16: "f16"}
# code formats: arithmetic type, JSON name, and the library's format code
FMT_DTYPE = {"fp8": "e4m3", "sym8": "s8", "e5m2": "e5m2", "oaken": "u4"}
FMT_NAME = {"fp8": "fp8 e4m3", "sym8": "symmetric int8", "e5m2": "fp8 e5m2",
            "oaken": "oaken group-shift (4-bit dense + 16 outlier slots)"}
# KVQ_FMT_INT, KVQ_FMT_FP8_E4M3, KVQ_FMT_INT8_SYM, KVQ_FMT_FP8_E5M2, KVQ_FMT_OAKEN
FMT_CODE = {"int": 0, "fp8": 1, "sym8": 2, "e5m2": 3, "oaken": 4}
OAKEN_SLOTS = 16
NOMINAL_HBM_GBS = 8000.0
# one graph in this many carries the event nodes that time the split-K kernel
INSTR_EVERY = 10
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=15000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    p.add_argument("--workload", default="llama3_8b_gqa_int4")
    p.add_argument("--batch", type=int, default=0,
                   help="override the workload's batch (smaller cases for profiling)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    return p.parse_args()


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def bytes_per_head_token(bits: int, group: int, head_dim: int = 128,
                         k_channels: bool = False, fmt: str = "int") -> int:
    """K plus V bytes of one (sequence, KV head, token): codes + (s, z) pairs
    (per-channel K: head_dim pairs per 32-token block, 16 bytes a token;
    the Oaken codec: 4-bit codes + 16 two-byte outlier slots per row)."""
    if fmt == "oaken":
        return 2 * (head_dim // 2 + 2 * OAKEN_SLOTS)
    meta = 0 if bits == 16 else (head_dim // group) * 4
    kmeta = head_dim * 4 // 32 if k_channels else meta
    return 2 * (head_dim * bits // 8) + meta + kmeta


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    # the decode kernels' sources and the headers they compile (the fused
    # append's quantizer included), and the host code whose split plan picks
    # the kernel build and the units of a launch
    for f in ("kvq_decode.cu", "kvq_decode_tm.cu", "kvq_decode_common.cuh", "kvq_device.cuh",
              "kvq_quant_core.cuh", "kvq_internal.h", "kvq_abi.cu", "kvq_oaken.cu"):
        with open(os.path.join(ROOT, "quantized_kv_cache_12_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def split_kernel_name(wl) -> str:
    """The decode kernel the library picks for this workload's formats: the
    tokens-on-M kernel when (head_dim / G) * g <= 8, else the 16-row one."""
    g = wl.q_heads // wl.kv_heads
    if wl.fmt == "oaken":  # one (s, z) per plane: a single group per token
        return "decode_tm_kernel"
    groups = [128, wl.group] if wl.chunk_tokens else [wl.group]  # + the FP16 segment
    ok = all((128 // G) * g <= 8 for G in groups)
    return "decode_tm_kernel" if ok else "decode_split_kernel"


def recorded_traffic(workload: str):
    """DRAM bytes per split-kernel launch from the committed ncu summary, or
    None when the kernel source changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(workload)
    except Exception:
        return None
    if not rec or rec.get("kernel_sha") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons (every 100 ms)."""
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 6:
                self.samples.append((time.time(), parts))

    def wait_first(self, timeout_s: float):
        """Return once the first sample has arrived (nvidia-smi takes a moment
        to start), or after timeout_s."""
        t_end = time.time() + timeout_s
        while self.proc is not None and not self.samples and time.time() < t_end:
            time.sleep(0.02)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        inside = [s for t, s in self.samples if t0 <= t <= t1]
        window = "timed region"
        if not inside:
            inside = [s for _, s in self.samples]
            window = "whole run (timed region shorter than the 100 ms sampling period)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in inside for i in range(4)
                          if s[2 + i].lower().startswith("active")})

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(s[0]) for s in inside if num(s[0]) is not None]
        mx = [num(s[1]) for s in inside if num(s[1]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(inside), "window": window}


# ---------------------------------------------------------------- reference arm

def segment_oracle_pairs(wl, k, v, q, pairs):
    """Oracle inputs of (sequence, KV head) pairs of an attention-only
    workload: K per channel over 32-token blocks and V per token, or both
    planes in the Oaken codec; each entry is (q patterns [1, g, D], the
    one-pair segment, its length)."""
    import numpy as np
    import torch

    import oracle
    import workloads
    g = wl.group_ratio
    out = []
    if wl.fmt == "oaken":
        kp, vp = workloads.oaken_params(wl, "k"), workloads.oaken_params(wl, "v")
    for b, h in pairs:
        kk = k[b, h].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        vv = v[b, h].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        if wl.fmt == "oaken":
            kc, km = oracle.oaken_quantize_rows(kk, *kp)
            vc, vm = oracle.oaken_quantize_rows(vv, *vp)
            seg = dict(k_codes=kc[None, None], k_meta=km[None, None], v_codes=vc[None, None],
                       v_meta=vm[None, None], bits=4, group=128, fmt="oaken", k_oaken=kp,
                       v_oaken=vp)
        else:
            kc, km = oracle.quantize_cache_channels(kk, wl.bits)
            vc, vm = oracle.quantize_rows(vv, wl.group, wl.bits)
            seg = dict(k_codes=kc[None, None], k_meta=km[None, None], v_codes=vc[None, None],
                       v_meta=vm[None, None], bits=wl.bits, group=wl.group, k_channels=True)
        qh = q[b, h * g:(h + 1) * g].cpu().contiguous().view(torch.int16).numpy()
        out.append((qh.view(np.uint16)[None], seg, [np.array([kk.shape[0]])]))
    return out


def run_reference(args, wl):
    """The CPU oracle as it stands, on this host's cores (one thread per
    core): each step attends one (sequence, KV head) of the workload after
    appending one token (attention alone for a workload without an
    append, as its GPU step)."""
    import numpy as np
    import torch

    import oracle
    import workloads
    if wl.chunk_tokens:
        sub = wl.scaled(batch=1, kv_heads=min(wl.kv_heads, 4), q_heads=min(wl.kv_heads, 4))
        k, v = workloads.kv_tokens(sub, wl.context, "cpu")
        q = workloads.queries(sub, "cpu")
        prepared, counts = prepare_mixed_oracle(wl, k, v, q, sub)

        def mixed_step(i):
            qh, segs, lens = prepared[i % len(prepared)]
            oracle.decode_attention(qh, False, segs, lens, 128 ** -0.5)
        for i in range(args.warmup):
            mixed_step(i)
        el = run_steps_parallel(mixed_step, args.steps)
        value = args.steps / wl.kv_heads / el
        sample = (f"each step: one (sequence, KV head) of {wl.name}: attention over its "
                  f"{wl.n_chunks} chunks as FP16/INT4/INT2 segments ({int(counts[0])}/"
                  f"{int(counts[1])}/{int(counts[2])} chunks); tokens/s = steps / kv_heads "
                  f"({wl.kv_heads}) / seconds")
        print(json.dumps(reference_line(args, wl, value, el, sample)), flush=True)
        return
    if wl.k_axis == "channel" or wl.fmt == "oaken":
        sub = wl.scaled(batch=1, kv_heads=min(wl.kv_heads, 4),
                        q_heads=min(wl.kv_heads, 4) * wl.group_ratio)
        k, v = workloads.kv_tokens(sub, wl.context, "cpu")
        q = workloads.queries(sub, "cpu")
        prepared = segment_oracle_pairs(wl, k, v, q, [(0, h) for h in range(sub.kv_heads)])

        def kpc_step(i):
            qh, seg, lens = prepared[i % len(prepared)]
            oracle.decode_attention(qh, wl.q_dtype == "bf16", [seg], lens, 128 ** -0.5)
        for i in range(args.warmup):
            kpc_step(i)
        el = run_steps_parallel(kpc_step, args.steps)
        value = args.steps / wl.kv_heads / el
        how = "Oaken codec" if wl.fmt == "oaken" else "K per channel"
        sample = (f"each step: one (sequence, KV head) of {wl.name}: attention of "
                  f"{wl.group_ratio} query heads over {wl.context} tokens, {how}; "
                  f"tokens/s = steps / kv_heads ({wl.kv_heads}) / seconds")
        print(json.dumps(reference_line(args, wl, value, el, sample)), flush=True)
        return
    sub = wl.scaled(batch=1, kv_heads=min(wl.kv_heads, 4),
                    q_heads=min(wl.kv_heads, 4) * wl.group_ratio)
    L = wl.context
    k, v = workloads.kv_tokens(sub, L, "cpu")
    kn, vn = workloads.kv_tokens(sub, 1, "cpu", stream_extra=1)
    q = workloads.queries(sub, "cpu")
    g = wl.group_ratio
    prepared = []
    for h in range(sub.kv_heads):
        kc, km = oracle.quantize_rows(k[0, h].numpy().view(np.uint16), wl.group, wl.bits, wl.fmt)
        vc, vm = oracle.quantize_rows(v[0, h].numpy().view(np.uint16), wl.group, wl.bits, wl.fmt)
        qh = q[0, h * g:(h + 1) * g].contiguous().view(torch.int16).numpy().view(np.uint16)
        prepared.append((kc, km, vc, vm, qh, kn[0, h].numpy().view(np.uint16),
                         vn[0, h].numpy().view(np.uint16)))

    def step(i):
        kc, km, vc, vm, qh, knew, vnew = prepared[i % len(prepared)]
        if not wl.append:  # the step is the attention over the prefilled cache
            oracle.attention_packed(qh, wl.q_dtype == "bf16", kc, km, wl.bits, vc, vm, wl.bits,
                                    wl.group, L, 128 ** -0.5, wl.fmt)
            return
        ck, mk = oracle.quantize_rows(knew, wl.group, wl.bits, wl.fmt)
        cv, mv = oracle.quantize_rows(vnew, wl.group, wl.bits, wl.fmt)
        kc2 = np.concatenate([kc, ck])
        km2 = np.concatenate([km, mk])
        vc2 = np.concatenate([vc, cv])
        vm2 = np.concatenate([vm, mv])
        oracle.attention_packed(qh, wl.q_dtype == "bf16", kc2, km2, wl.bits, vc2, vm2, wl.bits,
                                wl.group, L + 1, 128 ** -0.5, wl.fmt)

    for i in range(args.warmup):
        step(i)
    el = run_steps_parallel(step, args.steps)
    value = args.steps / wl.kv_heads / el
    what = (f"at {L + 1} tokens (append 1 token + attention of {g} query heads)" if wl.append
            else f"at {L} tokens (attention of {g} query heads, no append)")
    sample = (f"each step: one (sequence, KV head) of {wl.name} {what}; tokens/s = steps / "
              f"kv_heads ({wl.kv_heads}) / seconds")
    print(json.dumps(reference_line(args, wl, value, el, sample)), flush=True)


def run_steps_parallel(step, steps: int) -> float:
    """Run step(0) .. step(steps - 1) on one host thread per core (thread i
    takes steps i, i + n, ...; the oracle's C calls release the interpreter
    lock); returns the elapsed seconds."""
    import threading
    n = max(1, min(os.cpu_count() or 1, steps))
    t0 = time.perf_counter()
    ts = [threading.Thread(target=lambda i=i: [step(j) for j in range(i, steps, n)])
          for i in range(n)]
    for th in ts:
        th.start()
    for th in ts:
        th.join()
    return time.perf_counter() - t0


def reference_line(args, wl, value, el, sample):
    threads = max(1, min(os.cpu_count() or 1, args.steps))
    sample = f"{sample}; steps spread over {threads} host threads (one per core)"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": FMT_DTYPE.get(wl.fmt, DTYPE[wl.bits]),
        "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": min(os.cpu_count() or 1,
                                                                           args.steps),
                         "nproc": os.cpu_count(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def workload_config(wl, extra=None):
    cfg = {"workload": wl.name, "batch_per_gpu": wl.batch, "q_heads": wl.q_heads,
           "kv_heads": wl.kv_heads, "head_dim": wl.head_dim, "context": wl.context,
           "bits": wl.bits, "group": wl.group, "q_dtype": wl.q_dtype,
           **({"format": FMT_NAME[wl.fmt]} if wl.fmt != "int" else {}),
           **({"k_grouping": "per channel, 32-token blocks"} if wl.k_axis == "channel" else {}),
           "episode_steps": wl.steps if wl.append else 0}
    if extra:
        cfg.update(extra)
    return cfg


# ---------------------------------------------------------------- CPU baseline

def time_oracle_jobs(jobs, seconds: float, threads: int):
    """Run the oracle jobs round-robin on `threads` host threads for about
    `seconds` (each thread at least one job); returns (jobs done, seconds).
    The oracle is C called through ctypes, which releases the interpreter
    lock for the call, so the threads run on separate cores."""
    import threading
    done = [0] * threads
    t0 = time.perf_counter()

    def worker(i):
        n = 0
        while True:
            jobs[(i + n * threads) % len(jobs)]()
            n += 1
            if time.perf_counter() - t0 >= seconds:
                break
        done[i] = n
    ts = [threading.Thread(target=worker, args=(i,)) for i in range(threads)]
    for th in ts:
        th.start()
    for th in ts:
        th.join()
    return sum(done), time.perf_counter() - t0


def oracle_baseline(wl, jobs, seconds: float, what: str):
    """The oracle as it stands on a bounded sample: one host thread, then
    every host core (one thread per core).  tokens/s = (sequence, KV head)
    jobs / kv_heads / seconds (a job is one sequence's work for one KV head)."""
    nproc = os.cpu_count() or 1
    n1, el1 = time_oracle_jobs(jobs, seconds, 1)
    nn, eln = time_oracle_jobs(jobs, seconds, nproc)
    single = {"value": n1 / wl.kv_heads / el1, "unit": "tokens/s", "cores": 1,
              "sample": f"{n1} {what} cycling over {len(jobs)} (sequence, KV head) pairs, "
                        f"{el1:.1f} s on one host thread"}
    return {"value": nn / wl.kv_heads / eln, "unit": "tokens/s", "cores": nproc,
            "nproc": nproc, "kind": "oracle",
            "sample": f"{nn} {what} cycling over {len(jobs)} (sequence, KV head) pairs, "
                      f"{eln:.1f} s on {nproc} host threads (one per core, nproc = {nproc}); "
                      f"tokens/s = jobs / kv_heads / seconds",
            "single_thread": single}


def cpu_baseline(wl, k, v, kn, vn, q, seconds: float):
    """The oracle (C, fp64 attention) on a bounded sample of the same inputs:
    (sequence, KV head) pairs, each one append + attention (kn, vn: the new
    token's rows), or attention alone for a workload without an append."""
    import numpy as np
    import torch

    import oracle
    g = wl.group_ratio
    pairs = [(b, h) for b in range(min(wl.batch, 2)) for h in range(min(wl.kv_heads, 4))]
    if wl.k_axis == "channel" or wl.fmt == "oaken":
        prep = segment_oracle_pairs(wl, k, v, q, pairs)

        def job_of(qh, seg, lens):
            return lambda: oracle.decode_attention(qh, wl.q_dtype == "bf16", [seg], lens,
                                                   128 ** -0.5)
        jobs = [job_of(*p) for p in prep]
        how = "Oaken codec" if wl.fmt == "oaken" else "K per channel"
        return oracle_baseline(wl, jobs, seconds,
                               f"attentions of {wl.name} over {k.shape[2]} tokens ({how})")
    L = k.shape[2]
    jobs = []
    for b, h in pairs:
        kk = k[b, h].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        vv = v[b, h].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        kc, km = oracle.quantize_rows(kk, wl.group, wl.bits, wl.fmt)
        vc, vm = oracle.quantize_rows(vv, wl.group, wl.bits, wl.fmt)
        qh = q[b, h * g:(h + 1) * g].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        if kn is None:  # no append: attention over the prefilled tokens
            def job(kc=kc, km=km, vc=vc, vm=vm, qh=qh):
                oracle.attention_packed(qh, wl.q_dtype == "bf16", kc, km, wl.bits, vc, vm,
                                        wl.bits, wl.group, L, 128 ** -0.5, fmt=wl.fmt)
            jobs.append(job)
            continue
        knew = kn[b, h].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        vnew = vn[b, h].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

        def job(kc=kc, km=km, vc=vc, vm=vm, qh=qh, knew=knew, vnew=vnew):
            ck, mk = oracle.quantize_rows(knew, wl.group, wl.bits, wl.fmt)
            cv, mv = oracle.quantize_rows(vnew, wl.group, wl.bits, wl.fmt)
            oracle.attention_packed(qh, wl.q_dtype == "bf16", np.concatenate([kc, ck]),
                                    np.concatenate([km, mk]), wl.bits,
                                    np.concatenate([vc, cv]), np.concatenate([vm, mv]),
                                    wl.bits, wl.group, L + 1, 128 ** -0.5, fmt=wl.fmt)
        jobs.append(job)
    what = (f"decode steps (append + attention) of {wl.name} at {L + 1} tokens" if kn is not None
            else f"attentions of {wl.name} over {L} tokens")
    return oracle_baseline(wl, jobs, seconds, what)


def prepare_mixed_oracle(wl, k, v, q, wlr):
    """Oracle inputs for (sequence 0, KV head h) pairs of the chunk-level mixed
    workload: its own chunk classes (fp64 similarity), reorder and
    quantization.  Returns (prepared pairs, class counts)."""
    import numpy as np
    import torch

    import oracle
    import workloads
    emb, qemb = workloads.chunk_embeddings(wlr.scaled(batch=1), "cpu")
    _, cls = oracle.chunk_assign(emb[0].numpy(), qemb[0].numpy(), wl.alpha, wl.beta)
    perm, counts = oracle.chunk_partition(cls)
    T = wl.chunk_tokens
    prepared = []
    for h in range(min(wl.kv_heads, 4)):
        segs, lens, start = [], [], 0
        for bits, cnt in zip((16,) + wl.low_bits, counts):
            idx = perm[start:start + cnt]
            start += cnt
            tok = (idx[:, None] * T + np.arange(T)[None]).reshape(-1)
            kk = k[0, h, torch.from_numpy(tok).to(k.device)].cpu().contiguous()
            vv = v[0, h, torch.from_numpy(tok).to(v.device)].cpu().contiguous()
            k16 = kk.view(torch.int16).numpy().view(np.uint16)[None, None]
            v16 = vv.view(torch.int16).numpy().view(np.uint16)[None, None]
            if bits == 16:
                seg = dict(k_codes=k16.view(np.uint8).reshape(1, 1, -1, 256),
                           v_codes=v16.view(np.uint8).reshape(1, 1, -1, 256), k_meta=None,
                           v_meta=None, bits=16, group=128)
            else:
                kc, km = oracle.quantize_cache(k16, wl.group, bits)
                vc, vm = oracle.quantize_cache(v16, wl.group, bits)
                seg = dict(k_codes=kc, v_codes=vc, k_meta=km, v_meta=vm, bits=bits,
                           group=wl.group)
            segs.append(seg)
            lens.append(np.array([len(tok)]))
        qh = q[0:1, h:h + 1].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        prepared.append((qh, segs, lens))
    return prepared, counts


def cpu_baseline_mixed(wl, k, v, q, seconds: float, wlr):
    """The oracle's timed fp64 attention over the three segments of sampled
    (sequence, KV head) pairs of the chunk-level mixed workload."""
    import oracle
    prepared, counts = prepare_mixed_oracle(wl, k, v, q, wlr)

    def job_of(qh, segs, lens):
        return lambda: oracle.decode_attention(qh, False, segs, lens, 128 ** -0.5)
    jobs = [job_of(*p) for p in prepared]
    return oracle_baseline(wl, jobs, seconds,
                           f"attention steps of {wl.name} over its {int(sum(counts))} chunks "
                           f"({int(counts[0])} FP16, {int(counts[1])} INT4, {int(counts[2])} "
                           f"INT2)")


# ---------------------------------------------------------------- kvq arm

def oaken_outlier_stats(x, params) -> dict:
    """Outliers per token row of one plane of an Oaken workload's prompt:
    values outside [T_lo, T_hi] (T_lo = -z_in s_in, T_hi = (15 - z_in) s_in,
    exact for an fp16 s_in and an integer z_in), and the rows with more than
    the 16 slots hold (those past the 16th reconstruct to their threshold)."""
    s_in, z_in, _, _ = params
    t_lo, t_hi = -z_in * s_in, (15 - z_in) * s_in
    xf = x.float()
    cnt = ((xf < t_lo) | (xf > t_hi)).sum(-1).flatten()
    total = int(cnt.sum())
    dropped = int((cnt - 16).clamp(min=0).sum())
    return {"rows": int(cnt.numel()), "rows_over_16": int((cnt > 16).sum()),
            "frac_rows_over_16": float((cnt > 16).float().mean()),
            "mean_outliers_per_row": total / max(1, int(cnt.numel())),
            "max_outliers_per_row": int(cnt.max()), "outliers_dropped": dropped,
            "frac_outliers_dropped": dropped / max(1, total)}


def max_over_ranks(x: float, device) -> float:
    """The largest of every rank's value (a job is as slow as its slowest
    rank); `device` is where the backend wants its tensors."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(wl, rank: int):
    """Weak scaling: every rank attends its own batch of sequences, drawn from
    its own seeds; no sequence is shared, so no collective touches the data."""
    return wl.scaled(seed=wl.seed + 1000 * rank)


def run_kvq(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import workloads
    from quantized_kv_cache_12_b200 import kvq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, H, Hq, D = wl.batch, wl.kv_heads, wl.q_heads, wl.head_dim
    ctx = wl.context
    episode = wl.steps if wl.append else min(wl.steps, 100)
    wlr = rank_workload(wl, rank)
    kpc = wl.k_axis == "channel"  # K grouped per channel over 32-token blocks

    # ---- resident inputs (untimed set-up)
    prefill = None  # set by the single-cache set-up below
    outlier_stats = None  # Oaken codec: how often a row overflows its 16 slots
    chunk_timing = None  # set by the chunk-level mixed set-up below
    if wl.chunk_tokens:
        # chunk-level mixed precision: search, reorder, quantize the prompt
        # into FP16 / INT4 / INT2 segments once; each step attends over them
        emb, qemb = workloads.chunk_embeddings(wlr, dev)
        cbits = torch.empty((B, wl.n_chunks), dtype=torch.uint8, device=dev)
        kvq.kvq_chunk_assign(emb, qemb, wl.alpha, wl.beta, cbits)
        k, v = workloads.kv_tokens(wlr, ctx, dev)
        segs = [kvq.QuantizedKVCache.allocate(B, H, D, workloads.round_up(ctx, 64), bits,
                                              wl.group, dev) for bits in (16,) + wl.low_bits]
        perm = torch.empty((B, wl.n_chunks), dtype=torch.int32, device=dev)
        kvq.kvq_chunk_reorder(segs, k, v, wl.chunk_tokens, cbits, perm)
        seg_lens = [c.seq_lens.cpu().numpy().astype(np.int64) for c in segs]
        # the chunk search and the reorder (one-off per prompt), timed on their
        # own, 3 launches each: the search reads the chunk and query embeddings
        # once; the reorder reads the fp16 K and V once and writes each class's
        # codes and (s, z) once
        ca_ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        torch.cuda.synchronize()
        ca_ev[0].record()
        for _ in range(3):
            kvq.kvq_chunk_assign(emb, qemb, wl.alpha, wl.beta, cbits)
        ca_ev[1].record()
        for _ in range(3):
            kvq.kvq_chunk_reorder(segs, k, v, wl.chunk_tokens, cbits, perm)
        ca_ev[2].record()
        torch.cuda.synchronize()
        assign_us = ca_ev[0].elapsed_time(ca_ev[1]) * 1e3 / 3
        reorder_us = ca_ev[1].elapsed_time(ca_ev[2]) * 1e3 / 3
        assign_bytes = emb.numel() * 4 + qemb.numel() * 4
        reorder_bytes = B * H * ctx * 2 * D * 2 + sum(
            int(ln.sum()) * H * bytes_per_head_token(c.bits, wl.group, D)
            for ln, c in zip(seg_lens, segs))
        chunk_timing = {"assign_us": assign_us, "assign_bytes": assign_bytes,
                        "reorder_us": reorder_us, "reorder_bytes": reorder_bytes,
                        "reorder_gbs": reorder_bytes / (reorder_us / 1e6) / 1e9,
                        "kernels": "chunk_assign_kernel, chunk_partition_kernel + chunk_bulk_kernel",
                        "note": "3 launches each; reorder bytes: fp16 K and V read + every "
                                "segment's codes and (s, z) written"}
        del emb, qemb
        seg_bits = [c.bits for c in segs]
        k_cpu_src = (k, v, cbits)
        base_lens = None
        kn = None
    else:
        max_tokens = workloads.round_up(ctx + episode + 1, 64)
        k, v = workloads.kv_tokens(wlr, ctx, dev)
        oaken = ({"k_oaken": workloads.oaken_params(wl, "k"),
                  "v_oaken": workloads.oaken_params(wl, "v")} if wl.fmt == "oaken" else {})
        cache = kvq.QuantizedKVCache.allocate(
            B, H, D, max_tokens, wl.bits, wl.group, dev,
            fmt=FMT_CODE[wl.fmt], k_axis=1 if kpc else 0, **oaken)
        cache.seq_lens.zero_()
        kvq.kvq_quantize_append(cache, k, v, ctx, advance_seq_lens=True)
        base_lens = cache.seq_lens.clone()
        if wl.fmt == "oaken":
            outlier_stats = {"k": oaken_outlier_stats(k, oaken["k_oaken"]),
                             "v": oaken_outlier_stats(v, oaken["v_oaken"])}
        # the prefill quantize (bulk quantize-on-write of the whole context),
        # timed on its own: HBM-bound, fp16 K/V read once, codes and (s, z)
        # written once
        # each call timed alone (the seq_lens reset between calls is not)
        pf_reps = 5
        pf_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(pf_reps)]
        torch.cuda.synchronize()
        for e0, e1 in pf_ev:
            cache.seq_lens.zero_()
            e0.record()
            kvq.kvq_quantize_append(cache, k, v, ctx, advance_seq_lens=True)
            e1.record()
        torch.cuda.synchronize()
        pf_us = statistics.median(e0.elapsed_time(e1) * 1e3 for e0, e1 in pf_ev)
        pf_bytes = B * H * ctx * (2 * D * 2 + bytes_per_head_token(wl.bits, wl.group, D, kpc,
                                                                   wl.fmt))
        prefill = {"tokens": B * ctx, "us": pf_us, "bytes": pf_bytes,
                   "gbs": pf_bytes / (pf_us / 1e6) / 1e9,
                   "kernel": ("oaken_bulk_kernel" if wl.fmt == "oaken" else
                              "quantize_k_channels_kernel + quantize_bulk_kernel" if kpc
                              else "quantize_bulk_kernel"),
                   "note": "fp16 K and V read + packed codes and (s, z) written, per "
                           "kvq_quantize_append call (median of 5 calls, each timed alone "
                           "after a 4-byte seq_lens reset)"}
        segs = [cache]
        seg_bits = [wl.bits]
        seg_lens = None
        k_cpu_src = None
        kn = torch.stack([torch.stack(workloads.kv_tokens(wlr, 1, dev, stream_extra=1 + e))
                          for e in range(episode)]) if wl.append else None  # [E, 2, B, H, 1, D]
    qs = torch.stack([workloads.queries(wlr, dev, step=e) for e in range(episode)])
    hint = ctx + episode if wl.append else ctx
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    ws = kvq.alloc_workspace(segs, Hq, hint, device=dev)
    ws_bytes = kvq.kvq_decode_workspace_bytes(segs, Hq, hint)
    bh = B * Hq
    r256 = lambda n: (n + 255) // 256 * 256  # noqa: E731

    def ws_for(p):  # kvq_decode_workspace_bytes' layout for p partials
        return 256 + r256(B * 4) + r256(bh * p * 8) + r256(bh * p * D * 4)
    parts = next(p for p in range(1, 1 << 16) if ws_for(p) == ws_bytes)
    # kernels of the library per step: one split-K launch per segment (the
    # append runs inside it), then the merge when there are several partials
    launches_per_step = len(segs) + (1 if parts > 1 else 0)
    stream = torch.cuda.current_stream()

    def reset_fn(e):  # the episode restarts from the prefilled lengths
        cache.seq_lens.copy_(base_lens, non_blocking=True)

    def partials_fn(e):  # the timed kernel(s): append + split-K attention
        if wl.append:
            kvq.kvq_decode_step_partials(cache, kn[e, 0], kn[e, 1], qs[e], out, lse, ws,
                                         max_len_hint=hint)
        else:
            kvq.kvq_decode_partials(segs, qs[e], out, lse, ws, max_len_hint=hint)

    def merge_fn(e):
        kvq.kvq_decode_merge(segs, qs[e], out, lse, ws, max_len_hint=hint)

    def phases_at(e):
        return ([reset_fn] if wl.append and e == 0 else []) + [partials_fn, merge_fn]

    def step(s):
        for f in phases_at(s % episode):
            f(s % episode)

    def kv_bytes_at(s):
        """Algorithmic K+V bytes of the split kernel(s) at step s."""
        if seg_lens is not None:
            return sum(int(ln.sum()) * H * bytes_per_head_token(bits, wl.group, D)
                       for ln, bits in zip(seg_lens, seg_bits))
        L = ctx + (s % episode) + 1 if wl.append else ctx
        return B * H * L * bytes_per_head_token(wl.bits, wl.group, D, kpc, wl.fmt)

    # ---- warm-up (eager; also makes the one-time kernel attribute settings)
    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    # ---- every episode position as one CUDA graph (reset at the start of an
    # episode, split-K partials, merge), so the timed loop is paced by the
    # device and the merge is a programmatic dependent of the split-K kernel
    # inside the graph.  In every INSTR_EVERY-th position's graph, event-record
    # nodes bracket the split-K launch; after the loop each pair holds the
    # time of its graph's last replay.  The other graphs carry no timing
    # nodes, so most timed steps run as a caller's would.
    from cuda.bindings import runtime as cudart

    # instrumented positions: those of timed steps 0, INSTR_EVERY, 2 INSTR_EVERY,
    # ... within the first episode (the first timed step's always among them)
    instr = sorted({(args.warmup + i) % episode
                    for i in range(0, min(args.steps, episode), INSTR_EVERY)})
    split_evs = {e: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for e in instr}
    for e0, e1 in split_evs.values():  # create the events before the capture
        e0.record(stream)
        e1.record(stream)
    torch.cuda.synchronize()

    def record_in_graph(ev, st):
        err, = cudart.cudaEventRecordWithFlags(ev.cuda_event, st.cuda_stream,
                                               cudart.cudaEventRecordExternal)
        if err != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaEventRecordWithFlags: {err}")

    graphs = []
    cap = torch.cuda.Stream(dev)
    side = torch.cuda.Stream(dev)  # the end-of-split record branches off here
    fork, join = torch.cuda.Event(), torch.cuda.Event()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        for e in range(episode):
            g = torch.cuda.CUDAGraph()
            g.capture_begin()
            if wl.append and e == 0:
                reset_fn(e)
            if e in split_evs:
                record_in_graph(split_evs[e][0], cap)
                partials_fn(e)
                # the end event hangs off the split-K node on a branch, so the
                # merge still follows that node directly (programmatic edge)
                fork.record(cap)
                side.wait_event(fork)
                record_in_graph(split_evs[e][1], side)
                join.record(side)
                merge_fn(e)
                cap.wait_event(join)
            else:
                partials_fn(e)
                merge_fn(e)
            g.capture_end()
            graphs.append(g)
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    # one full episode of replays (uploads the graphs; the state returns to
    # the same episode position)
    for j in range(episode):
        graphs[(args.warmup + j) % episode].replay()
    torch.cuda.synchronize()

    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_id) if rank == 0 else None
    if sampler:
        sampler.wait_first(10.0)  # sampling is running before the timed region opens
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    # A step whose packed K/V fits in L2 would find it there on the next step:
    # then every step is preceded by a write of twice the L2 size, outside
    # the step's own pair of events, and the steps' times are summed.
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_l2 = max(kv_bytes_at(args.warmup + i)
                   for i in range(min(args.steps, episode))) < l2_bytes
    if flush_l2:
        flush_buf = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev)
        step_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    h0 = time.time()
    torch.cuda.nvtx.range_push("kvq_timed")  # lets a profiler select the timed launches
    t_start.record(stream)
    for i in range(args.steps):
        if flush_l2:
            flush_buf.zero_()
            step_evs[i][0].record(stream)
            graphs[(args.warmup + i) % episode].replay()
            step_evs[i][1].record(stream)
        else:
            graphs[(args.warmup + i) % episode].replay()
    t_end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    h1 = time.time()
    ms = (sum(a.elapsed_time(b) for a, b in step_evs) if flush_l2
          else t_start.elapsed_time(t_end))
    # the split-K time of each instrumented graph's last replay in the timed
    # region
    last_step = {(args.warmup + i) % episode: args.warmup + i for i in range(args.steps)
                 if (args.warmup + i) % episode in split_evs}
    split_us = {e: split_evs[e][0].elapsed_time(split_evs[e][1]) * 1e3 for e in last_step}
    assert kvq.workspace_error_word(ws) == 0, "device wait gave up (error word set)"
    if world > 1:
        ms = max_over_ranks(ms, dev)
    clocks = sampler.summary(h0, h1) if sampler else None
    if sampler:
        sampler.stop()

    kv_bytes = [kv_bytes_at(args.warmup + i) for i in range(args.steps)]
    q_bytes = B * Hq * D * 2
    # roofline over the timed split-K launches: their algorithmic bytes over
    # their summed device time
    split_bytes = sum(kv_bytes_at(s_) + q_bytes for s_ in last_step.values())
    split_total_us = sum(split_us.values())
    tokens = B * args.steps * world
    value = tokens / (ms / 1e3)

    # ---- end to end through the public call with pinned host buffers: every
    # step copies its inputs in (the new K/V token and q) and its results out
    # (out, lse).  The copies run on two copy streams, double-buffered, so a
    # step's input copy overlaps the previous step's attention and its output
    # copy overlaps the next one's; the attention calls stay in order on the
    # compute stream.
    # inputs of a step (new K and V token, q) in one pinned host row and one
    # device slot, results (out, lse) likewise: one copy each way per step
    nk = kn[0, 0].numel() if kn is not None else 0  # fp16 elements of k_new (= v_new)
    nq = qs[0].numel()
    in_h = torch.empty((episode, 2 * nk + nq), dtype=torch.float16).pin_memory()
    for e in range(episode):
        if kn is not None:
            in_h[e, :nk].copy_(kn[e, 0].reshape(-1))
            in_h[e, nk:2 * nk].copy_(kn[e, 1].reshape(-1))
        in_h[e, 2 * nk:].copy_(qs[e].reshape(-1))
    in_d = [torch.empty(2 * nk + nq, dtype=torch.float16, device=dev) for _ in range(2)]
    k_d = [b[:nk].view(kn[0, 0].shape) for b in in_d] if kn is not None else None
    v_d = [b[nk:2 * nk].view(kn[0, 1].shape) for b in in_d] if kn is not None else None
    q_d = [b[2 * nk:].view(qs[0].shape) for b in in_d]
    no, nl = out.numel(), lse.numel()
    res_d = [torch.empty(no + nl, dtype=torch.float32, device=dev) for _ in range(2)]
    out_d = [r[:no].view(out.shape) for r in res_d]
    lse_d = [r[no:].view(lse.shape) for r in res_d]
    res_h = [torch.empty(no + nl, dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_read = [torch.cuda.Event() for _ in range(2)]
    if wl.append:
        cache.seq_lens.copy_(base_lens)

    def e2e_step(s, n):  # n: steps since the start of this loop
        e, j = s % episode, n % 2
        with torch.cuda.stream(s_in):
            if n >= 2:
                s_in.wait_event(done[j])  # step n-2 no longer reads slot j
            in_d[j].copy_(in_h[e], non_blocking=True)
            in_ready[j].record(s_in)
        stream.wait_event(in_ready[j])
        if n >= 2:
            stream.wait_event(out_read[j])  # step n-2's results were copied out
        if wl.append:
            if e == 0:
                cache.seq_lens.copy_(base_lens, non_blocking=True)
            kvq.kvq_decode_step(cache, k_d[j], v_d[j], q_d[j], out_d[j], lse_d[j], ws,
                                max_len_hint=hint)
        else:
            kvq.kvq_decode_attention(segs, q_d[j], out_d[j], lse_d[j], ws, max_len_hint=hint)
        done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done[j])
            res_h[j].copy_(res_d[j], non_blocking=True)
            out_read[j].record(s_out)

    for n in range(args.warmup):
        e2e_step(n, n)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(args.steps):
        e2e_step(args.warmup + i, i)
    for j in range(2):  # the region ends after the last results reached the host
        stream.wait_event(out_read[j])
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    if world > 1:
        e_ms = max_over_ranks(e_ms, dev)
    h2d = (kn[0].numel() * 2 if kn is not None else 0) + qs[0].numel() * 2
    d2h = out.numel() * 4 + lse.numel() * 4

    if rank != 0:
        return None
    peak, peak_kind = measured_peak()
    achieved = split_bytes / (split_total_us / 1e6) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": FMT_DTYPE.get(wl.fmt, DTYPE[wl.bits]), "data": "synthetic",
        "config": workload_config(wl, {
            "global_batch": B * world, "parallelism": f"dp{world} (sequences sharded)",
            "cache_tokens_per_step": f"{ctx + 1}..{ctx + episode}" if wl.append else ctx,
            **({"chunk_tokens": wl.chunk_tokens, "alpha": wl.alpha, "beta": wl.beta,
                "segments": {f"bits{b}": int(ln.sum()) for b, ln in zip(seg_bits, seg_lens)}}
               if seg_lens is not None else {}),
            "launch": "each step replayed from one CUDA graph per episode position "
                      + ("(split-K kernel, then the merge as a programmatic dependent); "
                         if parts > 1 else
                         "(one split: the attention kernel writes the output, no merge); ")
                      + f"event-record nodes in one graph of every {INSTR_EVERY} time the split-K "
                      "launch",
            "l2": (f"L2 flushed before every step ({sum(kv_bytes) / args.steps / 1e3:.0f} KB "
                   f"of packed K/V per step, L2 {l2_bytes / 1e6:.0f} MB): a write of twice the "
                   "L2 size outside each step's events; ms_per_step sums the steps' event times"
                   if flush_l2 else
                   f"inputs larger than L2: {sum(kv_bytes) / args.steps / 1e6:.0f} MB of packed "
                   f"K/V read per step per GPU (L2 {l2_bytes / 1e6:.0f} MB)"),
            "step": ("kvq_decode_step: quantize-on-write of 1 token/seq inside the split-K "
                     "decode attention kernel" + (", then the LSE merge" if parts > 1 else "")
                     if wl.append else
                     "split-K decode attention over the FP16/INT4/INT2 segments" +
                     (" + LSE merge" if parts > 1 else "")
                     if wl.chunk_tokens else
                     "split-K decode attention over the prefilled cache" +
                     (" + LSE merge" if parts > 1 else ""))}),
        "kv_read_gbs": sum(kv_bytes) / (ms / 1e3) / 1e9 * world,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "traffic": recorded_traffic(wl.name), "kernel": split_kernel_name(wl),
                     "alg_bytes_per_launch": split_bytes / len(last_step),
                     "avg_launch_us": split_total_us / len(last_step),
                     "launches_timed": len(last_step)},
        "e2e": {"value": B * args.steps * world / (e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "kvq_decode_step (append workloads) or kvq_decode_attention through the "
                        "Python binding; pinned host buffers, one input and one result copy per "
                        "step, double-buffered on two copy streams"},
        # device latency of one step and of its kernel(s), and of the prefill
        # quantize of the whole context (for the 256-token tiny workload, the
        # latency-bound case, these are the figures that matter)
        "latency_us": {"step": ms / args.steps * 1e3,
                       "decode_kernels": split_total_us / len(last_step),
                       **({"prefill_quantize": prefill["us"]} if prefill else {})},
        "gpu_launches": launches_per_step * args.steps,
        **({"prefill_quantize": {**prefill, "frac": prefill["gbs"] / peak}} if prefill else {}),
        **({"oaken_outliers": outlier_stats} if outlier_stats else {}),
        **({"chunk_reorder": {**chunk_timing, "frac": chunk_timing["reorder_gbs"] / peak}}
           if chunk_timing else {}),
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        if wl.chunk_tokens:
            line["cpu_baseline"] = cpu_baseline_mixed(wl, k, v, qs[0], args.cpu_seconds, wlr)
        else:
            line["cpu_baseline"] = cpu_baseline(wl, k, v, kn[0, 0] if kn is not None else None,
                                                kn[0, 1] if kn is not None else None, qs[0],
                                                args.cpu_seconds)
    return line


def main():
    args = parse_args()
    import workloads
    wl = workloads.WORKLOADS[args.workload]
    if args.batch > 0:
        wl = wl.scaled(batch=args.batch)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_kvq(args, wl, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
