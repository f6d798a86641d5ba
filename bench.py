"""Benchmark: ring-attention forward TFLOP/s on B200 (bf16), % of tensor peak; merge HBM GB/s;
backward TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one ra_ring_forward call over the whole workload (default: batch 1, 8 heads,
1M tokens, d = 128, bf16, causal, zig-zag over 16 virtual positions, emitting O and lse);
the call is three kernel launches: two short passes that bound each head's key norms (0.04% of
the step) and the attention kernel that runs every step of the path (layout walk, Q/K/V
staging, QK^T, causal predicate, online softmax, PV, finalise). Inputs are synthetic (seeded i.i.d.
N(0, 1)), resident in HBM and 6.4 GB in total, so they exceed the 126 MB L2 between steps.

Rank 0 prints one JSON line. With N > 1 (torchrun), the default (--multi ring) runs the
pages' own partition of the same workload over the N GPUs: each rank holds the tokens of one
virtual ring position (zig-zag: chunks r and 2N-1-r), keeps its queries, and K||V rotates
around the ring over NCCL while ra_partial_fold folds each block into the running state
("Ring Attention 논문 분석", listing ring_attention_forward). The total work is fixed (strong
scaling). --multi replicas instead runs an independent replica of the workload per rank
(weak scaling, no collective on the data path). Time is the max over ranks of CUDA-event
time.

Sub-measurements in the same line: "merge" (ra_merge, HBM-bound) and "backward"
(ra_ring_backward on the 128K-token zig-zag workload).

--impl reference times the fp64 CPU oracle on this host's cores on a bounded sample of the
same workload (rows of one head against all their visible keys) in the same unit.

--report prints one JSON line per named workload (the toy, 4K non-causal and its Q x 4
variant, 32K causal, 128K zig-zag and striped, 1M zig-zag) and per merge workload (n = 2 and
n = 16 partial states): device time, TFLOP/s (or GB/s) and roofline fractions, clocks, the
error against the fp64 oracle (every row on the small workloads, sampled rows on the long
ones) and the oracle's CPU time (measured in full on the small workloads, measured on the
sampled rows and extrapolated by visible pairs on the long ones).
"""

from __future__ import annotations

import argparse
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

METRIC = "ring-attn fwd TFLOP/s (bf16, 1 B200), % of tensor peak; merge HBM GB/s"
PROFILE_JSON = os.path.join(ROOT, "profiles", "counters.json")
KERNEL_SOURCES = {
    "attn_fwd_tc": ["sequence_softmax_b200/csrc/attn_tc.cuh", "sequence_softmax_b200/csrc/common.cuh"],
    "merge": ["sequence_softmax_b200/csrc/merge.cuh"],
    "attn_bwd_dkdv_tc": ["sequence_softmax_b200/csrc/bwd_tc.cuh", "sequence_softmax_b200/csrc/bwd.cuh",
                         "sequence_softmax_b200/csrc/common.cuh"],
    "attn_bwd_dq_tc": ["sequence_softmax_b200/csrc/bwd_dq_tc.cuh", "sequence_softmax_b200/csrc/bwd.cuh",
                       "sequence_softmax_b200/csrc/common.cuh"],
}
BWD_WORKLOAD = "seq128k-d128-causal-zigzag16"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-merge", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--merge-rows", type=int, default=8 * (1 << 20),
                    help="rows of the merge workload (smaller values for profiler captures)")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--bwd-workload", default=BWD_WORKLOAD)
    ap.add_argument("--bwd-steps", type=int, default=3)
    ap.add_argument("--multi", choices=["ring", "replicas"], default="ring",
                    help="with N > 1 GPUs: the ring over NCCL (one virtual position per rank) or replicas")
    ap.add_argument("--report", action="store_true", help="one JSON line per named workload (see the docstring)")
    ap.add_argument("--report-rows", type=int, default=512,
                    help="sampled query rows per head checked against the oracle on the long workloads")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def kernel_src_sha(kernel: str) -> str:
    """Hash of the sources a kernel is built from (stored next to its ncu counters)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel: str, workload: str, units: float):
    """DRAM bytes per launch from the committed ncu counters, if taken on the current source."""
    if not os.path.exists(PROFILE_JSON):
        return None
    with open(PROFILE_JSON) as f:
        prof = json.load(f)
    e = prof.get(kernel)
    if not e or e.get("kernel_src_sha") != kernel_src_sha(kernel):
        return None
    # traffic per unit processed in the captured case, scaled to this launch's units
    return e["dram_bytes"] / e["units"] * units if e.get("workload") != workload else e["dram_bytes"]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------
# CPU oracle sample (the reference arm and the cpu_baseline of the GPU arm).
# ------------------------------------------------------------------------------------------

ORACLE_ROWS_PER_CALL = 256  # query rows per oracle call: one fixed sample size for both arms


def blas_threads() -> int:
    """Host threads the oracle's BLAS runs on: the cores this process may use."""
    return cpu_cores()


def oracle_sample(w, calls: int = 0, seconds: float = 0.0, seed: int = 0):
    """Times the fp64 oracle, as it stands, on fixed-size samples of one head's query rows.

    Every call evaluates ORACLE_ROWS_PER_CALL random query rows against all their visible
    keys (``oracle.attention`` with its default row blocks), so its fixed per-call cost
    (widening the head's K and V to fp64) is amortised the same way in every measurement.
    Runs ``calls`` calls, or as many as fill ``seconds``. BLAS threads are pinned to the
    cores this process may use. Work is counted with the GPU metric's rule: 4 d FLOPs per
    visible (query, key) pair.

    Returns (tflops, elapsed_s, n_rows, threads, n_calls).
    """
    import numpy as np
    import torch
    from threadpoolctl import threadpool_limits

    import oracle
    from sequence_softmax_b200.inputs import make_qkv

    g = torch.Generator().manual_seed(1000 + seed)
    q, k, v = make_qkv(1, 1, w.N, w.d, w.torch_dtype, seed=w.seed, device="cpu", q_scale=w.q_scale)
    qn, kn, vn = (t.float().numpy() for t in (q, k, v))
    threads = blas_threads()
    done_flops, t_total, rows_done, n = 0, 0.0, 0, 0
    R = min(ORACLE_ROWS_PER_CALL, w.N)
    with threadpool_limits(limits=threads):
        while (calls and n < calls) or (not calls and (t_total < seconds or n == 0)):
            rows = torch.randint(0, w.N, (R,), generator=g).numpy()
            t0 = time.perf_counter()
            oracle.attention(qn, kn, vn, w.scale, w.causal, rows=rows)
            t_total += time.perf_counter() - t0
            vis = (rows + 1) if w.causal else np.full(R, w.N)
            done_flops += int(4 * w.d * vis.sum())
            rows_done += R
            n += 1
    return done_flops / t_total / 1e12, t_total, rows_done, threads, n


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(a, w):
    """The reference arm: the fp64 oracle on this host's cores, one fixed-size sample of the
    workload per step (rank 0 only; other ranks exit without work)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    oracle_sample(w, calls=a.warmup, seed=0)
    tf, secs, rows, threads, n = oracle_sample(w, calls=a.steps, seed=1)
    line = {
        "impl": "reference", "metric": METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} calls x {ORACLE_ROWS_PER_CALL} random query rows of head 0 against all "
                                   f"their visible keys (fp64 NumPy oracle, BLAS pinned to {threads} threads), "
                                   f"{secs:.1f} s total"},
        "e2e": {"value": tf, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time: every rank contributes its own CUDA-event time."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(w):
    return {"workload": w.name, "batch": w.B, "heads": w.H, "seq_len": w.N, "head_dim": w.d,
            "causal": w.causal, "layout": w.layout, "n_chunks": w.n_chunks, "emit_lse": w.emit_lse,
            "flops_per_step": w.flops(), "l2": "inputs exceed L2 (Q, K, V, O are GBs): no flush needed"}


# ------------------------------------------------------------------------------------------
# GPU arm.
# ------------------------------------------------------------------------------------------

def main():
    a = parse()
    from sequence_softmax_b200.inputs import BENCH_WORKLOAD, WORKLOADS
    w = WORKLOADS[a.workload or BENCH_WORKLOAD]
    if a.impl == "reference":
        return run_reference(a, w)
    if a.report:
        return run_report(a)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and a.multi == "ring":
        return run_ring(a, w)
    return run_single(a, w)


def run_single(a, w):
    """One ra_ring_forward call per step on each rank's own replica of the workload."""
    import torch
    import torch.distributed as dist

    from sequence_softmax_b200 import binding
    from sequence_softmax_b200.inputs import workload_qkv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    pk = peaks()

    # Inputs resident in HBM: a per-rank replica of the workload (weak scaling).
    q, k, v = workload_qkv(w, device=dev, batch_offset=rank)
    out = torch.empty_like(q)
    lse = torch.empty(w.B, w.H, w.N, device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream()

    def step():
        binding.ring_forward(q, k, v, w.n_chunks, w.causal, w.layout, out=out, lse=lse)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    if binding.get_device_error() != binding.RA_OK:
        raise RuntimeError("device error during warm-up")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        start.record(stream)
        for _ in range(a.steps):
            step()
        end.record(stream)
        barrier()
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    if binding.get_device_error() != binding.RA_OK:
        raise RuntimeError("device error during the timed region")
    ms_step = ms / a.steps
    flops = w.flops()
    value = world * flops * a.steps / (ms / 1e3) / 1e12
    # the attention kernel's rate over the whole step: the two key-bound passes (0.04% of it)
    # count against it, so the kernel's own rate is slightly higher
    achieved = flops / (ms_step / 1e3) / 1e12
    peak = pk["bf16_tflops"]
    traffic = stored_traffic("attn_fwd_tc", w.name, w.B * w.H * w.N)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(w), parallelism=f"replicas{world}" if world > 1 else "single"),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{pk['source']} bf16 burst",
                     "frac_of_sustained": achieved / pk.get("bf16_tflops_sustained", peak),
                     "frac_of_datasheet_2250": achieved / 2250.0,
                     "kernel": "attn_fwd_tc_kernel<128>"},
        "clocks": clk.summary(),
        "gpu_launches": 3 * a.steps,
    }
    del out

    if not a.no_merge:
        line["merge"] = bench_merge(binding, torch, dev, pk, a)

    if not a.no_e2e:
        line["e2e"] = bench_e2e(binding, torch, w, q, k, v, world, a)
    del q, k, v
    torch.cuda.empty_cache()

    if not a.no_backward:
        line["backward"] = bench_backward(binding, torch, dev, pk, a, rank, world)
        torch.cuda.empty_cache()

    if rank == 0 and not a.no_cpu_baseline and world == 1:
        tf, el, nr, threads, n = oracle_sample(w, seconds=a.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": f"{n} calls x {ORACLE_ROWS_PER_CALL} random query rows of head 0 against "
                                          f"all their visible keys, fp64 NumPy oracle, BLAS pinned to {threads} "
                                          f"threads, {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def bench_merge(binding, torch, dev, pk, a):
    """ra_merge on 2 fp32 partial states shaped like the 1M-token workload -> bf16 O + fp32 lse."""
    n, rows, d = 2, a.merge_rows, 128
    g = torch.Generator(device=dev).manual_seed(99)
    o_parts = torch.randn(n, rows, d, device=dev, generator=g)
    lse_parts = torch.randn(n, rows, device=dev, generator=g) + 10.0
    out = torch.empty(rows, d, device=dev, dtype=torch.bfloat16)
    lse = torch.empty(rows, device=dev, dtype=torch.float32)
    for _ in range(3):
        binding.merge(o_parts, lse_parts, out=out, lse=lse)
    iters = 20
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(iters):
        binding.merge(o_parts, lse_parts, out=out, lse=lse)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / iters
    nbytes = n * rows * (4 * d + 4) + rows * (2 * d + 4)
    gbs = nbytes / (ms / 1e3) / 1e9
    traffic = stored_traffic("merge", f"merge-n2-rows{rows}-d128", rows)
    return {"value": gbs, "unit": "GB/s", "ms": ms, "bytes": nbytes, "launches": iters,
            "workload": f"n={n} fp32 partials, rows={rows}, d={d} -> bf16 O + fp32 lse",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": traffic,
                         "peak_source": f"{pk['source']} copy"}}


def bench_backward(binding, torch, dev, pk, a, rank, world=1):
    """ra_ring_backward on its own workload: dQ, dK, dV of the forward's output for a seeded
    upstream gradient. FLOPs = 2.5x the forward's (five GEMMs per visible pair instead of two).
    With N ranks each runs its own replica; the step time is the slowest rank's and the value
    is the whole job's throughput (weak scaling, as the headline)."""
    from sequence_softmax_b200.inputs import WORKLOADS, make_qkv, workload_qkv
    w = WORKLOADS[a.bwd_workload]
    q, k, v = workload_qkv(w, device=dev, batch_offset=rank)
    do = make_qkv(w.B, w.H, w.N, w.d, w.torch_dtype, seed=1000 + rank, device=dev)[0]
    o, lse = binding.ring_forward(q, k, v, w.n_chunks, w.causal, w.layout)
    ws = torch.empty(binding.ring_backward_workspace_bytes(q.dtype, w.B, w.H, w.N, w.d), device=dev,
                     dtype=torch.uint8)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))

    def step():
        binding.ring_backward(q, k, v, o, do, lse, w.n_chunks, w.causal, w.layout, workspace=ws, out=grads)

    step()
    torch.cuda.synchronize()
    if binding.get_device_error() != binding.RA_OK:
        raise RuntimeError("device error in the backward warm-up")
    stream = torch.cuda.current_stream()
    # one ra_ring_backward call per timed step, on the stream its kernels are launched on
    kernel_ms = []
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    for _ in range(a.bwd_steps):
        s.record(stream)
        step()
        e.record(stream)
        e.synchronize()
        kernel_ms.append(s.elapsed_time(e))
    if binding.get_device_error() != binding.RA_OK:
        raise RuntimeError("device error in the timed backward")
    ms = max_over_ranks(statistics.median(kernel_ms), world, dev)
    flops = 2.5 * w.flops()
    tf = world * flops / (ms / 1e3) / 1e12
    per_gpu = flops / (ms / 1e3) / 1e12
    peak = pk["bf16_tflops"]
    parts = [stored_traffic(k, w.name, w.B * w.H * w.N) for k in ("attn_bwd_dkdv_tc", "attn_bwd_dq_tc")]
    traffic = None if any(t is None for t in parts) else sum(parts)
    return {"value": tf, "unit": "TFLOP/s", "ms_per_step": ms, "steps": a.bwd_steps,
            "workload": workload_config(w), "flops_per_step": flops,
            "gpu_launches_per_step": 3,
            "note": "one step = ra_ring_backward: D, the dK/dV kernel, the dQ kernel",
            "roofline": {"bound": "tensor", "achieved": per_gpu, "peak": peak, "unit": "TFLOP/s",
                         "frac": per_gpu / peak,
                         "traffic": traffic, "peak_source": f"{pk['source']} bf16 burst",
                         "kernel": "attn_bwd_dkdv_tc_kernel<128> + attn_bwd_dq_tc_kernel<128> (+ D, <1% of the step)"},
            "wall_s": time.time() - t0}


def bench_e2e(binding, torch, w, q, k, v, world, a):
    """The same metric through the public call with pinned host buffers (copies timed)."""
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
    lh = torch.empty(w.B, w.H, w.N, dtype=torch.float32, pin_memory=True)
    steps = a.steps
    binding.ring_forward(qh, kh, vh, w.n_chunks, w.causal, w.layout, out=oh, lse=lh)  # warm
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        binding.ring_forward(qh, kh, vh, w.n_chunks, w.causal, w.layout, out=oh, lse=lh)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + lh.numel() * lh.element_size()
    return {"value": world * w.flops() / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


# ------------------------------------------------------------------------------------------
# N > 1: the ring across GPUs.
# ------------------------------------------------------------------------------------------

def position_tokens(t, segs):
    """The tokens of one virtual ring position (segments (tok0, stride, count)) of a
    [B, H, N, d] tensor, in increasing token order: [B, H, N / W, d], contiguous."""
    import torch
    return torch.cat([t[:, :, t0:t0 + stride * n:stride] for (t0, stride, n) in segs], dim=2).contiguous()


class CountingKernels:
    """The binding's entry points, counting the library launches made through them."""

    def __init__(self, binding):
        self._binding = binding
        self.launches = 0

    def __getattr__(self, name):
        fn = getattr(self._binding, name)

        def call(*args, **kwargs):
            self.launches += 1  # partial_fold and key_norm_max: one kernel launch per call
            return fn(*args, **kwargs)
        return call


def run_ring(a, w):
    """The workload's attention over the N ranks as the pages partition it: rank r holds the
    tokens of virtual position r (the workload's layout over N positions), keeps its queries,
    and K||V rotates around the ring over NCCL (ring_dist.ring_forward_dist). The total work
    is the workload's (strong scaling)."""
    import datetime

    import torch
    import torch.distributed as dist

    from sequence_softmax_b200 import binding
    from sequence_softmax_b200.inputs import workload_qkv
    from sequence_softmax_b200.ring_dist import position_segments, ring_forward_dist

    world = int(os.environ["WORLD_SIZE"])
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    pk = peaks()

    # The whole problem, drawn identically on every rank; each rank keeps its position's tokens.
    q, k, v = workload_qkv(w, device=dev)
    segs = position_segments(w.layout, w.N, world, rank)
    ql, kl, vl = (position_tokens(t, segs) for t in (q, k, v))
    del q, k, v
    torch.cuda.empty_cache()
    kern = CountingKernels(binding)

    def step():
        return ring_forward_dist(ql, kl, vl, w.N, w.layout, w.causal, kernels=kern)

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    if binding.get_device_error() != binding.RA_OK:
        raise RuntimeError("device error during warm-up")
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    kern.launches = 0
    with ClockSampler(local) as clk:
        dist.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(a.steps):
            step()
        end.record(stream)
        dist.barrier()
        torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end), world, dev)
    launches = torch.tensor([kern.launches], device=dev, dtype=torch.int64)
    dist.all_reduce(launches)
    if binding.get_device_error() != binding.RA_OK:
        raise RuntimeError("device error during the timed region")
    ms_step = ms / a.steps
    flops = w.flops()
    value = flops / (ms_step / 1e3) / 1e12
    per_gpu = value / world
    peak = pk["bf16_tflops"]
    cfg = dict(workload_config(w), n_chunks=world, parallelism=f"ring{world}",
               partition=f"rank r holds virtual position r of {world} ({w.layout}); K||V rotates over NCCL")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "roofline": {"bound": "tensor", "achieved": per_gpu, "peak": peak, "unit": "TFLOP/s",
                     "frac": per_gpu / peak, "traffic": None, "peak_source": f"{pk['source']} bf16 burst",
                     "note": "per-GPU step throughput of the ring (ra_partial_fold's attn_fwd_tc_kernel<128> "
                             "launches, one ra_key_norm_max per folded K segment, and the exchange), "
                             "not one launch",
                     "kernel": "attn_fwd_tc_kernel<128> via ra_partial_fold"},
        "clocks": clk.summary(),
        "gpu_launches": int(launches.item()),
    }
    if not a.no_e2e:
        qh, kh, vh = (t.cpu().pin_memory() for t in (ql, kl, vl))
        qd, kd, vd = torch.empty_like(ql), torch.empty_like(kl), torch.empty_like(vl)
        oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
        lh = torch.empty(qh.shape[:3], dtype=torch.float32, pin_memory=True)

        def e2e_step():
            for d_, h_ in ((qd, qh), (kd, kh), (vd, vh)):
                d_.copy_(h_, non_blocking=True)
            o, l = ring_forward_dist(qd, kd, vd, w.N, w.layout, w.causal)
            oh.copy_(o, non_blocking=True)
            lh.copy_(l, non_blocking=True)

        e2e_step()
        dist.barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(a.steps):
            e2e_step()
        end.record(stream)
        dist.barrier()
        torch.cuda.synchronize()
        ems = max_over_ranks(start.elapsed_time(end), world, dev) / a.steps
        h2d = world * sum(t.numel() * t.element_size() for t in (qh, kh, vh))
        d2h = world * (oh.numel() * oh.element_size() + lh.numel() * lh.element_size())
        line["e2e"] = {"value": flops / (ems / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ems,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": a.steps,
                       "note": "bytes summed over all ranks"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()


# ------------------------------------------------------------------------------------------
# --report: one line per named workload.
# ------------------------------------------------------------------------------------------

REPORT_WORKLOADS = ["toy-4dev-seq32-d16", "seq4k-d64-noncausal-8chunks", "seq4k-d64-noncausal-8chunks-qx4",
                    "seq32k-d128-causal-contig8", "seq128k-d128-causal-zigzag16", "seq128k-d128-causal-striped16",
                    "seq1m-d128-causal-zigzag16"]
REPORT_MERGES = [(2, 8 * (1 << 20), 128), (16, 32 * (1 << 17), 128)]
L2_FLUSH_BYTES = 256 << 20  # written between timed iterations: twice the 126 MB L2


def _time_each(fn, n_iter, flush, stream, torch):
    """Median CUDA-event time of fn over n_iter iterations, L2 flushed before each."""
    times = []
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(n_iter):
        flush.zero_()
        s.record(stream)
        fn()
        e.record(stream)
        e.synchronize()
        times.append(s.elapsed_time(e))
    return statistics.median(times), times


def run_report(a):
    import numpy as np
    import torch
    from threadpoolctl import threadpool_limits

    import oracle
    from sequence_softmax_b200 import binding
    from sequence_softmax_b200.inputs import WORKLOADS, sample_rows, workload_qkv

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pk = peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    threads = blas_threads()
    for name in REPORT_WORKLOADS:
        w = WORKLOADS[name]
        q, k, v = workload_qkv(w, device=dev)
        out = torch.empty_like(q)
        lse = torch.empty(w.B, w.H, w.N, device=dev, dtype=torch.float32)

        def step():
            binding.ring_forward(q, k, v, w.n_chunks, w.causal, w.layout, out=out, lse=lse)

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        if binding.get_device_error() != binding.RA_OK:
            raise RuntimeError(f"{name}: device error during warm-up")
        n_iter = max(a.steps, 10) if w.N < (1 << 20) else max(a.steps, 3)
        with ClockSampler(0) as clk:
            ms, _ = _time_each(step, n_iter, flush, stream, torch)
        if binding.get_device_error() != binding.RA_OK:
            raise RuntimeError(f"{name}: device error in the timed region")
        tf = w.flops() / (ms / 1e3) / 1e12
        qn, kn, vn = (t.float().cpu().numpy() for t in (q, k, v))
        total_pairs = w.B * w.H * w.visible_pairs()
        with threadpool_limits(limits=threads):
            if w.N <= 4096:
                t0 = time.perf_counter()
                o_ref, l_ref = oracle.attention(qn, kn, vn, w.scale, w.causal)
                cpu_s = time.perf_counter() - t0
                og, lg = out.float().cpu().numpy(), lse.cpu().numpy()
                oracle_info = {"mode": "full", "cpu_s": cpu_s, "rows_per_head": w.N}
            else:
                rows = sample_rows(w.N, w.n_chunks, w.layout, count=a.report_rows)
                t0 = time.perf_counter()
                o_ref, l_ref = oracle.attention(qn, kn, vn, w.scale, w.causal, rows=rows)
                cpu_s = time.perf_counter() - t0
                ridx = torch.as_tensor(rows, device=dev)
                og, lg = out[:, :, ridx].float().cpu().numpy(), lse[:, :, ridx].cpu().numpy()
                sampled = w.B * w.H * int(((rows + 1) if w.causal else np.full(len(rows), w.N)).sum())
                oracle_info = {"mode": "sampled rows, time extrapolated by visible pairs", "cpu_s_sampled": cpu_s,
                               "rows_per_head": int(len(rows)), "cpu_s": cpu_s * total_pairs / sampled}
        oracle_info.update(cores=threads, kind="fp64 NumPy oracle")
        err = np.abs(og - o_ref)
        fin = np.isfinite(l_ref)
        lerr = float(np.abs(lg[fin] - l_ref[fin]).max()) if fin.any() else 0.0
        line = {"report": name, "config": workload_config(w), "dtype": w.dtype, "ms": ms, "iters": n_iter,
                "TFLOP/s": tf, "frac_of_burst": tf / pk["bf16_tflops"],
                "frac_of_sustained": tf / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                "peak_source": pk["source"], "l2": "flushed before every timed iteration",
                "clocks": clk.summary(), "max_abs_err": float(err.max()), "mean_abs_err": float(err.mean()),
                "lse_max_abs_err": lerr, "oracle": oracle_info,
                "gpu_over_oracle": oracle_info["cpu_s"] / (ms / 1e3)}
        print(json.dumps(line), flush=True)
        del q, k, v, out, lse
        torch.cuda.empty_cache()

    for n, rows, d in REPORT_MERGES:
        g = torch.Generator(device=dev).manual_seed(100 + n)
        o_parts = torch.randn(n, rows, d, device=dev, generator=g)
        # lse ~ N(ln Lk, 1) for KV chunks of Lk = 8192 keys, 1% of the entries -inf (chunks
        # wholly in a row's future)
        lse_parts = torch.randn(n, rows, device=dev, generator=g) + float(np.log(8192.0))
        lse_parts[torch.rand(n, rows, device=dev, generator=g) < 0.01] = float("-inf")
        out = torch.empty(rows, d, device=dev, dtype=torch.bfloat16)
        lse = torch.empty(rows, device=dev, dtype=torch.float32)

        def mstep():
            binding.merge(o_parts, lse_parts, out=out, lse=lse)

        for _ in range(3):
            mstep()
        torch.cuda.synchronize()
        with ClockSampler(0) as clk:
            ms, _ = _time_each(mstep, max(a.steps, 10), flush, stream, torch)
        nbytes = n * rows * (4 * d + 4) + rows * (2 * d + 4)
        gbs = nbytes / (ms / 1e3) / 1e9
        sr = torch.randint(0, rows, (4096,), generator=torch.Generator().manual_seed(7)).unique()
        sri = sr.to(dev)
        op, lp = o_parts[:, sri].cpu().numpy(), lse_parts[:, sri].cpu().numpy()
        with threadpool_limits(limits=threads):
            t0 = time.perf_counter()
            o_ref, l_ref = oracle.merge(op, lp)
            cpu_s = (time.perf_counter() - t0) * rows / len(sr)
        err = np.abs(out[sri].float().cpu().numpy() - o_ref)
        fin = np.isfinite(l_ref)
        line = {"report": f"merge-n{n}-rows{rows}-d{d}", "ms": ms, "GB/s": gbs, "bytes": nbytes,
                "frac_of_hbm": gbs / pk["hbm_gbs"], "peak_source": pk["source"],
                "l2": "flushed before every timed iteration", "clocks": clk.summary(),
                "max_abs_err": float(err.max()), "mean_abs_err": float(err.mean()),
                "lse_max_abs_err": float(np.abs(lse[sri].cpu().numpy()[fin] - l_ref[fin]).max()),
                "oracle": {"mode": f"{len(sr)} sampled rows, time extrapolated by rows", "cpu_s": cpu_s,
                           "cores": threads, "kind": "fp64 NumPy oracle"},
                "gpu_over_oracle": cpu_s / (ms / 1e3)}
        print(json.dumps(line), flush=True)
        del o_parts, lse_parts, out, lse
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
