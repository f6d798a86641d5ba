"""Benchmark: ring-attention forward TFLOP/s on B200 (bf16), % of tensor peak; merge HBM GB/s;
backward TFLOP/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one ra_ring_forward call over the whole workload (default: batch 1, 8 heads,
1M tokens, d = 128, bf16, causal, zig-zag over 16 virtual positions, emitting O and lse);
the call is one kernel launch that runs every step of the path (layout walk, Q/K/V staging,
QK^T, causal predicate, online softmax, PV, finalise). Inputs are synthetic (seeded i.i.d.
N(0, 1)), resident in HBM and 6.4 GB in total, so they exceed the 126 MB L2 between steps.

Rank 0 prints one JSON line. With N > 1 (torchrun) every rank runs an independent replica
of the workload with its own seed (weak scaling, no collective on the data path); time is
the max over ranks of CUDA-event time.

Sub-measurements in the same line: "merge" (ra_merge, HBM-bound) and "backward"
(ra_ring_backward on the 128K-token zig-zag workload).

--impl reference times the fp64 CPU oracle on this host's cores on a bounded sample of the
same workload (rows of one head against all their visible keys) in the same unit.
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

def oracle_sample(w, seconds: float, seed: int = 0):
    """Times the fp64 oracle on query rows of one head until ~`seconds` of CPU work.

    Returns (tflops, elapsed_s, n_rows, threads). Work is counted with the same rule as the
    GPU metric: 4 d FLOPs per visible (query, key) pair.
    """
    import numpy as np
    import torch

    import oracle
    from sequence_softmax_b200.inputs import make_qkv

    g = torch.Generator().manual_seed(1000 + seed)
    q, k, v = make_qkv(1, 1, w.N, w.d, w.torch_dtype, seed=w.seed, device="cpu", q_scale=w.q_scale)
    qn, kn, vn = (t.float().numpy() for t in (q, k, v))
    threads = torch.get_num_threads()
    done_flops, t_total, rows_done = 0, 0.0, 0
    batch = 8
    while t_total < seconds:
        rows = torch.randint(0, w.N, (batch,), generator=g).numpy()
        t0 = time.perf_counter()
        oracle.attention(qn, kn, vn, w.scale, w.causal, rows=rows, row_block=batch)
        t_total += time.perf_counter() - t0
        vis = (rows + 1) if w.causal else np.full(batch, w.N)
        done_flops += int(4 * w.d * vis.sum())
        rows_done += batch
        if t_total < seconds / 4:
            batch = min(batch * 2, 256)
    return done_flops / t_total / 1e12, t_total, rows_done, threads


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def run_reference(a, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = max(2.0, min(a.cpu_seconds, 20.0) / max(1, a.steps))
    for _ in range(a.warmup):
        oracle_sample(w, min(1.0, per_step))
    vals, secs, rows = [], 0.0, 0
    for s in range(a.steps):
        tf, el, nr, threads = oracle_sample(w, per_step, seed=s + 1)
        vals.append(tf)
        secs += el
        rows += nr
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": secs / a.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} query rows of head 0 against all their visible keys "
                                   f"(fp64 NumPy oracle), {secs:.1f} s total"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
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
    achieved = flops / (ms_step / 1e3) / 1e12  # one kernel launch per step
    peak = pk["bf16_tflops"]
    traffic = stored_traffic("attn_fwd_tc", w.name, w.B * w.H * w.N)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"{pk['source']} bf16 burst",
                     "frac_of_sustained": achieved / pk.get("bf16_tflops_sustained", peak),
                     "frac_of_datasheet_2250": achieved / 2250.0,
                     "kernel": "attn_fwd_tc_kernel<128>"},
        "clocks": clk.summary(),
        "gpu_launches": a.steps,
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
        tf, el, nr, threads = oracle_sample(w, a.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": f"{nr} random query rows of head 0 against all their visible keys, "
                                          f"fp64 NumPy oracle, {el:.1f} s (host has {cpu_cores()} cores)"}
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
    steps = max(1, min(a.steps, 3))
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


if __name__ == "__main__":
    main()
