"""Host-side logic of bench.py on the CPU: the max-over-ranks timing with two gloo ranks,
per-rank replica inputs, and the reference arm (the fp64 oracle timed on host cores)."""

import json
import os
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from sequence_softmax_b200.inputs import WORKLOADS, workload_qkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    port = 29500 + os.getpid() % 1000
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out[0] == out[1] == 15.0


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1, None) == 3.25


def test_rank_replicas_differ_but_share_shape():
    w = WORKLOADS["seq4k-d64-noncausal-8chunks"]
    small = type(w)(w.name + "-tiny", 1, 2, 64, 64, "bf16", False, 2, "contiguous", w.seed)
    a = workload_qkv(small, device="cpu", batch_offset=0)
    b = workload_qkv(small, device="cpu", batch_offset=1)
    assert a[0].shape == b[0].shape and not torch.equal(a[0], b[0])


def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "seq4k-d64-noncausal-8chunks", "--steps", "1", "--warmup", "0",
                        "--cpu-seconds", "1"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""
