"""Host-side logic of bench.py, on CPU: rank reduction over gloo (world size 2),
clock-sample parsing, the algorithmic work counts, and the reference arm."""

import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import oracle
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    total, mx = bench.reduce_over_ranks(10.0 * (rank + 1), 1.5 + rank, world)
    out[rank] = (total, mx)
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == (30.0, 2.5)


def test_reduce_single_rank_is_identity():
    assert bench.reduce_over_ranks(3.0, 4.0, 1) == (3.0, 4.0)


def test_clock_summary_parsing():
    c = bench.ClockSampler(0)
    c.proc = object()
    c.window = (100.0, 101.0)
    row = "2026/12/02 10:00:00.000, 0, {sm}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, {cap}"
    c.rows = [(99.0, row.format(sm=100, cap="Not Active")),
              (100.2, row.format(sm=1800, cap="Active")),
              (100.5, row.format(sm=1900, cap="Not Active")),
              (100.9, row.format(sm=1700, cap="Not Active"))]
    s = c.summary()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"] and s["samples"] == 3


def test_work_counts_match_oracle():
    for name in ("prefill_small", "prefill_gpt2", "prefill_llama8b", "prefill_llama8b_nc"):
        w = synth.WORKLOADS[name]
        assert bench.prefill_flops(w) == oracle.prefill_flops(w.B, w.Hq, w.N, w.d, w.causal)
    w = synth.WORKLOADS["decode_paged_t4"]
    case = synth.decode_inputs(2, w.T, w.Hq, w.Hkv, w.d, 0, 0, seed=1, paged=True, lengths=[20, 40])
    kv_bytes = (24 + 44) * w.Hkv * w.d * 4
    assert bench.decode_bytes(case, bench._shrink(w, 2)) == kv_bytes + 2 * 2 * 4 * 64 * 128 * 2 + 2 * 64 * 4 * 4 + 8 + (2 + 3) * 4


def test_reference_arm_runs_on_cpu():
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-step-budget", "0.05"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == "TFLOP/s"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""
