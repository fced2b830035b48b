"""Benchmark: prefill attention TFLOP/s and KV-cache decode GB/s on B200.

One step is one pass of the whole hot path on the Llama-3.1-8B attention-layer
shapes (Hq=32, Hkv=8, d=128, bf16 in, fp32 accumulation):

* causal prefill, B=4, N=4096 (attn_prefill, tcgen05 kernel);
* a decode step for B=16 sequences whose cache lengths are uniform in
  [1024, 32768]: kv_append of one new token per sequence, then split-KV
  attn_decode (split kernel + log-sum-exp combine) against the contiguous cache.

``value`` is the prefill throughput in TFLOP/s (algorithmic FLOPs: 4 d per
visible query-key pair, masked work not credited) over the prefill kernel's own
device time; the ``decode`` object gives the KV-cache GB/s (algorithmic bytes:
every valid K and V byte plus q, o, lse and lengths) over the attn_decode
device time.  Both are whole-job figures: summed over ranks, divided by the
slowest rank's time.  Inputs (192 MiB prefill, 1 GB cache) exceed the 126 MB
L2, so no explicit flush is needed.

The default run then times every configuration alone -- the oracle-sized causal
prefill (B1 Hq4 Hkv2 N256 d64), the GPT-2-small prefill (B8 H12 N1024 d64),
the Llama-3.1-8B causal N=4096 and non-causal N=8192 prefills, the contiguous
decode and the paged decode with 1 and 4 new tokens -- each with its own
roofline object under ``configs`` and its own clock record (L2 flushed before
each launch where the inputs fit in L2).

``--impl reference`` times the fp64 CPU oracle on bounded samples of the same
workload instead (rank 0 only).  ``--workload`` selects another shape set for
manual runs; the default is the one described above.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill attention TFLOP/s and decode KV-cache GB/s, % of B200 roofline"

# prefill workload / decode workload pairs (names from synth.WORKLOADS)
WORKLOAD_SETS = {
    "llama8b_layer": ("prefill_llama8b", "decode_contig"),
    "gpt2_prefill_paged_decode": ("prefill_gpt2", "decode_paged"),
    "llama8b_nc_paged_t4": ("prefill_llama8b_nc", "decode_paged_t4"),
    # the same layer with an FP8 (e4m3, per-KV-head scales) KV cache
    "llama8b_layer_fp8": ("prefill_llama8b", "decode_contig_fp8"),
    "llama8b_paged_fp8": ("prefill_llama8b", "decode_paged_fp8"),
    # prefill against an existing cache: 512-token prompt chunks on cached 4K..16K prefixes,
    # through attn_prefill_cache (the prefill kernel) or attn_decode (split-KV, row-tiled)
    "llama8b_prefill_cache": ("prefill_llama8b", "prefill_chunk_paged"),
    "llama8b_chunked_prefill": ("prefill_llama8b", "prefill_chunk_paged"),
    # eight new tokens per decode step: the tensor-core split kernel (64 rows per KV head)
    "llama8b_paged_t8": ("prefill_llama8b", "decode_paged_t8"),
    # the same over an FP8 cache (tensor-core kernel converting e4m3 tiles in shared memory)
    "llama8b_paged_t8_fp8": ("prefill_llama8b", "decode_paged_t8_fp8"),
}
PREFILL_CACHE_SETS = {"llama8b_prefill_cache"}   # sets whose attend step is attn_prefill_cache
DEFAULT_SET = "llama8b_layer"

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


# ----------------------------------------------------------------- ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist


def reduce_over_ranks(local_sum: float, local_max: float, world: int, device=None):
    """(sum over ranks of local_sum, max over ranks of local_max)."""
    if world == 1:
        return local_sum, local_max
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_sum], dtype=torch.float64, device=device)
    m = torch.tensor([local_max], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    dist.all_reduce(m, op=dist.ReduceOp.MAX)
    return float(t.item()), float(m.item())


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, kept only inside [t0, t1]."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.rows = []
        self.window = (0.0, 0.0)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)

    def summary(self):
        if self.proc is None:
            return None
        t0, t1 = self.window
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.rows:
            if not (t0 - 0.05 <= ts <= t1 + 0.05):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm.append(float(parts[2]))
                smax.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(names, parts[6:10]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- workload
def decode_bytes(case, w) -> int:
    """Algorithmic bytes of one attn_decode call: valid K and V (2 bytes per element,
    1 for an FP8 cache, plus its scales), q, o (bf16), lse, lengths (+ page table)."""
    eb = 1 if w.fp8 else 2
    kvb = int(case.seqlens_k.sum()) * w.Hkv * w.d * eb * 2
    scales = 2 * w.Hkv * 4 if w.fp8 else 0
    qo = 2 * w.B * w.T * w.Hq * w.d * 2
    lse = w.B * w.Hq * w.T * 4
    lens = w.B * 4
    table = 0
    if case.paged:
        table = int(sum((int(L) + 15) // 16 for L in case.seqlens_k)) * 4
    return kvb + scales + qo + lse + lens + table


def decode_flops(case, w) -> int:
    """4 d FLOPs per visible (query row, key) pair; new token t of T sees keys
    j <= L - T + t (causal) or all L keys."""
    pairs = 0
    for L in case.seqlens_k:
        L = int(L)
        pairs += w.T * (L - w.T) + w.T * (w.T + 1) // 2 if w.causal else w.T * L
    return 4 * w.d * w.Hq * pairs


def prefill_flops(w) -> int:
    pairs = w.N * (w.N + 1) // 2 if w.causal else w.N * w.N
    return 4 * w.B * w.Hq * w.d * pairs


def append_and_attend(kv, wd, kc, vc, q, k_new, v_new, cache_lens, seqlens, table, scales, o, lse, msk, ws, stream,
                      ev=None, prefill_cache=False):
    """kv_append then attn_decode (their FP8 forms for an FP8 cache, or attn_prefill_cache);
    events 2 and 3 around the attend."""
    if scales is None:
        kv.kv_append(kc, vc, k_new, v_new, cache_lens, page_table=table, stream=stream)
    else:
        kv.kv_append_fp8(kc, vc, k_new, v_new, scales[0], scales[1], cache_lens, page_table=table, stream=stream)
    if ev is not None:
        ev[2].record(stream)
    if prefill_cache:
        kv.attn_prefill_cache(q, kc, vc, seqlens, o, lse, page_table=table, scale=wd.scale, causal=wd.causal,
                              stream=stream)
    elif scales is None:
        kv.attn_decode(q, kc, vc, seqlens, o, lse, page_table=table, max_seqlen_k=msk, scale=wd.scale,
                       causal=wd.causal, workspace=ws, stream=stream)
    else:
        kv.attn_decode_fp8(q, kc, vc, scales[0], scales[1], seqlens, o, lse, page_table=table, max_seqlen_k=msk,
                           scale=wd.scale, causal=wd.causal, workspace=ws, stream=stream)
    if ev is not None:
        ev[3].record(stream)


def decode_via_prefill(wd) -> bool:
    """attn_decode with at least 256 new tokens on a bf16 cache (automatic splitting)
    runs the prefill kernel's cached form."""
    return not wd.fp8 and wd.T >= 256


def decode_kernel_name(wd, prefill_cache=False) -> str:
    if prefill_cache or decode_via_prefill(wd):
        return "prefill_kernel<128, paged cache>" if wd.paged else "prefill_kernel<128, cache>"
    return f"{decode_kernel(wd)[0]} + decode_combine_kernel"


def decode_kernel(wd):
    """(name, source files) of the kernel attn_decode picks for this shape: bf16 up
    to 16 query rows per KV head on warp-level MMAs, more on tcgen05; FP8 up to
    8 rows on the transposed-product kernel, up to 32 on the split kernel, more on
    tcgen05 (e4m3 tiles converted to f16 in shared memory)."""
    R = wd.Hq // wd.Hkv * wd.T
    if decode_via_prefill(wd):
        return "prefill_kernel<128, paged cache>" if wd.paged else "prefill_kernel<128, cache>", ("prefill.cu",)
    if wd.fp8:
        if R <= 8:
            return "decode_fp8_st_kernel", ("decode_fp8.cu", "split.cuh", "decode.cu")
        if R <= 32:
            return "decode_split_kernel<fp8>", ("decode.cu", "split.cuh")
        return "decode_tc_kernel<fp8>", ("decode_tc.cu", "decode.cu")
    if R <= 16:
        return "decode_split_kernel", ("decode.cu", "split.cuh")
    return "decode_tc_kernel", ("decode_tc.cu", "decode.cu")


def run_ours(args, world, rank, local):
    import torch

    import kv_cache_decode_attn_b200 as kv
    import synth

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    pf_name, dec_name = WORKLOAD_SETS[args.workload]
    wp = synth.WORKLOADS[pf_name]
    wd = synth.WORKLOADS[dec_name]
    seed_off = 7919 * rank   # weak scaling: every rank gets its own batch
    q, k, v = synth.prefill_inputs(wp.B, wp.Hq, wp.Hkv, wp.N, wp.d, synth.SEEDS[pf_name] + seed_off, dev)
    o = torch.empty(wp.B, wp.N, wp.Hq, wp.d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(wp.B, wp.Hq, wp.N, dtype=torch.float32, device=dev)
    case = synth.decode_inputs(wd.B, wd.T, wd.Hq, wd.Hkv, wd.d, wd.len_lo, wd.len_hi,
                               synth.SEEDS[dec_name] + seed_off, device=dev, paged=wd.paged, fp8=wd.fp8)
    cache_lens = torch.as_tensor(case.cache_lens.astype(np.int32), device=dev)
    seqlens = torch.as_tensor(case.seqlens_k.astype(np.int32), device=dev)
    table = None if case.page_table is None else torch.as_tensor(case.page_table, device=dev)
    kc = case.k_pool if wd.paged else case.k_cache
    vc = case.v_pool if wd.paged else case.v_cache
    msk = int(case.seqlens_k.max())
    od = torch.empty(wd.B, wd.T, wd.Hq, wd.d, dtype=torch.bfloat16, device=dev)
    ld = torch.empty(wd.B, wd.Hq, wd.T, dtype=torch.float32, device=dev)
    ws = kv.decode_workspace(wd.B, wd.T, wd.Hq, wd.Hkv, wd.d, msk, 0, dev)
    stream = torch.cuda.current_stream(dev)
    scales = ((torch.as_tensor(case.k_scale, device=dev), torch.as_tensor(case.v_scale, device=dev))
              if wd.fp8 else None)
    prefill_cache = args.workload in PREFILL_CACHE_SETS

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        kv.attn_prefill(q, k, v, o, lse, scale=wp.scale, causal=wp.causal, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        # the same token position is appended every step, so the cache length stays fixed
        append_and_attend(kv, wd, kc, vc, case.q, case.k_new, case.v_new, cache_lens, seqlens, table, scales, od,
                          ld, msk, ws, stream, ev, prefill_cache)



    kv.attn_get_device_status(clear=True)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    t_start.record(stream)
    for i in range(args.steps):
        step(events[i])
    t_stop.record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    clocks.window = (wall0, wall1)
    time.sleep(0.25)
    clocks.stop()
    status = kv.attn_get_device_status(clear=True)
    if status != 0:
        raise RuntimeError(f"device status {status} during the benchmark")

    total_ms = t_start.elapsed_time(t_stop)
    pf_ms = sum(e[0].elapsed_time(e[1]) for e in events)
    ap_ms = sum(e[1].elapsed_time(e[2]) for e in events)
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in events)
    K = args.steps
    flops = prefill_flops(wp)
    dbytes = decode_bytes(case, wd)
    dflops = decode_flops(case, wd)

    # whole-job: units summed over ranks / slowest rank's time
    tot_flops, pf_max = reduce_over_ranks(flops * K, pf_ms, world, dev)
    tot_bytes, dec_max = reduce_over_ranks(dbytes * K, dec_ms, world, dev)
    tot_dflops, _ = reduce_over_ranks(dflops * K, dec_ms, world, dev)
    _, total_max = reduce_over_ranks(0.0, total_ms, world, dev)
    pf_tflops = tot_flops / (pf_max * 1e-3) / 1e12
    dec_gbs = tot_bytes / (dec_max * 1e-3) / 1e9
    dec_tflops = tot_dflops / (dec_max * 1e-3) / 1e12

    # -------- every configuration alone (the default run only), inside the clock record
    configs = None
    if args.workload == DEFAULT_SET and not args.no_configs:
        peaks0, src0 = load_peaks()
        clocks2 = ClockSampler(local)
        clocks2.start()
        time.sleep(0.3)
        if world > 1:
            dist.barrier()
        c0 = time.time()
        configs = run_configs(kv, torch, dev, stream, args, world, peaks0, src0)
        c1 = time.time()
        clocks2.window = (c0, c1)
        time.sleep(0.25)
        clocks2.stop()
        configs["clocks"] = clocks2.summary()
        status = kv.attn_get_device_status(clear=True)
        if status != 0:
            raise RuntimeError(f"device status {status} during the configuration runs")

    # -------- end to end through the public API with host buffers (pinned)
    e2e = None if args.no_e2e else run_e2e(kv, torch, dev, stream, wp, wd, q, k, v, case, table, msk, ws, args,
                                           world, scales, prefill_cache)

    peaks, peak_src = load_peaks()
    pf_kernel_tflops = flops / (pf_ms / K * 1e-3) / 1e12          # per launch, this rank
    dec_kernel_gbs = dbytes / (dec_ms / K * 1e-3) / 1e9
    traffic = load_traffic(args.workload, wd, wp)
    # the kernels of this line are timed inside a long loop of steps: against the sustained
    # tensor peak (the burst figure is for a kernel timed alone, as in the configuration runs)
    roof_pf = {"bound": "tensor", "achieved": round(pf_kernel_tflops, 1), "peak": peaks["bf16_tflops_sustained"],
               "unit": "TFLOP/s", "frac": round(pf_kernel_tflops / peaks["bf16_tflops_sustained"], 4),
               "frac_of_burst": round(pf_kernel_tflops / peaks["bf16_tflops"], 4),
               "peak_source": f"{peak_src} (bf16 sustained)", "traffic": traffic.get("prefill"),
               "kernel": f"prefill_kernel<{wp.d}>", "flops_per_launch": flops,
               "launch_ms": round(pf_ms / K, 4)}
    # the decode call is HBM-bound unless its flops per byte pass the ridge (many new tokens: chunked prefill)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    dec_kernel_tflops = dflops / (dec_ms / K * 1e-3) / 1e12
    if dflops / dbytes > ridge:
        roof_dec = {"bound": "tensor", "achieved": round(dec_kernel_tflops, 1), "peak": peaks["bf16_tflops_sustained"],
                    "unit": "TFLOP/s", "frac": round(dec_kernel_tflops / peaks["bf16_tflops_sustained"], 4),
                    "frac_of_burst": round(dec_kernel_tflops / peaks["bf16_tflops"], 4),
                    "peak_source": f"{peak_src} (bf16 sustained)", "traffic": traffic.get("decode"),
                    "kernel": decode_kernel_name(wd, prefill_cache),
                    "flops_per_launch": dflops, "bytes_per_launch": dbytes, "launch_ms": round(dec_ms / K, 4)}
    else:
        roof_dec = {"bound": "hbm", "achieved": round(dec_kernel_gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(dec_kernel_gbs / peaks["hbm_gbs"], 4), "peak_source": f"{peak_src} (copy)",
                    "traffic": traffic.get("decode"),
                    "kernel": decode_kernel_name(wd, prefill_cache), "bytes_per_launch": dbytes,
                    "launch_ms": round(dec_ms / K, 4)}

    out = None
    if rank == 0:
        cpu = cpu_baseline(args, wp, wd, q, k, v, case) if (world == 1 and not args.no_cpu_baseline) else None
        out = {
            "metric": METRIC, "value": round(pf_tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(total_max / K, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {
                "workload": args.workload,
                "prefill": {"name": pf_name, "B": wp.B, "Hq": wp.Hq, "Hkv": wp.Hkv, "N": wp.N, "d": wp.d,
                            "causal": wp.causal, "o_dtype": "bf16"},
                "decode": {"name": dec_name, "B": wd.B, "T": wd.T, "Hq": wd.Hq, "Hkv": wd.Hkv, "d": wd.d,
                           "cache_len": [wd.len_lo, wd.len_hi], "paged": wd.paged, "append_before_attend": True,
                           "kv_dtype": "e4m3 + fp32 scale per KV head" if wd.fp8 else "bf16",
                           "kv_bytes_per_step": int(case.seqlens_k.sum()) * wd.Hkv * wd.d * (2 if wd.fp8 else 4)},
                "l2": "no flush: every step reads inputs larger than the 126 MB L2",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "seed": synth.SEEDS[pf_name],
            },
            "decode": {"value": round(dec_gbs, 1), "unit": "GB/s", "tflops": round(dec_tflops, 2),
                       "roofline": roof_dec, "append_ms_per_step": round(ap_ms / K, 4)},
            "roofline": roof_pf,
            "configs": configs,
            "cpu_baseline": cpu,
            "e2e": e2e,
            # per step: prefill, append, then decode split + combine (or one attn_prefill_cache launch);
            # the configuration runs are outside the timed region
            "gpu_launches": (3 if prefill_cache or decode_via_prefill(wd) else 4) * K,
            "clocks": clocks.summary(),
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


# Every configuration the method is specified on, timed in the default run after the step
# (name, workload, note).  Configuration 1 is the oracle-sized parity case.
CONFIG_RUNS = [
    ("1_prefill_small", "prefill_small", "parity-size case (the oracle's full-output case); L2 flushed before each launch"),
    ("2_prefill_gpt2", "prefill_gpt2", "GPT-2-small MHA; inputs fit in L2, so L2 is flushed before each launch"),
    ("3_prefill_llama8b_causal", "prefill_llama8b", "inputs larger than L2"),
    ("3_prefill_llama8b_noncausal_8192", "prefill_llama8b_nc", "inputs larger than L2"),
    ("4_decode_contig_t1", "decode_contig", "kv_append then attn_decode; cache larger than L2"),
    ("5_decode_paged_t1", "decode_paged", "kv_append then attn_decode; cache larger than L2"),
    ("5_decode_paged_t4", "decode_paged_t4", "speculative-verify shape, offset mask; cache larger than L2"),
]
L2_FLUSH_BYTES = 256 << 20   # twice the 126 MB L2


def run_configs(kv, torch, dev, stream, args, world, peaks, peak_src):
    """Each configuration alone: warm-up launches, then n timed launches, CUDA events
    around the kernel call only (an L2 flush, where the inputs fit in L2, runs between
    the events of consecutive launches).  Whole-job: units summed over ranks over the
    slowest rank's summed time."""
    import synth
    n = max(5, min(args.steps, 50))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    out = {}
    for key, name, note in CONFIG_RUNS:
        w = synth.WORKLOADS[name]
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        small = False
        if isinstance(w, synth.Prefill):
            q, k, v = synth.prefill_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, synth.SEEDS[name], dev)
            o = torch.empty(w.B, w.N, w.Hq, w.d, dtype=torch.bfloat16, device=dev)
            lse = torch.empty(w.B, w.Hq, w.N, dtype=torch.float32, device=dev)
            small = 4 * q.numel() * 2 < 126e6

            def call():
                kv.attn_prefill(q, k, v, o, lse, scale=w.scale, causal=w.causal, stream=stream)
            units, unit_name = prefill_flops(w), "flops"
            kernel = f"prefill_kernel<{w.d}>"
        else:
            case = synth.decode_inputs(w.B, w.T, w.Hq, w.Hkv, w.d, w.len_lo, w.len_hi, synth.SEEDS[name], device=dev,
                                       paged=w.paged, fp8=w.fp8)
            cl = torch.as_tensor(case.cache_lens.astype(np.int32), device=dev)
            sl = torch.as_tensor(case.seqlens_k.astype(np.int32), device=dev)
            tab = None if case.page_table is None else torch.as_tensor(case.page_table, device=dev)
            kc = case.k_pool if w.paged else case.k_cache
            vc = case.v_pool if w.paged else case.v_cache
            msk = int(case.seqlens_k.max())
            od = torch.empty(w.B, w.T, w.Hq, w.d, dtype=torch.bfloat16, device=dev)
            ld = torch.empty(w.B, w.Hq, w.T, dtype=torch.float32, device=dev)
            ws = kv.decode_workspace(w.B, w.T, w.Hq, w.Hkv, w.d, msk, 0, dev)
            kv.kv_append(kc, vc, case.k_new, case.v_new, cl, page_table=tab, stream=stream)

            def call():
                kv.attn_decode(case.q, kc, vc, sl, od, ld, page_table=tab, max_seqlen_k=msk, scale=w.scale,
                               causal=w.causal, workspace=ws, stream=stream)
            units, unit_name = decode_bytes(case, w), "bytes"
            kernel = decode_kernel_name(w)
        for _ in range(3):
            call()
        for i in range(n):
            if small:
                flush.fill_(float(i))
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        ms = sum(a.elapsed_time(b) for a, b in ev)
        tot, ms_max = reduce_over_ranks(units * n, ms, world, dev)
        per_launch = units / (ms / n * 1e-3)
        if unit_name == "flops":
            value, unit = tot / (ms_max * 1e-3) / 1e12, "TFLOP/s"
            roof = {"bound": "tensor", "achieved": round(per_launch / 1e12, 1), "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": round(per_launch / 1e12 / peaks["bf16_tflops"], 4),
                    "frac_of_sustained": round(per_launch / 1e12 / peaks["bf16_tflops_sustained"], 4),
                    "peak_source": f"{peak_src} (bf16 burst)", "flops_per_launch": units}
        else:
            value, unit = tot / (ms_max * 1e-3) / 1e9, "GB/s"
            roof = {"bound": "hbm", "achieved": round(per_launch / 1e9, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(per_launch / 1e9 / peaks["hbm_gbs"], 4), "peak_source": f"{peak_src} (copy)",
                    "bytes_per_launch": units}
        roof["kernel"] = kernel
        roof["launch_ms"] = round(ms / n, 4)
        desc = {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d}
        if isinstance(w, synth.Prefill):
            desc.update(N=w.N, causal=w.causal, o_dtype="bf16")
        else:
            desc.update(T=w.T, cache_len=[w.len_lo, w.len_hi], paged=w.paged, o_dtype="bf16")
        out[key] = {"workload": name, "shape": desc, "value": round(value, 2), "unit": unit, "launches": n,
                    "note": note, "roofline": roof}
        del call
        torch.cuda.synchronize(dev)
    del flush
    torch.cuda.empty_cache()
    return out


def run_e2e(kv, torch, dev, stream, wp, wd, q, k, v, case, table, msk, ws, args, world, scales=None,
            prefill_cache=False):
    """Same step through the public API, inputs copied from pinned host memory
    and results read back every step (the KV cache stays resident: it is state)."""
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty(wp.B, wp.Hq, wp.N, dtype=torch.float32).pin_memory()
    hdq, hkn, hvn = (t.cpu().pin_memory() for t in (case.q, case.k_new, case.v_new))
    hcl = torch.as_tensor(case.cache_lens.astype(np.int32)).pin_memory()
    hsl = torch.as_tensor(case.seqlens_k.astype(np.int32)).pin_memory()
    hdo = torch.empty(case.q.shape, dtype=torch.bfloat16).pin_memory()
    hdl = torch.empty(wd.B, wd.Hq, wd.T, dtype=torch.float32).pin_memory()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    do = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    dl = torch.empty(wp.B, wp.Hq, wp.N, dtype=torch.float32, device=dev)
    ddq, dkn, dvn = torch.empty_like(case.q), torch.empty_like(case.k_new), torch.empty_like(case.v_new)
    dcl = torch.empty(wd.B, dtype=torch.int32, device=dev)
    dsl = torch.empty(wd.B, dtype=torch.int32, device=dev)
    ddo = torch.empty(case.q.shape, dtype=torch.bfloat16, device=dev)
    ddl = torch.empty(wd.B, wd.Hq, wd.T, dtype=torch.float32, device=dev)
    kc = case.k_pool if wd.paged else case.k_cache
    vc = case.v_pool if wd.paged else case.v_cache

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        kv.attn_prefill(dq, dk, dv, do, dl, scale=wp.scale, causal=wp.causal, stream=stream)
        ho.copy_(do, non_blocking=True)
        hl.copy_(dl, non_blocking=True)
        if ev is not None:
            ev[1].record(stream)
        ddq.copy_(hdq, non_blocking=True)
        dkn.copy_(hkn, non_blocking=True)
        dvn.copy_(hvn, non_blocking=True)
        dcl.copy_(hcl, non_blocking=True)
        dsl.copy_(hsl, non_blocking=True)
        append_and_attend(kv, wd, kc, vc, ddq, dkn, dvn, dcl, dsl, table, scales, ddo, ddl, msk, ws, stream,
                          prefill_cache=prefill_cache)
        hdo.copy_(ddo, non_blocking=True)
        hdl.copy_(ddl, non_blocking=True)
        if ev is not None:
            ev[2].record(stream)

    n = max(3, min(args.steps, 20))
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    for i in range(n):
        step(evs[i])
    torch.cuda.synchronize(dev)
    pf_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    flops, pf_max = reduce_over_ranks(prefill_flops(wp) * n, pf_ms, world, dev)
    dbytes, dec_max = reduce_over_ranks(decode_bytes(case, wd) * n, dec_ms, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdq, hkn, hvn, hcl, hsl))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hl, hdo, hdl))
    return {"value": round(flops / (pf_max * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": n,
            "decode": {"value": round(dbytes / (dec_max * 1e-3) / 1e9, 1), "unit": "GB/s"}}


def source_hash(files) -> str:
    """First 16 hex digits of the sha256 over the named csrc files, in order."""
    import hashlib
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "kv_cache_decode_attn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload, wd, wp):
    """Per-launch DRAM bytes (ncu dram__bytes_read.sum + dram__bytes_write.sum,
    summed over the leg's kernels) from the committed profile summary, for this
    workload only, and kept only while the kernel sources it was measured on are
    unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entries = json.load(f)["entries"]
    except (OSError, ValueError, KeyError):
        return {}
    prefill_cache = workload in PREFILL_CACHE_SETS
    want = {"prefill": (f"prefill_kernel<{wp.d}>", ("prefill.cu",)),
            "decode": (decode_kernel_name(wd, True), ("prefill.cu",)) if prefill_cache else decode_kernel(wd)}
    out = {}
    for e in entries:
        leg = e.get("leg")
        if e.get("workload") != workload or leg not in want:
            continue
        kernel, files = want[leg]
        try:
            ok = e.get("kernel") == kernel and tuple(e["sources"]) == tuple(files) \
                and e.get("sha256_16") == source_hash(files)
        except (OSError, KeyError):
            ok = False
        if ok:
            out[leg] = e["bytes"]
    return out


# ------------------------------------------------------------ CPU oracle legs
def _threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            return int(max(i.get("num_threads", 1) for i in info))
    except Exception:
        pass
    return os.cpu_count() or 1


ORACLE_ROWS = 256   # query rows per oracle prefill sample


def oracle_prefill_sample(wp, q, k, v, budget_s, rng):
    """Blocks of 256 query rows of one (b, h) head through the oracle until the
    budget is spent.  q, k, v are host bf16 tensors; each block's slices are
    converted to float64 before its clock starts."""
    import oracle
    flops, t, blocks = 0, 0.0, 0
    G = wp.Hq // wp.Hkv
    while True:
        b, h = int(rng.integers(wp.B)), int(rng.integers(wp.Hq))
        i0 = int(rng.integers(0, max(1, wp.N - ORACLE_ROWS + 1)))
        i1 = min(wp.N, i0 + ORACLE_ROWS)
        nk = i1 if wp.causal else wp.N      # rows i0..i1-1 are the last rows of the first i1 keys
        g = h // G
        qs = q[b, i0:i1, h].double().numpy()
        ks = k[b, :nk, g].double().numpy()
        vs = v[b, :nk, g].double().numpy()
        t0 = time.perf_counter()
        oracle.attend_head(qs, ks, vs, wp.scale, wp.causal)
        t += time.perf_counter() - t0
        flops += 4 * wp.d * oracle.visible_pairs(i1 - i0, nk, wp.causal)
        blocks += 1
        if t >= budget_s:
            return flops, t, blocks


def oracle_decode_sample(wd, case_h, budget_s, rng):
    """One KV head group of one sequence (its Hq/Hkv query heads, all T tokens)
    through the oracle per sample, until the budget is spent."""
    import oracle
    nbytes, t, units = 0, 0.0, 0
    G = wd.Hq // wd.Hkv
    while True:
        b = int(rng.integers(case_h["q"].shape[0]))
        g = int(rng.integers(wd.Hkv))
        L = int(case_h["seqlens_k"][b])
        qs = case_h["q"][b:b + 1, :, g * G:(g + 1) * G]
        kc, vc = case_h["k"][b:b + 1, :L, g:g + 1], case_h["v"][b:b + 1, :L, g:g + 1]
        t0 = time.perf_counter()
        oracle.decode(qs, kc, vc, [L], wd.scale, wd.causal)
        t += time.perf_counter() - t0
        nbytes += L * wd.d * (2 if wd.fp8 else 4) + 2 * wd.T * G * wd.d * 2
        units += 1
        if t >= budget_s:
            return nbytes, t, units


def host_decode_case(case, wd, max_seqs=4):
    """fp64 host copies of a few sequences of the decode workload (cache as it is
    after the append: stored rows followed by the new tokens; an FP8 cache is
    dequantised, and its new tokens quantised, by the oracle)."""
    import torch

    def values(rows, which):
        if not wd.fp8:
            return rows.float().cpu().numpy()
        import oracle
        s = case.k_scale if which == 0 else case.v_scale
        return oracle.fp8.dequantize(rows.cpu().numpy(), s)

    def new_values(rows, which):
        if not wd.fp8:
            return rows.float().cpu().numpy()
        import oracle
        s = case.k_scale if which == 0 else case.v_scale
        return oracle.fp8.dequantize(oracle.fp8.quantize_rows(rows.float().cpu().numpy(), s), s)

    idx = list(range(min(max_seqs, wd.B)))
    Lmax = int(max(case.seqlens_k[i] for i in idx))
    k = np.zeros((len(idx), Lmax, wd.Hkv, wd.d))
    v = np.zeros_like(k)
    for j, b in enumerate(idx):
        L0 = int(case.cache_lens[b])
        if case.paged:
            nb = (L0 + wd.T + 15) // 16
            ids = torch.as_tensor(case.page_table[b, :nb].astype(np.int64), device=case.k_pool.device)
            kb = case.k_pool.index_select(0, ids).reshape(nb * 16, wd.Hkv, wd.d)[:L0]
            vb = case.v_pool.index_select(0, ids).reshape(nb * 16, wd.Hkv, wd.d)[:L0]
        else:
            kb, vb = case.k_cache[b, :L0], case.v_cache[b, :L0]
        k[j, :L0] = values(kb, 0)
        v[j, :L0] = values(vb, 1)
        k[j, L0:L0 + wd.T] = new_values(case.k_new[b], 0)
        v[j, L0:L0 + wd.T] = new_values(case.v_new[b], 1)
    return {"q": case.q[idx].float().cpu().numpy().astype(np.float64), "k": k, "v": v,
            "seqlens_k": case.seqlens_k[idx]}


def cpu_baseline(args, wp, wd, q, k, v, case):
    rng = np.random.default_rng(0)
    qh, kh, vh = (t.cpu() for t in (q, k, v))
    fl, tp, blocks = oracle_prefill_sample(wp, qh, kh, vh, args.cpu_budget, rng)
    ch = host_decode_case(case, wd)
    nb, td, units = oracle_decode_sample(wd, ch, args.cpu_budget / 2, rng)
    return {"value": round(fl / tp / 1e12, 5), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{blocks} blocks of {ORACLE_ROWS} query rows of single (b, h) heads of the prefill "
                      f"workload ({tp:.1f} s); decode: {units} (sequence, KV head) groups with all their "
                      f"query heads ({td:.1f} s)",
            "decode": {"value": round(nb / td / 1e9, 4), "unit": "GB/s"}}


def run_reference(args):
    """The oracle, as it stands, on the host cores: bounded samples of the same workload per step."""
    import synth
    pf_name, dec_name = WORKLOAD_SETS[args.workload]
    wp, wd = synth.WORKLOADS[pf_name], synth.WORKLOADS[dec_name]
    q, k, v = synth.prefill_inputs(wp.B, wp.Hq, wp.Hkv, wp.N, wp.d, synth.SEEDS[pf_name], "cpu")
    n_seq = 2   # sequences of the decode workload held on the host for sampling
    case = synth.decode_inputs(n_seq, wd.T, wd.Hq, wd.Hkv, wd.d, wd.len_lo, wd.len_hi, synth.SEEDS[dec_name],
                               device="cpu", paged=wd.paged, fp8=wd.fp8)
    ch = host_decode_case(case, _shrink(wd, n_seq), max_seqs=n_seq)
    rng = np.random.default_rng(1)
    # each step is a bounded sample, sized so the whole run stays within a few minutes
    per_step = min(args.ref_step_budget, 150.0 / (args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_prefill_sample(wp, q, k, v, per_step * 0.7, rng)
    fl_tot = t_pf = nb_tot = t_dec = 0.0
    blocks = units = 0
    for _ in range(args.steps):
        fl, tp, nbk = oracle_prefill_sample(wp, q, k, v, per_step * 0.7, rng)
        nb, td, nu = oracle_decode_sample(wd, ch, per_step * 0.3, rng)
        fl_tot += fl
        t_pf += tp
        blocks += nbk
        nb_tot += nb
        t_dec += td
        units += nu
    value = fl_tot / t_pf / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round((t_pf + t_dec) / args.steps * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "prefill": pf_name, "decode": dec_name,
                   "sample": f"each step: blocks of {ORACLE_ROWS} prefill query rows for ~70% and (sequence, KV "
                             f"head) decode groups for ~30% of a {per_step:.3f} s budget"},
        "decode": {"value": round(nb_tot / t_dec / 1e9, 5), "unit": "GB/s"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
                         "sample": f"{blocks} prefill row blocks, {units} decode groups over {args.steps} steps"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def _shrink(wd, B):
    import dataclasses
    return dataclasses.replace(wd, B=B)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_SETS), default=DEFAULT_SET)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration runs")
    ap.add_argument("--ref-step-budget", type=float, default=1.5, help="seconds of oracle work per reference step")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    if world != args.gpus and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    out = run_ours(args, world, rank, local)
    if out is not None:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
