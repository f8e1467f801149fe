#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole path on synthetic, seeded inputs resident
in HBM: the fused prefill forward (fa_fwd) on the causal MHA workload
B=4, H=16, S=2048, d=128 with Q ~ N(0,1)*8, followed by single-query split-KV
decode (fa_decode_splitkv + fa_combine) on B=64, Hq=32, Hkv=8, d=128 with KV
lengths uniform in [4096, 16384].  L2 is flushed (a 256 MB write) before
every step, outside the event-timed regions.

`value` is the prefill's TFLOP/s (FLOPs = 4*B*Hq*Sq*Skv*d, halved for the
causal mask) over all ranks; the decode's HBM GB/s is reported beside it.
With N > 1 (torchrun) every rank runs the same per-GPU work on its own seed
(weak scaling, no data-path collective); times are the max over ranks.

`--impl reference` times the fp64 CPU oracle instead, on a bounded sample of
the prefill workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

PREFILL_WORKLOAD = "causal_mha_s2048_d128_qx8"
DECODE_WORKLOAD = "decode_b64_splitkv_d128"
METRIC = "attn fwd TFLOPS bf16 & % tensor peak; decode HBM GB/s & % of 8 TB/s"
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PREFILL_SOURCES = ["io_aware_exact_flashattention_b200/csrc/prefill_sm100.cuh",
                   "io_aware_exact_flashattention_b200/csrc/sm100.cuh"]
DECODE_SOURCES = ["io_aware_exact_flashattention_b200/csrc/decode_sm100.cuh",
                  "io_aware_exact_flashattention_b200/csrc/sm100.cuh"]
BACKWARD_SOURCES = ["io_aware_exact_flashattention_b200/csrc/backward_sm100.cuh",
                    "io_aware_exact_flashattention_b200/csrc/sm100.cuh"]


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=PREFILL_WORKLOAD,
                    help="prefill workload name (io_aware_exact_flashattention_b200.inputs)")
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                    help="restrict the step (for profiling captures)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="override the decode workload's batch (smaller profiling captures)")
    ap.add_argument("--decode-splits", type=int, default=None,
                    help="override the decode split count (default: fa_decode_default_splits)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-paged", action="store_true",
                    help="skip the paged-cache decode measurement")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward measurement on the prefill workload")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the E4M3-input forward on the prefill workload")
    ap.add_argument("--no-bpt", action="store_true",
                    help="skip the blockwise feed-forward network after the prefill attention")
    ap.add_argument("--bpt-chunk", type=int, default=16,
                    help="query tiles per chunk of the blockwise feed-forward network")
    ap.add_argument("--page-size", type=int, default=16,
                    help="page size of the paged-cache decode measurement")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# small helpers
# ---------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def sources_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(summary_name, paths):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the kernel source as it is now (else None)."""
    path = os.path.join(ROOT, "profiles", summary_name)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != sources_sha(paths):
        return None
    return int(m_tr.group(1))


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index, period_s=0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self._nv = None
            self.error = str(e)

    def _sample(self):
        nv = self._nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
        mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for bit, name in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        busy = [s for s in self.samples if s > 0]
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return world, rank, local  # rank 0 alone runs the oracle; no process group
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(values, world):
    """Element-wise max of per-rank timings (the slowest rank sets the time)."""
    if world == 1:
        return list(values)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(values, dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def rank_seed(seed, rank):
    """Each rank draws its own inputs (independent replicas, weak scaling)."""
    return seed + 1000 * rank


def aggregate_rate(world, work_per_step, steps, max_ms):
    """Whole-job throughput: the work all ranks did over the slowest rank's time."""
    return world * work_per_step * steps / (max_ms * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# the CPU oracle as a baseline (bounded sample of the prefill workload)
# ---------------------------------------------------------------------------

def oracle_sample_seconds(q, k, v, c, heads):
    """Time the fp64 oracle on all query rows of `heads` (b, h) pairs."""
    import oracle
    lib = oracle.load()
    grp = c.Hq // c.Hkv
    t0 = time.perf_counter()
    for (b, h) in heads:
        oracle.attn_fwd(q[b:b + 1, h:h + 1], k[b:b + 1, h // grp:h // grp + 1],
                        v[b:b + 1, h // grp:h // grp + 1], c.causal, c.scale, lib=lib)
    return time.perf_counter() - t0


def cpu_baseline(c, target_s=15.0):
    """Oracle on whole heads of the workload (CPU copies of the same seeded
    inputs), sized to about `target_s` seconds.  Returns the JSON object."""
    import oracle
    from io_aware_exact_flashattention_b200.inputs import prefill_inputs_for
    q, k, v = prefill_inputs_for(c, device="cuda")
    q, k, v = (t.cpu().double() for t in (q, k, v))
    all_heads = [(b, h) for b in range(c.B) for h in range(c.Hq)]
    t1 = oracle_sample_seconds(q, k, v, c, all_heads[:1])
    n = max(1, min(len(all_heads), int(target_s / max(t1, 1e-3))))
    heads = all_heads[:n]
    t = oracle_sample_seconds(q, k, v, c, heads)
    flops = c.flops() * n / len(all_heads)
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "fp64 oracle on all %d query rows of %d of the %d (b, head) pairs of %s "
                      "(%.3g GFLOP in %.2f s)" % (c.Sq, n, len(all_heads), c.name, flops / 1e9, t)}


def run_reference(args, world, rank):
    """The oracle as the reference arm: each step is one (b, head) of the
    prefill workload, all query rows, fp64 on the host cores."""
    if rank != 0:
        return
    import oracle
    from io_aware_exact_flashattention_b200.inputs import CONFIGS, prefill_inputs
    c = CONFIGS[args.workload]
    q, k, v = prefill_inputs(c.B, c.Hq, c.Hkv, c.Sq, c.Skv, c.d, c.seed, c.q_mult, device="cpu")
    q, k, v = (t.double() for t in (q, k, v))
    heads = [(b, h) for b in range(c.B) for h in range(c.Hq)]
    for i in range(args.warmup):
        oracle_sample_seconds(q, k, v, c, [heads[i % len(heads)]])
    t = 0.0
    for i in range(args.steps):
        t += oracle_sample_seconds(q, k, v, c, [heads[(args.warmup + i) % len(heads)]])
    flops = c.flops() / len(heads) * args.steps
    value = flops / t / 1e12
    sample = ("fp64 oracle, one (b, head) of %s per step (all %d query rows)" % (c.name, c.Sq))
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": c.name, "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "Sq": c.Sq,
                   "Skv": c.Skv, "d": c.d, "causal": c.causal, "q_mult": c.q_mult,
                   "sample_per_step": "1 of %d heads" % len(heads)},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our CUDA path
# ---------------------------------------------------------------------------

def decode_bytes(c, seqlens):
    """Algorithmic HBM bytes of one decode call: every visible K and V row
    once, q, O and LSE.  Split partials are overhead and not counted."""
    total_len = int(seqlens.sum().item())
    kv = 2 * total_len * c.Hkv * c.d * 2
    return kv + c.B * c.Hq * c.d * 2 + c.B * c.Hq * c.d * 2 + c.B * c.Hq * 4


def run_ours(args, world, rank, local):
    from io_aware_exact_flashattention_b200 import fa
    from io_aware_exact_flashattention_b200.inputs import CONFIGS, decode_inputs, prefill_inputs
    fa.lib()  # fail loudly when the CUDA library is missing
    dev = torch.device("cuda", local)
    peaks, peaks_kind = load_peaks()
    do_pre = args.only in ("all", "prefill")
    do_dec = args.only in ("all", "decode")

    c = CONFIGS[args.workload]
    cd = CONFIGS[DECODE_WORKLOAD]
    q, k, v = prefill_inputs(c.B, c.Hq, c.Hkv, c.Sq, c.Skv, c.d, rank_seed(c.seed, rank),
                             c.q_mult, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((c.B, c.Hq, c.Sq), device=dev, dtype=torch.float32)
    if do_dec:
        if args.decode_batch is not None:
            import dataclasses
            cd = dataclasses.replace(cd, B=args.decode_batch,
                                     name="%s_b%d" % (cd.name, args.decode_batch))
        qd, kc, vc, sl = decode_inputs(cd.B, cd.Hq, cd.Hkv, cd.Lmin, cd.Lmax, cd.d,
                                       rank_seed(cd.seed, rank), device=dev)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        n_split = args.decode_splits or fa.decode_default_splits(cd.B, cd.Hkv, cd.Lmax, sms)
        op = torch.empty((cd.B, cd.Hq, n_split, cd.d), device=dev, dtype=torch.float32)
        lp = torch.empty((cd.B, cd.Hq, n_split), device=dev, dtype=torch.float32)
        od = torch.empty((cd.B, cd.Hq, cd.d), device=dev, dtype=torch.bfloat16)
        lsed = torch.empty((cd.B, cd.Hq), device=dev, dtype=torch.float32)
        dec_bytes = decode_bytes(cd, sl)
    flush = torch.empty(64 * 1024 * 1024, device=dev, dtype=torch.float32)  # 256 MB > L2
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        flush.fill_(1.0)
        if evs is not None:
            evs[0].record(stream)
        if do_pre:
            fa.fa_fwd(q, k, v, o, lse, c.causal, c.scale, stream=stream)
        if evs is not None:
            evs[1].record(stream)
        if do_dec:
            fa.fa_decode_splitkv(qd, kc, vc, sl, op, lp, cd.scale, stream=stream)
            fa.fa_combine(op, lp, od, lsed, stream=stream)
        if evs is not None:
            evs[2].record(stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        torch.cuda.nvtx.range_push("bench_timed")
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize(dev)
    barrier(world)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    pre_ms, dec_ms, tot_ms = max_over_ranks([pre_ms, dec_ms, pre_ms + dec_ms], world)
    K = args.steps
    flops = c.flops()
    prefill_tflops = aggregate_rate(world, flops, K, pre_ms) / 1e12 if do_pre else None
    dec_gbs = aggregate_rate(world, dec_bytes, K, dec_ms) / 1e9 if do_dec else None

    # e2e: the user-level call with pinned host buffers, copies inside the region
    e2e = None
    if not args.no_e2e and do_pre:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        for _ in range(max(args.warmup, 1)):
            fa.flash_attention(qh, kh, vh, causal=c.causal, scale=c.scale, out=(oh, lh))
        barrier(world)
        torch.cuda.synchronize(dev)
        e2e_evs = []
        for _ in range(K):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fa.flash_attention(qh, kh, vh, causal=c.causal, scale=c.scale, out=(oh, lh))
            b.record(stream)
            e2e_evs.append((a, b))
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in e2e_evs)], world)[0]
        e2e = {"value": aggregate_rate(world, flops, K, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int((q.numel() + k.numel() + v.numel()) * 2),
               "d2h_bytes_per_step": int(o.numel() * 2 + lse.numel() * 4),
               "api": "io_aware_exact_flashattention_b200.flash_attention (host tensors)"}

    # Backward on the prefill workload (dq, dk, dv from the forward's O and
    # LSE), measured on its own after the step.
    backward = None
    if do_pre and not args.no_backward:
        from io_aware_exact_flashattention_b200.inputs import grad_output
        d_o = grad_output(q.shape, rank_seed(c.seed, rank), device=dev)
        fa.fa_fwd(q, k, v, o, lse, c.causal, c.scale, stream=stream)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(fa.bwd_workspace_bytes(c.B, c.Hq, c.Sq, c.d), dtype=torch.uint8,
                         device=dev)
        for _ in range(max(args.warmup, 1)):
            fa.fa_bwd(q, k, v, o, lse, d_o, dq, dk, dv, ws, c.causal, c.scale, stream=stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        bevs = []
        for _ in range(K):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fa.fa_bwd(q, k, v, o, lse, d_o, dq, dk, dv, ws, c.causal, c.scale, stream=stream)
            b.record(stream)
            bevs.append((a, b))
        torch.cuda.synchronize(dev)
        barrier(world)
        bw_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in bevs)], world)[0]
        bw_flops = 2.5 * flops
        bw_tf = bw_flops / (bw_ms * 1e-3 / K) / 1e12
        backward = {"value": aggregate_rate(world, bw_flops, K, bw_ms) / 1e12, "unit": "TFLOP/s",
                    "ms_per_call": bw_ms / K, "frac_of_measured_burst": bw_tf / float(peaks["bf16_tflops"]),
                    "frac_of_nominal_2250": bw_tf / NOMINAL_BF16_TFLOPS,
                    "algorithmic": "%.4g FLOP per call (2.5 x the forward's: five products)" % bw_flops,
                    "kernels": "fa_bwd_dsum_kernel (also zeroes the dq workspace) + fa_bwd_kernel<128> + fa_bwd_dq_kernel",
                    "traffic_main_kernel": profiled_traffic("backward_causal_mha_s2048_d128.md",
                                                            BACKWARD_SOURCES),
                    "gpu_launches": 3 * K,
                    "note": "dq, dk, dv from the forward's O and LSE; measured outside the step"}
        del dq, dk, dv, ws, d_o

    # The prefill workload with E4M3 inputs (per-(batch, kv-head) factors),
    # measured on its own after the step.
    prefill_fp8 = None
    if do_pre and not args.no_fp8 and c.d == 128:
        from io_aware_exact_flashattention_b200.inputs import fp8_prefill_inputs
        q8, k8, v8, dq8, dk8, dv8 = fp8_prefill_inputs(c.B, c.Hq, c.Hkv, c.Sq, c.Skv, c.d,
                                                      rank_seed(c.seed, rank), c.q_mult,
                                                      device=dev)
        for _ in range(max(args.warmup, 1)):
            fa.fa_fwd_fp8(q8, k8, v8, dq8, dk8, dv8, o, lse, c.causal, c.scale, stream=stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        fevs = []
        for _ in range(K):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fa.fa_fwd_fp8(q8, k8, v8, dq8, dk8, dv8, o, lse, c.causal, c.scale, stream=stream)
            b.record(stream)
            fevs.append((a, b))
        torch.cuda.synchronize(dev)
        barrier(world)
        f8_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in fevs)], world)[0]
        f8_tf = flops / (f8_ms * 1e-3 / K) / 1e12
        f8_peak = 2.0 * float(peaks["bf16_tflops"])  # E4M3 dense rate = 2 x bf16 (4.5 / 2.25)
        prefill_fp8 = {
            "value": aggregate_rate(world, flops, K, f8_ms) / 1e12, "unit": "TFLOP/s",
            "ms_per_call": f8_ms / K, "dtype": "e4m3 (fp32 accumulate)",
            "roofline": {"bound": "tensor", "achieved": f8_tf, "peak": f8_peak,
                         "unit": "TFLOP/s", "frac": f8_tf / f8_peak,
                         "peak_source": "2 x measured bf16 burst (nominal e4m3:bf16 ratio 4.5:2.25)",
                         "traffic": profiled_traffic("prefill_fp8_causal_mha_s2048_d128.md",
                                                     PREFILL_SOURCES)},
            "frac_of_nominal_4500": f8_tf / (2.0 * NOMINAL_BF16_TFLOPS),
            "kernels": "fa_prefill_kernel<128, true>", "gpu_launches": K,
            "note": "same shape and FLOP count as the bf16 prefill; measured outside the step"}
        del q8, k8, v8, dq8, dk8, dv8

    # Blockwise feed-forward network (F = 4 D) on the forward's attention
    # output, chunk by chunk; random stand-in weights.  Measured on its own.
    bpt = None
    if do_pre and not args.no_bpt and (c.Hq * c.d) % 256 == 0:
        from io_aware_exact_flashattention_b200.inputs import ffn_inputs
        D = c.Hq * c.d
        F = 4 * D
        _, w1, w2 = ffn_inputs(1, c.Hq, 1, c.d, F, rank_seed(c.seed, rank), device=dev)
        chunk = max(1, args.bpt_chunk)
        y = torch.empty((c.B, c.Sq, D), device=dev, dtype=torch.bfloat16)
        ws = torch.empty(max(16, fa.bpt_workspace_bytes(F, chunk)), dtype=torch.uint8, device=dev)
        fa.fa_fwd(q, k, v, o, lse, c.causal, c.scale, stream=stream)
        for _ in range(max(args.warmup, 1)):
            fa.fa_bpt_ffn(o, w1, w2, y, ws, chunk, stream=stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        pevs = []
        for _ in range(K):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fa.fa_bpt_ffn(o, w1, w2, y, ws, chunk, stream=stream)
            b.record(stream)
            pevs.append((a, b))
        torch.cuda.synchronize(dev)
        barrier(world)
        bpt_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in pevs)], world)[0]
        ffn_flops = 4.0 * c.B * c.Sq * D * F
        bpt_tf = ffn_flops / (bpt_ms * 1e-3 / K) / 1e12
        tiles = c.B * ((c.Sq + 127) // 128)
        n_chunks = (tiles + chunk - 1) // chunk
        bpt = {"value": aggregate_rate(world, ffn_flops, K, bpt_ms) / 1e12, "unit": "TFLOP/s",
               "ms_per_call": bpt_ms / K,
               "frac_of_measured_burst": bpt_tf / float(peaks["bf16_tflops"]),
               "algorithmic": "%.4g FLOP per call (two products, 2 x 2 x tokens x D x F; "
                              "D = %d, F = %d)" % (ffn_flops, D, F),
               "chunk_tiles": chunk, "hidden_bytes_per_chunk": chunk * 128 * F * 2,
               "hidden_bytes_unblocked": c.B * c.Sq * F * 2,
               "kernels": "fa_ffn_gemm_kernel, two launches per chunk",
               "gpu_launches": 2 * n_chunks * K, "traffic_main_kernel": None,
               "note": "y = W2 gelu(W1 x_t) on the forward's output; measured outside the step"}
        del y, ws, w1, w2

    # Paged cache: the same decode workload stored in page_size-key pages
    # scattered over a pool, read through a block table.  Measured on its own,
    # outside the step.
    paged = None
    if do_dec and not args.no_paged:
        from io_aware_exact_flashattention_b200.inputs import paginate
        kp, vp, bt = paginate(kc, vc, sl, args.page_size, rank_seed(cd.seed, rank))
        del kc, vc
        torch.cuda.empty_cache()
        ps_bytes = dec_bytes + int(sum((int(L) + args.page_size - 1) // args.page_size
                                       for L in sl.tolist())) * 4
        for _ in range(max(args.warmup, 1)):
            fa.fa_decode_paged_splitkv(qd, kp, vp, bt, sl, op, lp, cd.scale, stream=stream)
            fa.fa_combine(op, lp, od, lsed, stream=stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        pevs = []
        for _ in range(K):
            flush.fill_(1.0)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fa.fa_decode_paged_splitkv(qd, kp, vp, bt, sl, op, lp, cd.scale, stream=stream)
            fa.fa_combine(op, lp, od, lsed, stream=stream)
            b.record(stream)
            pevs.append((a, b))
        torch.cuda.synchronize(dev)
        barrier(world)
        pg_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in pevs)], world)[0]
        pg_gbs = aggregate_rate(world, ps_bytes, K, pg_ms) / 1e9
        per_gbs = ps_bytes / (pg_ms * 1e-3 / K) / 1e9
        paged = {"value": pg_gbs, "unit": "GB/s", "page_size": args.page_size,
                 "ms_per_call": pg_ms / K,
                 "frac_of_measured_copy": per_gbs / float(peaks["hbm_gbs"]),
                 "frac_of_8TBs": per_gbs / NOMINAL_HBM_GBS,
                 "bytes_per_call": ps_bytes, "gpu_launches": 2 * K,
                 "traffic": (profiled_traffic("decode_paged_b64_p16_d128.md", DECODE_SOURCES)
                             if args.page_size == 16 else None),
                 "kernels": "fa_decode_split_kernel<128,4> (paged loads) + fa_combine_kernel<128>",
                 "algorithmic": "K,V visible rows + q + O + LSE + block-table entries read",
                 "note": "same workload, pages scattered over the pool by a seeded permutation; "
                         "measured outside the step"}

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline and do_pre:
        cpu = cpu_baseline(c)

    line = {
        "metric": METRIC,
        "value": prefill_tflops if do_pre else dec_gbs,
        "unit": "TFLOP/s" if do_pre else "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": tot_ms / K,
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": c.name, "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "Sq": c.Sq,
                   "Skv": c.Skv, "d": c.d, "causal": c.causal, "q_mult": c.q_mult,
                   "decode_workload": cd.name if do_dec else None,
                   "l2": "flushed before every step (256 MB write), outside the timed regions",
                   "step": "fa_fwd on the prefill workload, then fa_decode_splitkv + fa_combine "
                           "on the decode workload",
                   "parallelism": "dp%d (independent replicas, per-rank seeds)" % world},
        "gpu_launches": K * ((1 if do_pre else 0) + (2 if do_dec else 0)),
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if do_pre:
        pre_launch_s = pre_ms * 1e-3 / K
        achieved = flops / pre_launch_s / 1e12
        peak = float(peaks["bf16_tflops"])
        line["prefill"] = {
            "tflops": prefill_tflops, "ms_per_launch": pre_ms / K,
            "frac_of_nominal_2250": achieved / NOMINAL_BF16_TFLOPS,
            "frac_of_measured_burst": achieved / peak,
            "frac_of_measured_sustained": achieved / float(peaks.get(
                "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))}
        line["roofline"] = {
            "bound": "tensor", "kernel": "fa_prefill_kernel<128>", "achieved": achieved,
            "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": "%s bf16 burst (MEASURED_PEAKS.json bf16_tflops)" % peaks_kind
            if peaks_kind == "measured" else "fallback 1590 TFLOP/s",
            "traffic": profiled_traffic("prefill_causal_mha_s2048_d128.md", PREFILL_SOURCES),
            "algorithmic": "%.4g FLOP per launch (4*B*Hq*Sq*Skv*d/2)" % flops}
    if do_dec:
        dec_launch_s = dec_ms * 1e-3 / K
        dec_achieved = dec_bytes / dec_launch_s / 1e9
        hbm = float(peaks["hbm_gbs"])
        line["decode"] = {
            "value": dec_gbs, "unit": "GB/s", "ms_per_step": dec_ms / K,
            "frac_of_8TBs": dec_achieved / NOMINAL_HBM_GBS,
            "frac_of_measured_copy": dec_achieved / hbm, "num_splits": n_split,
            "bytes_per_call": dec_bytes}
        line["roofline_decode"] = {
            "bound": "hbm", "kernel": "fa_decode_split_kernel<128,4> + fa_combine_kernel<128> (timed together)",
            "achieved": dec_achieved, "peak": hbm, "unit": "GB/s", "frac": dec_achieved / hbm,
            "peak_source": "%s copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" % peaks_kind,
            "traffic": profiled_traffic("decode_b64_splitkv_d128.md", DECODE_SOURCES),
            "algorithmic": "%d bytes per call (K,V visible rows + q + O + LSE)" % dec_bytes}
    # `roofline` describes the kernel that takes most of the step's time.
    if do_pre and do_dec and dec_ms > pre_ms:
        line["roofline_prefill"] = line.pop("roofline")
        line["roofline"] = line.pop("roofline_decode")
    elif do_dec and not do_pre:
        line["roofline"] = line.pop("roofline_decode")
    if paged is not None:
        line["decode_paged"] = paged
    if backward is not None:
        line["backward"] = backward
    if prefill_fp8 is not None:
        line["prefill_fp8"] = prefill_fp8
    if bpt is not None:
        line["bpt_ffn"] = bpt
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
