#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole path on synthetic, seeded inputs resident
in HBM: the fused prefill forward (fa_fwd) on the largest workload, causal GQA
B=1, Hq=32, Hkv=8, S=32768, d=128, followed by single-query split-KV decode
(fa_decode_splitkv + fa_combine) on B=64, Hq=32, Hkv=8, d=128 with KV lengths
uniform in [4096, 16384].  L2 is flushed (a 256 MB write) before every step,
outside the event-timed regions.

`value` is the prefill's TFLOP/s on that workload (FLOPs = 4*B*Hq*Sq*Skv*d,
halved for the causal mask) over all ranks; the decode's HBM GB/s is reported
beside it.  The three smaller prefill workloads are timed after the step, each
on its own (`configs`).  With N > 1 (torchrun) every rank runs the same per-GPU
work on its own seed (weak scaling, no data-path collective); times are the
max over ranks.

`--impl reference` times the fp64 CPU oracle instead, on a bounded sample of
the headline prefill workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

PREFILL_WORKLOAD = "causal_gqa_s32768_d128"
SIDE_WORKLOADS = ["mha_s512_d64", "causal_mha_s2048_d128_qx8", "causal_gqa_s8192_d128"]
EXTRAS_WORKLOAD = "causal_mha_s2048_d128_qx8"   # backward, E4M3 and feed-forward measurements
DECODE_WORKLOAD = "decode_b64_splitkv_d128"
METRIC = "attn fwd TFLOPS bf16 & % tensor peak; decode HBM GB/s & % of 8 TB/s"
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
CSRC = "io_aware_exact_flashattention_b200/csrc/"
SOURCES = {
    "prefill": [CSRC + "prefill_sm100.cuh", CSRC + "sm100.cuh"],
    "decode": [CSRC + "decode_sm100.cuh", CSRC + "sm100.cuh", CSRC + "launch_dep.cuh"],
    # the host file chooses the backward's CTA order, which sets its traffic
    "backward": [CSRC + "backward_sm100.cuh", CSRC + "sm100.cuh", CSRC + "launch_dep.cuh",
                 CSRC + "fa_api.cu"],
    "ffn": [CSRC + "ffn_sm100.cuh", CSRC + "sm100.cuh", CSRC + "launch_dep.cuh"],
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=PREFILL_WORKLOAD,
                    help="prefill workload of the step (io_aware_exact_flashattention_b200.inputs)")
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all",
                    help="restrict the step (for profiling captures)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="override the decode workload's batch (smaller profiling captures)")
    ap.add_argument("--decode-splits", type=int, default=None,
                    help="override the decode split count (default: fa_decode_default_splits)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the side measurements of the smaller prefill workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-paged", action="store_true",
                    help="skip the paged-cache decode measurement")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the backward measurement")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the E4M3-input forward measurement")
    ap.add_argument("--no-bpt", action="store_true",
                    help="skip the blockwise feed-forward network measurement")
    ap.add_argument("--extras-workload", default=EXTRAS_WORKLOAD,
                    help="workload of the backward, E4M3 and feed-forward measurements")
    ap.add_argument("--bpt-chunk", type=int, default=16,
                    help="query tiles per chunk of the blockwise feed-forward network")
    ap.add_argument("--bpt-layer-chunk", type=int, default=4,
                    help="query tiles per sequence per chunk of the blockwise layer")
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


def profiled_traffic(key):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    recorded in profiles/ncu_traffic.json for `key`, if they were taken on the
    kernel source as it is now (else None)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        entry = json.load(f).get(key)
    if not entry or entry.get("source_sha256_16") != sources_sha(SOURCES[entry["sources"]]):
        return None
    return int(entry["traffic_bytes_per_launch"])


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index, period_s=0.005):
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


def timed_calls(fn, steps, warmup, flush, stream, world, settle_s=1.0):
    """Run `fn` `warmup` times, then `steps` times with L2 flushed before each
    call (outside the timed region); return the total CUDA-event milliseconds
    of the timed calls, max over ranks.  Each side measurement starts after
    `settle_s` seconds idle, so it does not inherit the power-capped clocks
    of the long step before it."""
    torch.cuda.synchronize()
    time.sleep(settle_s)
    for _ in range(max(warmup, 1)):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    evs = []
    for _ in range(steps):
        flush.fill_(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks([sum(a.elapsed_time(b) for a, b in evs)], world)[0]


def row_sample(Sq, n_rows):
    """n_rows query rows spread evenly over [0, Sq): every causal row length
    from the shortest to the longest is represented."""
    n = max(1, min(Sq, n_rows))
    return sorted({(i * (Sq - 1)) // max(1, n - 1) for i in range(n)}) if n > 1 else [Sq - 1]


def row_flops(c, rows):
    """Exact multiply-add work of the named query rows: 4*d per visible key."""
    off = c.Skv - c.Sq
    keys = [min(c.Skv, i + off + 1) if c.causal else c.Skv for i in rows]
    return 4.0 * c.d * sum(max(0, k) for k in keys)


# ---------------------------------------------------------------------------
# the CPU oracle as a baseline (bounded sample of the prefill workload)
# ---------------------------------------------------------------------------

def oracle_rows_seconds(q, k, v, c, b, h, rows, lib):
    """Time the fp64 oracle on the named query rows of head (b, h)."""
    import oracle
    import numpy as np
    g = h // (c.Hq // c.Hkv)
    # exact fp64 copies made before the clock starts: only the oracle is timed
    qr = np.ascontiguousarray(q[b, h, rows].double().numpy())
    kb = np.ascontiguousarray(k[b:b + 1, g:g + 1].double().numpy())
    vb = np.ascontiguousarray(v[b:b + 1, g:g + 1].double().numpy())
    idx = [(0, 0, i) for i in rows]
    t0 = time.perf_counter()
    oracle.attn_rows(qr, kb, vb, idx, 1, c.Sq, c.causal, c.scale, lib=lib)
    return time.perf_counter() - t0


def cpu_baseline(c, q, k, v, target_s=15.0):
    """The oracle on an even row sample of one head of the workload (CPU copies
    of the same seeded inputs), sized to about `target_s` seconds."""
    import oracle
    lib = oracle.load()
    qc, kc, vc = (t[0:1].cpu() for t in (q, k, v))
    probe = row_sample(c.Sq, 64)
    t1 = oracle_rows_seconds(qc, kc, vc, c, 0, 0, probe, lib)
    n = int(64 * target_s / max(t1, 1e-3))
    rows = row_sample(c.Sq, n)
    t = oracle_rows_seconds(qc, kc, vc, c, 0, 0, rows, lib)
    flops = row_flops(c, rows)
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "fp64 oracle on %d query rows spread evenly over head (0, 0) of %s "
                      "(%.4g GFLOP of exact per-row work in %.2f s)"
                      % (len(rows), c.name, flops / 1e9, t)}


def run_reference(args, world, rank):
    """The oracle as the reference arm: each step is 1024 query rows, spread
    evenly over one (b, head) of the headline prefill workload, fp64 on the
    host cores."""
    if rank != 0:
        return
    import oracle
    from io_aware_exact_flashattention_b200.inputs import CONFIGS, prefill_inputs
    c = CONFIGS[args.workload]
    q, k, v = prefill_inputs(c.B, c.Hq, c.Hkv, c.Sq, c.Skv, c.d, c.seed, c.q_mult, device="cpu")
    lib = oracle.load()
    heads = [(b, h) for b in range(c.B) for h in range(c.Hq)]
    rows = row_sample(c.Sq, 1024)
    for i in range(args.warmup):
        b, h = heads[i % len(heads)]
        oracle_rows_seconds(q, k, v, c, b, h, rows, lib)
    t = 0.0
    for i in range(args.steps):
        b, h = heads[(args.warmup + i) % len(heads)]
        t += oracle_rows_seconds(q, k, v, c, b, h, rows, lib)
    flops = row_flops(c, rows) * args.steps
    value = flops / t / 1e12
    sample = ("fp64 oracle, %d query rows spread evenly over one (b, head) of %s per step"
              % (len(rows), c.name))
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": c.name, "B": c.B, "Hq": c.Hq, "Hkv": c.Hkv, "Sq": c.Sq,
                   "Skv": c.Skv, "d": c.d, "causal": c.causal, "q_mult": c.q_mult,
                   "sample_per_step": "%d rows of 1 of %d heads" % (len(rows), len(heads))},
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


def prefill_bytes(c):
    """Compulsory HBM bytes of one forward: Q, K, V read once; O, LSE written once."""
    return 2 * c.d * (2 * c.B * c.Hq * c.Sq + 2 * c.B * c.Hkv * c.Skv) + 4 * c.B * c.Hq * c.Sq


def tensor_fracs(tflops, peaks):
    return {"frac_of_measured_burst": tflops / float(peaks["bf16_tflops"]),
            "frac_of_measured_sustained": tflops / float(peaks.get(
                "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])),
            "frac_of_nominal_2250": tflops / NOMINAL_BF16_TFLOPS}


def run_ours(args, world, rank, local):
    from io_aware_exact_flashattention_b200 import fa
    from io_aware_exact_flashattention_b200.inputs import CONFIGS, decode_inputs, prefill_inputs
    fa.lib()  # fail loudly when the CUDA library is missing
    dev = torch.device("cuda", local)
    peaks, peaks_kind = load_peaks()
    do_pre = args.only in ("all", "prefill")
    do_dec = args.only in ("all", "decode")
    K = args.steps
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(64 * 1024 * 1024, device=dev, dtype=torch.float32)  # 256 MB > L2

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
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(K):
            step(evs[i])
        torch.cuda.synchronize(dev)
    barrier(world)
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    pre_ms, dec_ms, tot_ms = max_over_ranks([pre_ms, dec_ms, pre_ms + dec_ms], world)
    flops = c.flops()
    prefill_tflops = aggregate_rate(world, flops, K, pre_ms) / 1e12 if do_pre else None
    dec_gbs = aggregate_rate(world, dec_bytes, K, dec_ms) / 1e9 if do_dec else None

    # The smaller prefill workloads, each timed on its own after the step.
    side = {}
    if do_pre and not args.no_configs:
        for name in SIDE_WORKLOADS:
            cs = CONFIGS[name]
            qs, ks, vs = prefill_inputs(cs.B, cs.Hq, cs.Hkv, cs.Sq, cs.Skv, cs.d,
                                        rank_seed(cs.seed, rank), cs.q_mult, device=dev)
            os_, ls_ = torch.empty_like(qs), torch.empty((cs.B, cs.Hq, cs.Sq), device=dev)
            torch.cuda.synchronize()
            time.sleep(1.0)  # idle first: the step before ran power-capped
            with ClockSampler(local) as sclk:
                ms = timed_calls(lambda: fa.fa_fwd(qs, ks, vs, os_, ls_, cs.causal, cs.scale,
                                                   stream=stream), K, args.warmup, flush, stream,
                                 world, settle_s=0.0)
            tf = cs.flops() / (ms * 1e-3 / K) / 1e12
            side[name] = dict({"tflops": aggregate_rate(world, cs.flops(), K, ms) / 1e12,
                               "ms_per_launch": ms / K, "flops_per_launch": cs.flops(),
                               "B": cs.B, "Hq": cs.Hq, "Hkv": cs.Hkv, "S": cs.Sq, "d": cs.d,
                               "causal": cs.causal, "q_mult": cs.q_mult,
                               "clocks": sclk.summary()},
                              **tensor_fracs(tf, peaks))
            del qs, ks, vs, os_, ls_

    # e2e: the user-level call with pinned host buffers, copies inside the region
    e2e = None
    if not args.no_e2e and do_pre:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        lh = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        e2e_ms = timed_calls(lambda: fa.flash_attention(qh, kh, vh, causal=c.causal,
                                                        scale=c.scale, out=(oh, lh)),
                             K, args.warmup, flush, stream, world)
        e2e = {"value": aggregate_rate(world, flops, K, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int((q.numel() + k.numel() + v.numel()) * 2),
               "d2h_bytes_per_step": int(o.numel() * 2 + lse.numel() * 4),
               "ms_per_step": e2e_ms / K,
               "api": "io_aware_exact_flashattention_b200.flash_attention (host tensors)"}
        del qh, kh, vh, oh, lh

    extras = measure_extras(args, world, rank, dev, stream, flush, peaks, do_pre, do_dec,
                            cd if do_dec else None, (qd, kc, vc, sl, op, lp, od, lsed,
                                                      dec_bytes) if do_dec else None)

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline and do_pre:
        cpu = cpu_baseline(c, q, k, v)

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
                   "l2": "flushed before every step and every side measurement (256 MB "
                         "write), outside the timed regions; the step's inputs (0.7 GB "
                         "prefill, 2.8 GB decode) are larger than L2 as well",
                   "step": "fa_fwd on the prefill workload, then fa_decode_splitkv + fa_combine "
                           "on the decode workload",
                   "parallelism": "dp%d (independent replicas, per-rank seeds)" % world},
        "gpu_launches": K * ((1 if do_pre else 0) + (2 if do_dec else 0)),
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if do_pre:
        achieved = flops / (pre_ms * 1e-3 / K) / 1e12
        peak = float(peaks["bf16_tflops"])
        line["prefill"] = dict({"tflops": prefill_tflops, "ms_per_launch": pre_ms / K},
                               **tensor_fracs(achieved, peaks))
        line["roofline"] = {
            "bound": "tensor", "kernel": "fa_prefill_kernel<128>", "achieved": achieved,
            "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": ("measured bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
                            if peaks_kind == "measured" else "fallback 1590 TFLOP/s"),
            "traffic": profiled_traffic("prefill:" + c.name),
            "algorithmic": "%.4g FLOP per launch (4*B*Hq*Sq*Skv*d/2); compulsory bytes %d"
                           % (flops, prefill_bytes(c))}
        if side:
            line["configs"] = side
    if do_dec:
        dec_achieved = dec_bytes / (dec_ms * 1e-3 / K) / 1e9
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
            "traffic": profiled_traffic("decode:" + cd.name),
            "algorithmic": "%d bytes per call (K,V visible rows + q + O + LSE)" % dec_bytes}
    # `roofline` describes the kernel that takes most of the step's time.
    if do_pre and do_dec and dec_ms > pre_ms:
        line["roofline_prefill"] = line.pop("roofline")
        line["roofline"] = line.pop("roofline_decode")
    elif do_dec and not do_pre:
        line["roofline"] = line.pop("roofline_decode")
    line.update(extras)
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def measure_extras(args, world, rank, dev, stream, flush, peaks, do_pre, do_dec, cd, dec):
    """The rows beyond the hot path, each timed on its own after the step:
    backward, E4M3 inputs and the blockwise feed-forward network on the extras
    workload; decode over a paged cache on the decode workload."""
    from io_aware_exact_flashattention_b200 import fa
    from io_aware_exact_flashattention_b200.inputs import CONFIGS, prefill_inputs
    out = {}
    K = args.steps
    ce = CONFIGS[args.extras_workload]
    if do_pre and not (args.no_backward and args.no_fp8 and args.no_bpt):
        q, k, v = prefill_inputs(ce.B, ce.Hq, ce.Hkv, ce.Sq, ce.Skv, ce.d,
                                 rank_seed(ce.seed, rank), ce.q_mult, device=dev)
        o = torch.empty_like(q)
        lse = torch.empty((ce.B, ce.Hq, ce.Sq), device=dev, dtype=torch.float32)
        flops = ce.flops()
        fa.fa_fwd(q, k, v, o, lse, ce.causal, ce.scale, stream=stream)

        if not args.no_backward:
            from io_aware_exact_flashattention_b200.inputs import grad_output
            d_o = grad_output(q.shape, rank_seed(ce.seed, rank), device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            ws = torch.empty(fa.bwd_workspace_bytes(ce.B, ce.Hq, ce.Sq, ce.d), dtype=torch.uint8,
                             device=dev)
            bw_ms = timed_calls(lambda: fa.fa_bwd(q, k, v, o, lse, d_o, dq, dk, dv, ws, ce.causal,
                                                  ce.scale, stream=stream),
                                K, args.warmup, flush, stream, world)
            bw_flops = 2.5 * flops
            bw_tf = bw_flops / (bw_ms * 1e-3 / K) / 1e12
            out["backward"] = dict(
                {"value": aggregate_rate(world, bw_flops, K, bw_ms) / 1e12, "unit": "TFLOP/s",
                 "workload": ce.name, "ms_per_call": bw_ms / K},
                **tensor_fracs(bw_tf, peaks),
                algorithmic="%.4g FLOP per call (2.5 x the forward's: five products; the "
                            "kernel executes 3.5 x, its dQ CTAs recompute S and dP)" % bw_flops,
                kernels="fa_bwd_dsum_kernel (D and -LSE*log2e per query tile) + "
                        "fa_bwd_kernel<128> (dK/dV CTAs, then dQ CTAs)",
                traffic_main_kernel=profiled_traffic("backward:" + ce.name),
                gpu_launches=2 * K,
                note="dq, dk, dv from the forward's O and LSE; measured outside the step")
            del dq, dk, dv, ws, d_o

        if not args.no_fp8 and ce.d == 128:
            from io_aware_exact_flashattention_b200.inputs import fp8_prefill_inputs
            q8, k8, v8, dq8, dk8, dv8 = fp8_prefill_inputs(ce.B, ce.Hq, ce.Hkv, ce.Sq, ce.Skv,
                                                          ce.d, rank_seed(ce.seed, rank),
                                                          ce.q_mult, device=dev)
            f8_ms = timed_calls(lambda: fa.fa_fwd_fp8(q8, k8, v8, dq8, dk8, dv8, o, lse,
                                                      ce.causal, ce.scale, stream=stream),
                                K, args.warmup, flush, stream, world)
            f8_tf = flops / (f8_ms * 1e-3 / K) / 1e12
            f8_peak = 2.0 * float(peaks["bf16_tflops"])  # E4M3 dense rate = 2 x bf16 (4.5 / 2.25)
            out["prefill_fp8"] = {
                "value": aggregate_rate(world, flops, K, f8_ms) / 1e12, "unit": "TFLOP/s",
                "workload": ce.name, "ms_per_call": f8_ms / K, "dtype": "e4m3 (fp32 accumulate)",
                "roofline": {"bound": "tensor", "achieved": f8_tf, "peak": f8_peak,
                             "unit": "TFLOP/s", "frac": f8_tf / f8_peak,
                             "peak_source": "2 x measured bf16 burst (nominal e4m3:bf16 ratio "
                                            "4.5:2.25)",
                             "traffic": profiled_traffic("prefill_fp8:" + ce.name)},
                "frac_of_nominal_4500": f8_tf / (2.0 * NOMINAL_BF16_TFLOPS),
                "kernels": "fa_prefill_kernel<128, true>", "gpu_launches": K,
                "note": "same shape and FLOP count as the bf16 forward; measured outside the step"}
            del q8, k8, v8, dq8, dk8, dv8

        if not args.no_bpt and (ce.Hq * ce.d) % 256 == 0:
            from io_aware_exact_flashattention_b200.inputs import ffn_inputs
            D = ce.Hq * ce.d
            F = 4 * D
            _, w1, w2 = ffn_inputs(1, ce.Hq, 1, ce.d, F, rank_seed(ce.seed, rank), device=dev)
            chunk = max(1, args.bpt_chunk)
            y = torch.empty((ce.B, ce.Sq, D), device=dev, dtype=torch.bfloat16)
            ws = torch.empty(max(16, fa.bpt_workspace_bytes(F, chunk)), dtype=torch.uint8,
                             device=dev)
            bpt_ms = timed_calls(lambda: fa.fa_bpt_ffn(o, w1, w2, y, ws, chunk, stream=stream),
                                 K, args.warmup, flush, stream, world)
            ffn_flops = 4.0 * ce.B * ce.Sq * D * F
            bpt_tf = ffn_flops / (bpt_ms * 1e-3 / K) / 1e12
            tiles = ce.B * ((ce.Sq + 127) // 128)
            n_chunks = (tiles + chunk - 1) // chunk
            out["bpt_ffn"] = dict(
                {"value": aggregate_rate(world, ffn_flops, K, bpt_ms) / 1e12, "unit": "TFLOP/s",
                 "workload": ce.name, "ms_per_call": bpt_ms / K},
                **tensor_fracs(bpt_tf, peaks),
                algorithmic="%.4g FLOP per call (two products, 2 x 2 x tokens x D x F; D = %d, "
                            "F = %d)" % (ffn_flops, D, F),
                chunk_tiles=chunk, hidden_bytes_per_chunk=chunk * 128 * F * 2,
                hidden_bytes_unblocked=ce.B * ce.Sq * F * 2,
                kernels="fa_ffn_gemm_kernel, two launches per chunk",
                gpu_launches=2 * n_chunks * K,
                traffic_main_kernel=profiled_traffic("ffn:" + ce.name),
                note="y = W2 gelu(W1 x_t) on the forward's output; measured outside the step")
            # The blockwise layer: attention then the network, chunk by chunk.
            lchunk = max(1, args.bpt_layer_chunk)
            lse_l = torch.empty_like(lse)
            wsl = torch.empty(max(16, fa.bpt_layer_workspace_bytes(ce.B, ce.Hq, ce.d, F, lchunk)),
                              dtype=torch.uint8, device=dev)
            lay_ms = timed_calls(lambda: fa.fa_bpt_layer(q, k, v, w1, w2, y, lse_l, wsl,
                                                         ce.causal, ce.scale, lchunk,
                                                         stream=stream),
                                 K, args.warmup, flush, stream, world)
            lay_flops = flops + ffn_flops
            lay_tf = lay_flops / (lay_ms * 1e-3 / K) / 1e12
            n_chunks_l = (((ce.Sq + 127) // 128) + lchunk - 1) // lchunk
            out["bpt_layer"] = dict(
                {"value": aggregate_rate(world, lay_flops, K, lay_ms) / 1e12, "unit": "TFLOP/s",
                 "workload": ce.name, "ms_per_call": lay_ms / K},
                **tensor_fracs(lay_tf, peaks),
                algorithmic="%.4g FLOP per call (attention %.4g + network %.4g)"
                            % (lay_flops, flops, ffn_flops),
                chunk_tiles_per_sequence=lchunk,
                workspace_bytes=fa.bpt_layer_workspace_bytes(ce.B, ce.Hq, ce.d, F, lchunk),
                unblocked_activation_bytes=ce.B * ce.Sq * (D + F) * 2,
                kernels="per chunk: fa_prefill_kernel<128> (query-tile range) + two "
                        "fa_ffn_gemm_kernel",
                gpu_launches=3 * n_chunks_l * K,
                note="attention and network block by block; only one chunk's attention output "
                     "and hidden activations exist at a time; measured outside the step")
            del y, ws, w1, w2, wsl, lse_l
        del q, k, v, o, lse

    if do_dec and not args.no_paged:
        from io_aware_exact_flashattention_b200.inputs import paginate
        qd, kc, vc, sl, op, lp, od, lsed, dec_bytes = dec
        kp, vp, bt = paginate(kc, vc, sl, args.page_size, rank_seed(cd.seed, rank))
        ps_bytes = dec_bytes + int(sum((int(L) + args.page_size - 1) // args.page_size
                                       for L in sl.tolist())) * 4

        def paged_call():
            fa.fa_decode_paged_splitkv(qd, kp, vp, bt, sl, op, lp, cd.scale, stream=stream)
            fa.fa_combine(op, lp, od, lsed, stream=stream)
        pg_ms = timed_calls(paged_call, K, args.warmup, flush, stream, world)
        per_gbs = ps_bytes / (pg_ms * 1e-3 / K) / 1e9
        out["decode_paged"] = {
            "value": aggregate_rate(world, ps_bytes, K, pg_ms) / 1e9, "unit": "GB/s",
            "page_size": args.page_size, "ms_per_call": pg_ms / K,
            "frac_of_measured_copy": per_gbs / float(peaks["hbm_gbs"]),
            "frac_of_8TBs": per_gbs / NOMINAL_HBM_GBS,
            "bytes_per_call": ps_bytes, "gpu_launches": 2 * K,
            "traffic": profiled_traffic("decode_paged_p%d:%s" % (args.page_size, cd.name)),
            "kernels": "fa_decode_split_kernel<128,4> (paged loads) + fa_combine_kernel<128>",
            "algorithmic": "K,V visible rows + q + O + LSE + block-table entries read",
            "note": "same workload, pages scattered over the pool by a seeded permutation; "
                    "measured outside the step"}
        del kp, vp, bt
    return out


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
