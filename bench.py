"""Benchmark: Sol-Attn forward on one B200 per rank (effective TFLOP/s and ms per call).

Workload (default ``s64k``): B=1, H=32, d=128, N=65536 tokens (16x64x64 latent grid, t-major),
seeded BF16 Gaussian-random-field Q/K/V, tau tuned so 90 % of (query-block, key-block) pairs are
not exact.  A step is one ``sol_attn_fwd`` call: block summaries, threshold statistics, routing and
the fused attention kernel.  Inputs (3 x 537 MB) are larger than the 126 MB L2, so no flush is
needed between steps.

Effective FLOPs per step: 4 d (N^2 / Nb^2) E  for the exact pairs E (= 4 N^2 d H (1 - sp)) plus
4 d 64 (P - E) for the surrogate pairs, with P = B H Nb^2 and the realised sparsity sp reported by
the library.  ``value`` is the aggregate over all ranks (weak scaling: every rank runs its own
batch element on its own GPU; no data-path collective).

``--impl reference`` times the FP64 CPU oracle (the only reference implementation that exists for
this method) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn fwd ms & effective TFLOP/s vs BF16 peak, 32 heads d128, 32K–128K tok"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="s64k")
    ap.add_argument("--cpu-sample-heads", type=int, default=2,
                    help="heads (all query blocks each) the CPU oracle baseline evaluates")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--kv-splits", type=int, default=1,
                    help="split-KV shares per 128-row query tile (Sol-Attn only; 1 = off)")
    ap.add_argument("--m-tile", type=int, default=128, choices=[64, 128],
                    help="query rows per work unit of the fused kernel (128: two query blocks; 64: one)")
    ap.add_argument("--precision", default="bf16", choices=["bf16", "fp8"],
                    help="attention products in BF16 (default) or E4M3 with ExpCast weights (sol_attn*_fwd_fp8)")
    ap.add_argument("--no-fp8-leg", action="store_true",
                    help="skip the FP8 companion measurement that a one-GPU BF16 run adds to its line")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the other workloads of the metric's range that a one-GPU s64k run adds to its line")
    return ap.parse_args()


# the rest of the metric's range (32K-128K tokens, 32 heads), measured after the headline workload
LEG_WORKLOADS = ["sol2_64k", "s32k_80", "s32k_85", "s32k_90", "s128k"]


def rank_seed(workload, rank: int) -> int:
    """Seed of a rank's inputs: every rank runs its own batch element (weak scaling, no exchange)."""
    return workload.seed + 100 * rank


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of a list of floats over all ranks (the timing rule: slowest rank counts)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


TRAFFIC = {  # committed ncu DRAM records and the kernel source each was taken with
    "bf16": (os.path.join(ROOT, "profiles", "attn_fwd_dram_traffic.json"),
             os.path.join(ROOT, "block_sparse_attention_sum_b200", "csrc", "attn_fwd.cu")),
    "fp8": (os.path.join(ROOT, "profiles", "attn_fwd_fp8_dram_traffic.json"),
            os.path.join(ROOT, "block_sparse_attention_sum_b200", "csrc", "attn_fwd_fp8.cu")),
}


def kernel_source_digest(path: str) -> str:
    import hashlib

    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def measured_traffic(workload_name: str, precision: str = "bf16"):
    """DRAM bytes per launch of the fused kernel from a committed ncu capture, if that capture was
    taken on this workload with the current kernel source (else None)."""
    record, source = TRAFFIC[precision]
    if not os.path.exists(record):
        return None
    with open(record) as f:
        rec = json.load(f)
    entry = rec.get(workload_name)
    if not entry or entry.get("source_sha256") != kernel_source_digest(source):
        return None
    return entry["dram_bytes_per_launch"]


def union_useful_fraction(mask):
    """Share of the fused kernel's exact-tile work that is useful: a work unit pairs query blocks
    2u and 2u + 1 and computes both rows against every key block in the union of their exact sets,
    so useful / computed = (|E_2u| + |E_2u+1|) / (rows x |E_2u | E_2u+1|).  mask: bool [B, H, Nb, Nb]."""
    import numpy as np

    m = np.asarray(mask, dtype=bool)
    Nb = m.shape[-1]
    if Nb % 2:
        m = np.concatenate([m, np.zeros(m.shape[:-2] + (1, Nb), dtype=bool)], axis=-2)
    a, b = m[..., 0::2, :], m[..., 1::2, :]
    rows = 1 + np.any(b, axis=-1)          # a unit without a second query block has one row
    useful = a.sum() + b.sum()
    computed = (rows * (a | b).sum(axis=-1)).sum()
    return float(useful / max(computed, 1))


def load_peaks():
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def effective_flops(B, N, H, exact_pairs, total_pairs, d=128):
    Nb = (N + 63) // 64
    per_exact = 4.0 * d * (N / Nb) ** 2          # = 4 * 64 * 64 * d for full blocks
    per_surrogate = 4.0 * d * (N / Nb)           # one pooled key per unselected block and query
    exact_flops = per_exact * exact_pairs
    return exact_flops + per_surrogate * (total_pairs - exact_pairs), exact_flops


# ------------------------------------------------------------------------------------------ clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = os.path.join(os.environ.get("SOL_BENCH_CLOCKS_DIR", tempfile.gettempdir()),
                                 f"sol_bench_clocks_rank{device_index}.csv")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(device_index), "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                     util=float(parts[4]), hw=parts[6], hwt=parts[7], swt=parts[8], pcap=parts[9]))
                except ValueError:
                    continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        loaded = [r for r in rows if r["util"] >= 50] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded)}


# ------------------------------------------------------------------------------------ CPU baseline

def cpu_baseline(workload, heads, n_blocks: int, q=None, k=None, v=None, block_seed: int = 7):
    """The FP64 oracle, as it stands, on a bounded sample of the workload: for each (b, h) in
    ``heads`` its summaries and thresholds in full and ``n_blocks`` seeded query blocks (all of them
    if ``n_blocks`` >= Nb).  Returns the oracle's effective TFLOP/s on that sample."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import sol_attn_oracle as orc

    if q is None:
        q, k, v = workload.make_inputs("cpu")
    tau = workload.resolved_tau()
    Nb = orc.num_blocks(workload.N)
    if n_blocks >= Nb:
        blocks = list(range(Nb))
    else:
        blocks = sorted(np.random.default_rng(block_seed).choice(Nb, size=n_blocks, replace=False).tolist())
    fn = getattr(orc, workload.entry)
    t0 = time.perf_counter()
    r = fn(q, k, v, tau, workload.sink_start, workload.sink_tokens, qblocks=blocks, heads=heads)
    dt = time.perf_counter() - t0
    exact = total = 0
    for b, h in heads:
        rows = r["mask"][b, h][blocks]
        exact += int(rows.sum())
        total += rows.size
    flops, _ = effective_flops(1, workload.N, 1, exact, total)
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{workload.name}: {len(heads)} of {workload.B * workload.H} heads, {len(blocks)} of {Nb} "
                      f"query blocks each (their summaries and thresholds in full), FP64 numpy, {dt:.1f} s",
            "seconds": dt, "flops": flops}


# ---------------------------------------------------------------------------------------------- main

def fp8_leg(sa, w, q, k, v, out_bf16, tau, stream, flops_step, peaks, steps):
    """The FP8 entry point on the same inputs, after the BF16 measurement: ms per call, effective
    TFLOP/s, the fused kernel's own time against the E4M3 peak, and the relative l2 distance of its
    output from the BF16 output.  Any failure is reported in the object, never raised."""
    import torch

    try:
        fn = sa.sol_attn_fwd_fp8 if w.entry == "sol_attn" else sa.sol_attn2_fwd_fp8
        out = torch.empty_like(q)

        def step():
            fn(q, k, v, tau, w.sink_start, w.sink_tokens, out=out, stream=stream)

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        if sa.get_device_status() != 0:
            return {"error": "device status reports a timed-out wait after the FP8 warm-up"}
        n = max(3, min(steps, 10))
        sa.set_kernel_timing(True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        kernel_ms = sa.kernel_ms_sum(n) / n
        launches = sa.last_launch_count()
        sa.set_kernel_timing(False)
        if sa.get_device_status() != 0:
            return {"error": "device status reports a timed-out wait in the FP8 timed calls"}
        ms = a.elapsed_time(b) / n
        bf16_burst = float(peaks["bf16_tflops"])
        bf16_sust = float(peaks.get("bf16_tflops_sustained", bf16_burst))
        value = flops_step / (ms * 1e-3) / 1e12
        kernel_tflops = flops_step / (kernel_ms * 1e-3) / 1e12
        rel = float((out.float() - out_bf16.float()).norm() / out_bf16.float().norm())
        return {"entry": fn.__name__, "dtype": "e4m3", "steps": n, "warmup": 3, "ms_per_step": ms,
                "value": value, "unit": "TFLOP/s", "frac_of_peak": value / bf16_burst,
                "frac_of_sustained_peak": value / bf16_sust,
                "roofline": {"bound": "tensor", "achieved": kernel_tflops, "peak": 2.0 * bf16_sust,
                             "unit": "TFLOP/s", "frac": kernel_tflops / (2.0 * bf16_sust),
                             "traffic": measured_traffic(w.name, "fp8"),
                             "kernel": "attn_fwd_fp8_kernel", "kernel_ms": kernel_ms,
                             "peak_kind": f"e4m3 dense sustained = 2 x measured bf16 ({peaks['source']})"},
                "gpu_launches": launches * n, "rel_l2_vs_bf16_output": rel,
                "note": "same workload, inputs resident in HBM; clocks sampled for the BF16 leg only"}
    except Exception as e:   # reported, so that the BF16 line is printed whatever happens here
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def workload_leg(sa, w, inputs, dev, stream, steps, peaks):
    """One more workload timed like the headline one (inputs resident in HBM, CUDA events around
    ``steps`` calls after 3 warm-up calls, the fused kernel's own time from the library's events,
    SM clocks sampled during the timed calls).  Any failure is reported in the object, never raised."""
    import torch

    try:
        q, k, v = inputs
        out = torch.empty_like(q)
        tau = w.resolved_tau()
        fn = sa.sol_attn_fwd if w.entry == "sol_attn" else sa.sol_attn2_fwd

        def step():
            fn(q, k, v, tau, w.sink_start, w.sink_tokens, out=out, stream=stream)

        for _ in range(3):
            step()
        torch.cuda.synchronize()
        if sa.get_device_status() != 0:
            return {"error": "device status reports a timed-out wait after the warm-up"}
        exact, total, min_row, max_row = sa.last_stats()
        launches = sa.last_launch_count()
        # at least ~0.4 s of timed calls, so that the clock sampler (every 100 ms) sees the leg
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        torch.cuda.synchronize()
        steps = int(min(200, max(steps, math.ceil(400.0 / max(a.elapsed_time(b), 1e-3)))))
        clocks = ClockSampler(dev.index or 0)
        time.sleep(0.3)   # the sampler's first reading
        sa.set_kernel_timing(True)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
        clock_info = clocks.stop()
        kernel_ms = sa.kernel_ms_sum(steps) / steps
        sa.set_kernel_timing(False)
        if sa.get_device_status() != 0:
            return {"error": "device status reports a timed-out wait in the timed calls"}
        ms = a.elapsed_time(b) / steps
        flops, exact_flops = effective_flops(w.B, w.N, w.H, exact, total)
        if w.entry == "sol_attn2":
            flops = sol2_flops(w.B, w.N, w.H, exact, total)
        burst = float(peaks["bf16_tflops"])
        sust = float(peaks.get("bf16_tflops_sustained", burst))
        value = flops / (ms * 1e-3) / 1e12
        kernel_tflops = flops / (kernel_ms * 1e-3) / 1e12
        kname = "attn_fwd_kernel" + ("<false>" if w.entry == "sol_attn" else "<true>")
        sched = scheduler_stats(sa, step)
        return {"entry": fn.__name__, "scheduler": sched, "workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d=128", "tau": tau,
                "sink": [w.sink_start, w.sink_tokens], "target_sparsity": w.target_sparsity,
                "realised_sparsity": 1.0 - exact / total, "min_row": min_row, "max_row": max_row,
                "steps": steps, "warmup": 3, "ms_per_step": ms, "value": value, "unit": "TFLOP/s",
                "frac_of_peak": value / burst, "frac_of_sustained_peak": value / sust,
                "exact_only_tflops": exact_flops / (ms * 1e-3) / 1e12,
                "roofline": {"bound": "tensor", "achieved": kernel_tflops, "peak": burst, "unit": "TFLOP/s",
                             "frac": kernel_tflops / burst, "kernel": kname + " (fused attention)",
                             "kernel_ms": kernel_ms, "peak_kind": f"bf16 dense burst ({peaks['source']})"},
                "gpu_launches": launches * steps, "clocks": clock_info}
    except Exception as e:   # reported, so that the headline line is printed whatever happens here
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def scheduler_stats(sa, step):
    """One more call with per-CTA timing on: how evenly the hardware's CTA scheduler spreads the
    fused kernel's work units over the SMs.  tail_frac = (last SM's finish - median SM's finish) /
    kernel span; busy_frac = time inside CTAs / (span x SMs used)."""
    import numpy as np
    import torch

    sa.set_unit_timing(True)
    try:
        step()
        torch.cuda.synchronize()
        ut = sa.last_unit_times()
    finally:
        sa.set_unit_timing(False)
    start, end, sm = ut[:, 0], ut[:, 1], ut[:, 2]
    t0 = start.min()
    span = float(end.max() - t0)
    sms = np.unique(sm)
    finish = np.array([end[sm == s].max() - t0 for s in sms], dtype=np.float64)
    return {"units": int(len(ut)), "sms": int(len(sms)), "span_ms": span / 1e6,
            "tail_frac": float((finish.max() - np.median(finish)) / span),
            "busy_frac": float((end - start).sum() / (span * len(sms))),
            "unit_ms_mean": float((end - start).mean()) / 1e6, "unit_ms_max": float((end - start).max()) / 1e6}


def sol2_flops(B, N, H, exact_pairs, total_pairs, d=128):
    """Sol-Attn2 effective FLOPs: the exact pairs as for Sol-Attn; the tail costs 12 d per
    (anchor, unselected block) pair (S against the two groups, then [kbar_g | vbar_g]) and the
    first-order correction 2 d per query token."""
    Nb = (N + 63) // 64
    exact_flops = 4.0 * d * (N / Nb) ** 2 * exact_pairs
    anchors_per_block = (N / Nb) / 32.0
    return exact_flops + 12.0 * d * anchors_per_block * (total_pairs - exact_pairs) + 2.0 * d * B * H * N


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from block_sparse_attention_sum_b200.workloads import WORKLOADS

    w = WORKLOADS[args.workload]
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    if args.impl == "reference":
        # the reference arm is the FP64 oracle: each step is one head with 64 seeded query blocks
        if rank != 0:
            return 0
        q, k, v = w.make_inputs("cpu")
        flops = secs = 0.0
        base = None
        for i in range(args.warmup + args.steps):
            head = (0, i % w.H)
            base = cpu_baseline(w, [head], 64, q, k, v, block_seed=i)
            if i >= args.warmup:
                flops += base["flops"]
                secs += base["seconds"]
        value = flops / secs / 1e12
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "seq_len": w.N, "global_batch": w.B,
                           "parallelism": "cpu"},
                "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": base["cores"], "kind": "oracle",
                                 "sample": f"{w.name}: per step one head (cycling), 64 seeded query blocks, "
                                           "its summaries and thresholds in full; FP64 numpy"},
                "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist

    from block_sparse_attention_sum_b200 import sol_attn as sa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # inputs: seeded on the CPU (deterministic), pinned for the end-to-end leg; each rank its own batch element
    from block_sparse_attention_sum_b200.inputs import grf_qkv, iid_qkv

    seed = rank_seed(w, rank)
    if w.kind == "grf":
        qh, kh, vh = grf_qkv(w.B, w.H, w.grid, seed_base=seed)
    else:
        qh, kh, vh = iid_qkv(w.B, w.N, w.H, seed=seed)
    qh, kh, vh = (t.pin_memory() for t in (qh, kh, vh))
    q, k, v = (t.to(dev, non_blocking=True) for t in (qh, kh, vh))
    out = torch.empty_like(q)
    tau = w.resolved_tau()
    fp8 = args.precision == "fp8"
    if fp8 and args.kv_splits != 1:
        raise SystemExit("--kv-splits is not available with --precision fp8")
    if fp8:
        fn = sa.sol_attn_fwd_fp8 if w.entry == "sol_attn" else sa.sol_attn2_fwd_fp8
    else:
        fn = sa.sol_attn_fwd if w.entry == "sol_attn" else sa.sol_attn2_fwd
    stream = torch.cuda.current_stream()

    extra = {"kv_splits": args.kv_splits} if args.kv_splits != 1 else {}
    if args.m_tile != 128:
        if fp8:
            raise SystemExit("--m-tile 64 is available with --precision bf16 only")
        extra["m_tile"] = args.m_tile

    def step():
        fn(q, k, v, tau, w.sink_start, w.sink_tokens, out=out, stream=stream, **extra)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0, "device status after warm-up"
    exact, total, min_row, max_row = sa.last_stats()
    launches_per_step = sa.last_launch_count()

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- timed region: inputs resident in HBM
    clocks = ClockSampler(local_rank)
    time.sleep(0.3)   # the sampler's first reading
    sa.set_kernel_timing(True)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clock_info = clocks.stop()
    elapsed_ms = e0.elapsed_time(e1)
    kernel_ms = sa.kernel_ms_sum(min(args.steps, 256)) / min(args.steps, 256)
    sa.set_kernel_timing(False)
    assert sa.get_device_status() == 0, "device status after the timed region"

    sched = None if fp8 else scheduler_stats(sa, step)
    elapsed_ms, kernel_ms = max_over_ranks([elapsed_ms, kernel_ms], world, dev)
    ms_per_step = elapsed_ms / args.steps
    flops_step, exact_flops_step = effective_flops(w.B, w.N, w.H, exact, total)
    if w.entry == "sol_attn2":
        flops_step = sol2_flops(w.B, w.N, w.H, exact, total)
    value = flops_step * world / (ms_per_step * 1e-3) / 1e12
    sp = 1.0 - exact / total
    gmask, _ = sa.debug_route(q, k, tau, w.sink_start, w.sink_tokens)
    union_frac = union_useful_fraction(gmask.cpu().numpy())
    del gmask

    # ---- end to end through the public API with host buffers: the host-buffer entry point, whose
    # copies in (pinned host -> device) and out (device -> pinned host) run inside the timed region,
    # pipelined with the computation over head slices
    e2e = None
    if not args.no_e2e and not fp8 and args.kv_splits == 1 and args.m_tile == 128:
        out_h = torch.empty_like(qh).pin_memory()
        e2e_steps = max(3, min(args.steps, 10))
        host_fn = sa.sol_attn_fwd_host if w.entry == "sol_attn" else sa.sol_attn2_fwd_host

        def e2e_step():
            host_fn(qh, kh, vh, tau, w.sink_start, w.sink_tokens, out=out_h)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks([a.elapsed_time(b) / e2e_steps], world, dev)[0]
        e2e = {"value": flops_step * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 3 * qh.numel() * qh.element_size(),
               "d2h_bytes_per_step": out_h.numel() * out_h.element_size(), "steps": e2e_steps,
               "call": host_fn.__name__ + " (pinned host tensors in and out, head slices pipelined)",
               "matches_device_call": bool(torch.equal(out_h, out.cpu()))}

    peaks = load_peaks()
    # E4M3 products: the measured BF16 peak times the nominal dense FP8 / BF16 ratio (4.5 / 2.25)
    ratio = 2.0 if fp8 else 1.0
    peak_sust = ratio * float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    peak_burst = ratio * float(peaks["bf16_tflops"])
    achieved = flops_step / (kernel_ms * 1e-3) / 1e12
    kname = ("attn_fwd_fp8_kernel" if fp8 else "attn_fwd_kernel") + ("<false>" if w.entry == "sol_attn" else "<true>")
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_sust, "unit": "TFLOP/s",
                "frac": achieved / peak_sust, "traffic": measured_traffic(w.name, "fp8" if fp8 else "bf16"),
                "kernel": kname + " (fused attention)",
                "kernel_ms": kernel_ms,
                "peak_kind": (f"e4m3 dense sustained = 2 x measured bf16 ({peaks['source']})" if fp8 else
                              f"bf16 dense sustained ({peaks['source']})"),
                "frac_of_burst": achieved / peak_burst}

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d=128 GRF t-major {w.grid.T}x{w.grid.Y}x{w.grid.X}"
                                   if w.grid else w.name,
                       "global_batch": w.B * world, "seq_len": w.N, "heads": w.H, "tau": tau,
                       "target_sparsity": w.target_sparsity, "realised_sparsity": sp,
                       "union_tile_useful_fraction": union_frac, "kv_splits": args.kv_splits,
                       "m_tile": args.m_tile,
                       "min_row": min_row, "max_row": max_row, "scheduler": sched,
                       "precision": args.precision,
                       "parallelism": f"independent replicas x{world} (head/batch sharding, no exchange)",
                       "l2": "inputs 1.6 GB per rank > 126 MB L2; no flush"},
            # the metric is effective TFLOP/s against the BF16 peak, whatever the products' precision
            "frac_of_peak": value / world / (peak_burst / ratio),
            "frac_of_sustained_peak": value / world / (peak_sust / ratio),
            "exact_only_tflops": exact_flops_step * world / (ms_per_step * 1e-3) / 1e12,
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "clocks": clock_info}

    if world == 1 and not fp8 and not args.no_fp8_leg:
        line["fp8"] = fp8_leg(sa, w, q, k, v, out, tau, stream, flops_step, peaks, args.steps)
    if world == 1 and not fp8 and not args.no_legs and w.name == "s64k" and args.kv_splits == 1 and args.m_tile == 128:
        def inputs_key(x):   # workloads that differ only in tau target or sink share their inputs
            return x.input_key().split("@")[0].split("+")[0]

        legs, cache = {}, {inputs_key(w): (q, k, v)}
        for name in LEG_WORKLOADS:
            lw = WORKLOADS[name]
            key = inputs_key(lw)
            if key not in cache:
                cache.clear()
                torch.cuda.empty_cache()
                cache[key] = tuple(t.to(dev) for t in lw.make_inputs("cpu"))
            legs[name] = workload_leg(sa, lw, cache[key], dev, stream, max(5, min(args.steps, 10)), peaks)
        cache.clear()
        line["workloads"] = legs
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, [(0, h) for h in range(args.cpu_sample_heads)], 1 << 30, qh, kh, vh)
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
    if rank == 0:
        print(json.dumps(line), flush=True)
    leg_errors = [n for n, leg in (line.get("workloads") or {}).items() if "error" in leg]
    if world == 1 and ("error" in (line.get("fp8") or {}) or leg_errors):
        # the FP8 leg failed after the line was complete: report it through the exit status, and
        # leave without tearing down a CUDA context that may be unusable
        for n in leg_errors:
            sys.stderr.write(f"{n} leg: {line['workloads'][n]['error']}\n")
        if "error" in (line.get("fp8") or {}):
            sys.stderr.write(f"fp8 leg: {line['fp8']['error']}\n")
        sys.stderr.flush()
        os._exit(1)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
