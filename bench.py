"""Benchmark of the fused sm_100a attention forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]

A step is one launch of the fused kernel over the whole workload: every
(b, h, query tile) unit, i.e. every step of the hot path.  Inputs are
resident in HBM when the timed region starts and are larger than L2 (the
default workload reads 403 MB of Q, K, V; L2 is 126 MB), so no explicit
flush is needed.  Timing: W untimed warm-up steps, then K steps bracketed by
a barrier and a device synchronise on both sides, measured with CUDA events
on the launching stream, max over ranks.

Metric: attention forward TFLOP/s with FLOPs = 4*B*H*N^2*d (halved when
causal), bf16 operands with fp32 accumulation, whole job over all ranks.
With N GPUs each rank runs its own replica of the workload (the units are
independent; no collective on the data path): weak scaling.

`--impl reference` times the fp64 CPU oracle instead (the method's plain
definition on the host cores), each step a bounded sample of query rows of
the same workload, reported in the same unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_52_b200 import _binding as fb  # noqa: E402
from exact_io_aware_52_b200 import workloads  # noqa: E402

DEFAULT_WORKLOAD = 4  # long-context causal B1 H32 N16384 d128: the tensor-bound headline
METRIC = "attention fwd TFLOP/s (bf16, 1xB200) and % of dense BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["fa_fwd_kernel.cuh", "fa_softmax_row.cuh", "sm100_ptx.cuh"]  # device code of the d <= 128 kernel
# Dense bf16 tensor FLOPs per SM per clock of tcgen05 kind::f16 (one 128x128x128
# product group every 512 cycles); times the SM count and the sampled SM clock it
# gives the clock-derived dense peak, the second denominator of every fraction.
SM_TENSOR_FLOP_PER_CLK = 8192
# The other workloads of the spec table, measured in the same invocation
# as the headline (one `per_config` entry each).
PER_CONFIG = (1, 2, 3, 5)
PER_CONFIG_MIN_MS = 300.0  # each per-config timed region lasts at least this long (clock samples)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def tensor_peak(peaks: dict, elapsed_ms: float, ratio: float = 1.0):
    """The dense tensor peak a timed region is held to: the sustained figure
    (a seconds-long cuBLAS loop under the power cap) when the region ran back
    to back for at least a second, else the burst figure; times `ratio` for
    another operand type (the nominal dense ratio).  Returns (peak, label,
    burst, sustained)."""
    burst = float(peaks["bf16_tflops"]) * ratio
    sustained = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * ratio
    if elapsed_ms >= 1000.0:
        return sustained, "bf16_tflops_sustained (timed region >= 1 s back to back)", burst, sustained
    return burst, "bf16_tflops (burst; timed region < 1 s)", burst, sustained


def clock_peak_tflops(num_sms: int, sm_mhz: float, ratio: float = 1.0) -> float:
    """Dense tensor peak at a given SM clock: SMs x 8192 FLOP/clk x clock (x the
    nominal dense ratio of another operand type)."""
    return num_sms * SM_TENSOR_FLOP_PER_CLK * sm_mhz * 1e6 * ratio / 1e12


def percentiles(xs) -> dict:
    """Median, p10, p90 (linear interpolation between order statistics) and mean."""
    v = sorted(float(x) for x in xs)
    if not v:
        return {"median": None, "p10": None, "p90": None, "mean": None, "n": 0}

    def q(f):
        pos = f * (len(v) - 1)
        lo = int(math.floor(pos))
        hi = min(lo + 1, len(v) - 1)
        return v[lo] + (v[hi] - v[lo]) * (pos - lo)
    return {"median": q(0.5), "p10": q(0.1), "p90": q(0.9), "mean": sum(v) / len(v), "n": len(v)}


def effective_flops(w, k_len) -> float:
    """4*d FLOPs per (query, key) pair the mask allows, keys beyond each batch
    element's length excluded (the work the kernel cannot skip; equals
    w.flops() without key padding, up to the causal diagonal)."""
    if k_len is None:
        return w.flops()
    N, Nk = w.N, w.keys
    tot = 0
    for b in range(w.B):
        L = max(0, min(Nk, int(k_len[b])))
        if w.causal:
            tot += sum(max(0, min(L, i + 1 + Nk - N)) for i in range(N))
        else:
            tot += N * L
    return 4.0 * w.H * w.d * tot


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for name in (sources or KERNEL_SOURCES):
        with open(os.path.join(ROOT, "exact_io_aware_52_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload_id: int):
    """DRAM bytes per launch from a committed ncu record (profiles/*traffic.txt)
    of this workload, if it was taken on the current device sources of its
    kernel (the record's `sources` line), else None."""
    import glob
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*traffic.txt"))):
        rec = {}
        with open(path) as f:
            for line in f:
                if line.startswith("#") or not line.strip():
                    continue
                k, _, v = line.partition(" ")
                rec[k] = v.strip()
        if rec.get("workload") != str(workload_id):
            continue
        sources = rec.get("sources", "").split() or None
        if rec.get("source_hash") != kernel_source_hash(sources):
            continue
        try:
            return float(rec["dram_bytes_per_launch"])
        except (KeyError, ValueError):
            continue
    return None


def algorithmic_bytes(w, k_len) -> float:
    """Compulsory HBM bytes of one launch: Q, K, V read once (valid keys only
    under key padding), O (fp32) and lse written once."""
    n_elem = w.B * w.H * w.N * w.d
    eb = 1.0 if w.dtype == "e4m3" else 2.0
    kv_rows = w.kv_heads * (sum(min(max(int(x), 0), w.keys) for x in k_len) if k_len is not None else w.B * w.keys)
    return eb * n_elem + 2 * eb * kv_rows * w.d + 4.0 * n_elem + 4.0 * w.B * w.H * w.N


def memory_footprint(w, workspace_bytes: int = 0) -> dict:
    """Device memory of one forward call against that of the plain definition
    (page "FlashAttention (ES)", sections "El problema de la atencion estandar"
    and "Resultados empiricos"): the fused path holds Q, K, V, O and lse only
    (plus a key-split workspace; the library allocates nothing), while the
    definition also materialises the score matrix S = Q K^T of every head,
    B*H*N*N_k fp32 values (counted once: the softmax can overwrite S in place)."""
    eb = 1 if w.dtype == "e4m3" else 2
    io = (eb * w.B * w.H * w.N * w.d + 2 * eb * w.B * w.kv_heads * w.keys * w.d
          + 4 * w.B * w.H * w.N * w.d + 4 * w.B * w.H * w.N)
    scores = 4 * w.B * w.H * w.N * w.keys
    fused = io + workspace_bytes
    return {"fused_bytes": fused, "definition_bytes": io + scores, "score_matrix_bytes": scores,
            "ratio": (io + scores) / fused}


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    FIELDS = ["pci.bus_id", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        # raw samples go to FA_BENCH_OUT (default: the system temp dir); the
        # JSON line carries their summary
        out_dir = os.environ.get("FA_BENCH_OUT") or tempfile.gettempdir()
        os.makedirs(out_dir, exist_ok=True)
        self.path = os.path.join(out_dir, f"clocks_rank{device_index}.csv")
        props = torch.cuda.get_device_properties(device_index)
        self.bus = None  # "BB:DD" (bus:device, hex) of the GPU this rank uses
        try:
            self.bus = "%02X:%02X" % (props.pci_bus_id, props.pci_device_id)
        except AttributeError:
            pass

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) != len(self.FIELDS):
                    continue
                bus_dev = ":".join(parts[0].upper().split(".")[0].split(":")[-2:])
                if self.bus and bus_dev != self.bus:
                    continue
                rows.append(parts)
        if not rows:
            return None
        try:
            sm = [float(r[1]) for r in rows]
            smax = max(float(r[2]) for r in rows)
            power = [float(r[3]) for r in rows]
        except ValueError:
            return None
        loaded = [r for r, p in zip(rows, power) if p > 0.5 * max(power)] or rows
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in loaded:
            for name, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(float(r[1]) for r in loaded), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(power), "sm_mhz_min": min(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl != "ours":
        return world, rank, local  # the reference arm runs on rank 0 alone, no process group
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def workload_config(w, world: int, q_bytes: int) -> dict:
    """The `config` object of the JSON line (identical for both arms)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.kv_heads, "N": w.N, "N_k": w.keys, "d": w.d,
            "causal": w.causal, "key_splits": w.splits, "pass": w.pass_,
            "out": "fp32 O + fp32 lse" if w.pass_ == "fwd" else "fp32 dQ, dK, dV",
            "flops_per_step_per_gpu": w.flops(),
            "l2": "inputs larger than L2 (Q,K,V %.0f MB > 126 MB); no flush" % (q_bytes / 1e6),
            "parallelism": f"replicas x{world}"}


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """Largest value of x over all ranks (the timing rule: the slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_rows_flops(w, rows, k_len) -> float:
    """Nominal FLOPs of the given rows: 4*d per allowed score."""
    tot = 0
    for r in rows:
        bh, i = divmod(int(r), w.N)
        b = bh // w.H
        e = w.keys if k_len is None else max(0, min(w.keys, int(k_len[b])))
        if w.causal:
            e = min(e, max(0, i + 1 + w.keys - w.N))
        tot += e
    return 4.0 * w.d * tot


def exact_bf16(t):
    """E4M3 inputs widened exactly to bf16 (the oracle reads bf16); others as they are."""
    return t.to(torch.bfloat16) if t.dtype == torch.float8_e4m3fn else t


def cpu_oracle_rate(w, q, k, v, k_len, budget_s: float, seed: int = 0):
    """Time the fp64 oracle on rows of the workload for about budget_s seconds;
    returns (TFLOP/s in the metric's unit, threads, description, seconds)."""
    import numpy as np

    import oracle
    q, k, v = exact_bf16(q), exact_bf16(k), exact_bf16(v)
    threads = os.cpu_count() or 1
    rng = np.random.default_rng(seed)
    n_rows = w.B * w.H * w.N
    kl = None if k_len is None else k_len.tolist()
    batch = max(threads, 8)
    flops = 0.0
    done = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        rows = np.sort(rng.choice(n_rows, size=min(batch, n_rows), replace=False)).astype(np.int64)
        oracle.attention_f64(q, k, v, w.causal, w.scale, k_len=kl, rows=rows, nthreads=threads)
        flops += oracle_rows_flops(w, rows, kl)
        done += len(rows)
    dt = time.perf_counter() - t0
    desc = f"{done} uniformly sampled query rows of the workload (all keys of each row), {dt:.1f} s"
    return flops / dt / 1e12, threads, desc, dt


def bwd_oracle_sample(w, q, k, v, do, threads: int):
    """A bounded sample of a backward workload for the fp64 backward oracle:
    the first min(H, threads) query heads (with their key/value heads) and the
    first 1024 queries and keys; returns (callable, its FLOPs, description)."""
    import oracle
    n = min(w.N, 1024)
    hs = max(1, min(w.H, threads) // max(1, w.H // w.kv_heads) * max(1, w.H // w.kv_heads))
    hk = max(1, hs // max(1, w.H // w.kv_heads))
    sub = workloads.custom(1, hs, n, w.d, w.causal, H_kv=hk)
    qs, ks, vs, ds = (t[:1, :h, :n].contiguous() for t, h in ((q, hs), (k, hk), (v, hk), (do, hs)))
    flops = sub.flops() * 2.5

    def run():
        oracle.attention_bwd_f64(qs, ks, vs, ds, w.causal, w.scale, nthreads=threads)
    return run, flops, f"backward of the first {hs} heads x {n} queries and keys (fp64 oracle)"


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle, bounded sample per step."""
    w = workloads.WORKLOADS[args.workload]
    if rank != 0:
        return  # rank 0 alone times the oracle
    if w.pass_ == "bwd":
        return run_reference_bwd(args, world, w)
    q, k, v, k_len = workloads.make_inputs(w)
    import numpy as np

    import oracle
    threads = os.cpu_count() or 1
    rng = np.random.default_rng(1)
    kl = None if k_len is None else k_len.tolist()
    rows_per_step = max(threads, 8)
    n_rows = w.B * w.H * w.N

    qo, ko, vo = exact_bf16(q), exact_bf16(k), exact_bf16(v)

    def step():
        rows = np.sort(rng.choice(n_rows, size=rows_per_step, replace=False)).astype(np.int64)
        oracle.attention_f64(qo, ko, vo, w.causal, w.scale, k_len=kl, rows=rows, nthreads=threads)
        return oracle_rows_flops(w, rows, kl)

    for _ in range(args.warmup):
        step()
    flops = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        flops += step()
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world, (q.numel() + k.numel() + v.numel()) * q.element_size()),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: the fp64 oracle on {rows_per_step} uniformly sampled query "
                                   f"rows of the workload (all keys of each row); {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_bwd(args, world, w):
    q, k, v, _ = workloads.make_inputs(w)
    do = workloads.make_dout(w)
    threads = os.cpu_count() or 1
    run, flops_step, desc = bwd_oracle_sample(w, q, k, v, do, threads)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = flops_step * args.steps / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world, (q.numel() + k.numel() + v.numel()) * q.element_size()),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: {desc}; {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours_bwd(args, world, rank, local, w):
    """The backward pass (fa_bwd) of a forward computed once, untimed, by fa_fwd_ex."""
    import ctypes
    dev = torch.device("cuda", local)
    q, k, v, k_len = workloads.make_inputs(w)
    do = workloads.make_dout(w)
    qd, kd, vd, dod = q.to(dev), k.to(dev), v.to(dev), do.to(dev)
    kld = None if k_len is None else k_len.to(dev)
    o = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.float32, device=dev)
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=dev)
    fb.fa_fwd_ex(qd, kd, vd, o, lse, w.causal, w.scale, k_len=kld)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty(k.shape, dtype=torch.float32, device=dev)
    dv = torch.empty(v.shape, dtype=torch.float32, device=dev)
    ws = torch.empty(max(fb.bwd_workspace_bytes(qd), 16), dtype=torch.uint8, device=dev)
    params = fb.make_bwd_params(qd, kd, vd, o, lse, dod, dq, dk, dv, w.causal, w.scale, k_len=kld, workspace=ws)
    lib = fb.load()
    stream = torch.cuda.Stream(device=dev)
    sptr = fb._stream(stream)
    pref = ctypes.byref(params)

    def launch():
        st = lib.fa_bwd(pref, sptr)
        if st != fb.FA_OK:
            raise fb.FaError(st, "fa_bwd")

    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            launch()
    stream.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            launch()
            ev[i][1].record(stream)
        t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop() if sampler else None
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    kernel_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), world)
    flops = w.flops()
    value = flops * args.steps * world / (elapsed_ms * 1e-3) / 1e12

    # end to end: inputs from pinned host memory, gradients back to it, copies timed
    e2e = None
    if args.e2e_steps > 0:
        hosts = [t.pin_memory() for t in (q, k, v, do)] + [o.cpu().pin_memory(), lse.cpu().pin_memory()]
        devs = [qd, kd, vd, dod, o, lse]
        outs_h = [torch.empty(t.shape, dtype=torch.float32).pin_memory() for t in (dq, dk, dv)]

        def e2e_step():
            with torch.cuda.stream(stream):
                for hsrc, dst in zip(hosts, devs):
                    dst.copy_(hsrc, non_blocking=True)
                launch()
                for dsrc, hdst in zip((dq, dk, dv), outs_h):
                    hdst.copy_(dsrc, non_blocking=True)
        e2e_step()
        stream.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        e1.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        h2d = sum(t.numel() * t.element_size() for t in hosts)
        d2h = sum(t.numel() * t.element_size() for t in outs_h)
        e2e = {"value": flops * args.e2e_steps * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "ms_per_step": e2e_ms / args.e2e_steps, "api": "fa_bwd with torch pinned-memory copies"}
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    peak, peak_label, burst, sustained = tensor_peak(peaks, elapsed_ms)
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    n_elem = w.B * w.H * w.N * w.d
    kv_elem = w.B * w.kv_heads * w.keys * w.d
    # Q, dO, K, V (bf16) and O, lse (fp32) read; dQ, dK, dV (fp32) written once
    alg_bytes = 2.0 * (2 * n_elem + 2 * kv_elem) + 4.0 * n_elem + 4.0 * w.B * w.H * w.N + 4.0 * (n_elem + 2 * kv_elem)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
                "traffic": measured_traffic(args.workload), "peak_source": f"{peak_src} {peak_label}",
                "kernel": "fa_bwd_sm100_kernel + fa_bwd_prep_kernel (one event pair)", "kernel_ms": kernel_ms,
                "algorithmic_bytes": alg_bytes, "hbm_gbs_algorithmic": alg_bytes / (kernel_ms * 1e-3) / 1e9,
                "hbm_peak_gbs": float(peaks["hbm_gbs"])}
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        threads = os.cpu_count() or 1
        run, f_step, desc = bwd_oracle_sample(w, q, k, v, do, threads)
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < 10.0:
            run()
            n += 1
        dt = time.perf_counter() - t0
        cpu = {"value": f_step * n / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} x {desc}, {dt:.1f} s"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, world, (q.numel() + k.numel() + v.numel() + do.numel()) * 2),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * 2,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def time_graph_launches(launch, stream, dev, min_launches: int, min_ms: float, est_us: float):
    """Device time per launch of `launch` from CUDA-graph replays: a graph of G
    back-to-back launches (G chosen so one replay lasts about half a
    millisecond or more), replayed R times, each replay bracketed by CUDA
    events on the launching stream.  The graph removes the host's per-call
    cost, which is larger than the kernel on the small workloads.  Returns
    (per-launch ms of each replay, G, R, total ms)."""
    group = int(min(100, max(1, math.ceil(500.0 / max(est_us, 1.0)))))
    reps = max(math.ceil(min_launches / group), math.ceil(min_ms * 1e3 / (max(est_us, 1.0) * group)), 5)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(group):
            launch()
    g.replay()
    stream.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    torch.cuda.synchronize(dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for a, b in ev:
            a.record(stream)
            g.replay()
            b.record(stream)
        t1.record(stream)
    stream.synchronize()
    per = [a.elapsed_time(b) / group for a, b in ev]
    total = t0.elapsed_time(t1)
    del g
    return per, group, reps, total


def measure_per_config(args, local, peaks, num_sms):
    """The other spec workloads, each measured on this device right after
    the headline: device time per launch (median, p10, p90 over graph
    replays), TFLOP/s at the median, and the fraction of the measured peak
    (burst or sustained by the region's length) and of the clock-derived
    peak at the region's median SM clock."""
    dev = torch.device("cuda", local)
    out = {}
    lib = fb.load()
    import ctypes
    for wid in PER_CONFIG:
        w = workloads.WORKLOADS[wid]
        q, k, v, k_len = workloads.make_inputs(w)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        kld = None if k_len is None else k_len.to(dev)
        o = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.float32, device=dev)
        lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=dev)
        stream = torch.cuda.Stream(device=dev)
        params = fb.make_params(qd, kd, vd, o, lse, w.causal, w.scale, k_len=kld)
        pref, sptr = ctypes.byref(params), fb._stream(stream)

        def launch():
            st = lib.fa_fwd_ex(pref, sptr)
            if st != fb.FA_OK:
                raise fb.FaError(st, "fa_fwd_ex")

        with torch.cuda.stream(stream):
            for _ in range(max(args.warmup, 3)):
                launch()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            launch()
            e1.record(stream)
        stream.synchronize()
        est_us = e0.elapsed_time(e1) * 1e3
        sampler = ClockSampler(local)
        sampler.start()
        per, group, reps, total_ms = time_graph_launches(launch, stream, dev, args.steps, PER_CONFIG_MIN_MS, est_us)
        clocks = sampler.stop()
        st = percentiles(per)
        flops = w.flops()
        peak, _, burst, sustained = tensor_peak(peaks, total_ms)
        med_s = st["median"] * 1e-3
        tf = flops / med_s / 1e12
        entry = {
            "workload": w.name, "flops": flops,
            "timing": f"CUDA graph of {group} launches replayed {reps} times; per-launch device time = "
                      "replay time / launches (CUDA events on the launching stream)",
            "launches": group * reps, "region_ms": total_ms,
            "kernel_us": {kk: (vv * 1e3 if isinstance(vv, float) else vv) for kk, vv in st.items()},
            "tflops": tf, "tflops_p10_time": flops / (st["p10"] * 1e-3) / 1e12,
            "tflops_p90_time": flops / (st["p90"] * 1e-3) / 1e12,
            "frac": tf / peak, "frac_of_burst": tf / burst, "frac_of_sustained": tf / sustained,
            "algorithmic_bytes": algorithmic_bytes(w, k_len), "traffic": measured_traffic(wid),
            "clocks": clocks, "memory": memory_footprint(w),
        }
        if clocks and clocks.get("sm_mhz"):
            cp = clock_peak_tflops(num_sms, clocks["sm_mhz"])
            entry["clock_peak_tflops"] = cp
            entry["frac_of_clock_peak"] = tf / cp
        if k_len is not None:
            ef = effective_flops(w, k_len.tolist())
            entry["eff_flops"] = ef
            entry["eff_tflops"] = ef / med_s / 1e12
            entry["eff_note"] = "effective FLOPs: 4*d per (query, key) pair with the key inside its length"
        out[f"w{wid}"] = entry
        del qd, kd, vd, o, lse, kld
        torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the CUDA library has no CPU path)")
    fb.load()
    w = workloads.WORKLOADS[args.workload]
    if w.pass_ == "bwd":
        return run_ours_bwd(args, world, rank, local, w)
    dev = torch.device("cuda", local)
    q, k, v, k_len = workloads.make_inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    kld = None if k_len is None else k_len.to(dev)
    o = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.float32, device=dev)
    lse = torch.empty(w.B, w.H, w.N, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    splits = fb.suggest_splits(qd, kd) if w.splits < 0 else w.splits
    ws = None
    if splits > 1:
        ws = torch.empty(max(fb.workspace_bytes(qd, kd, splits), 16), dtype=torch.uint8, device=dev)
    params = fb.make_params(qd, kd, vd, o, lse, w.causal, w.scale, k_len=kld, num_splits=splits, workspace=ws)
    lib = fb.load()
    sptr = fb._stream(stream)
    import ctypes
    pref = ctypes.byref(params)

    def launch():
        st = lib.fa_fwd_ex(pref, sptr)
        if st != fb.FA_OK:
            raise fb.FaError(st, "fa_fwd_ex")

    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 3)):
            launch()
    stream.synchronize()

    # per-launch events on the launching stream (for the kernel's own duration)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            launch()
            ev[i][1].record(stream)
        t_end.record(stream)
    stream.synchronize()
    torch.cuda.synchronize(dev)
    barrier(world)
    clocks = sampler.stop() if sampler else None
    elapsed_ms = t_start.elapsed_time(t_end)
    per_launch = [a.elapsed_time(b) for a, b in ev]
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    kernel_ms = max_over_ranks(statistics.mean(per_launch), world)

    flops = w.flops()
    total_flops = flops * args.steps * world
    value = total_flops / (elapsed_ms * 1e-3) / 1e12

    # end to end through the public C ABI on host buffers (copies included)
    e2e = None
    if args.e2e_steps > 0:
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
        klh = None if k_len is None else k_len.pin_memory()
        oh = torch.empty(w.B, w.H, w.N, w.d, dtype=torch.float32).pin_memory()
        lh = torch.empty(w.B, w.H, w.N, dtype=torch.float32).pin_memory()
        fb.fa_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, o, lse, w.causal, w.scale, k_len_h=klh, k_len_d=kld,
                       stream=stream, num_splits=splits, workspace=ws)
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            fb.fa_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, o, lse, w.causal, w.scale, k_len_h=klh,
                           k_len_d=kld, stream=stream, num_splits=splits, workspace=ws)
        e1.record(stream)
        e1.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        h2d = (qh.numel() + kh.numel() + vh.numel()) * qh.element_size() + (0 if klh is None else klh.numel() * 4)
        d2h = oh.numel() * 4 + lh.numel() * 4
        e2e = {"value": flops * args.e2e_steps * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "ms_per_step": e2e_ms / args.e2e_steps}

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    # E4M3 products: the measured bf16 peak times the nominal dense FP8 / BF16 ratio (4.5 / 2.25)
    fp8 = w.dtype == "e4m3"
    peak, peak_label, burst, sustained = tensor_peak(peaks, elapsed_ms, 2.0 if fp8 else 1.0)
    alg_bytes = algorithmic_bytes(w, k_len)
    traffic = measured_traffic(args.workload)
    dist = percentiles(per_launch)
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
                "kernel_ms_median": dist["median"], "kernel_ms_p10": dist["p10"], "kernel_ms_p90": dist["p90"],
                "achieved_at_median": flops / (dist["median"] * 1e-3) / 1e12,
                "traffic": traffic,
                "peak_source": f"{peak_src} {peak_label}" + (" x 2 (nominal FP8/BF16 dense ratio)" if fp8 else ""),
                "kernel": ("fa_fwd_onetile_kernel" if w.d == 256 else "fa_fwd_sm100_kernel")
                          + (" + fa_combine_kernel (split pass and merge, one event pair)" if splits > 1 else ""),
                "kernel_ms": kernel_ms,
                "algorithmic_bytes": alg_bytes, "hbm_gbs_algorithmic": alg_bytes / (kernel_ms * 1e-3) / 1e9,
                "hbm_peak_gbs": float(peaks["hbm_gbs"])}
    if clocks and clocks.get("sm_mhz"):
        # the second denominator: SMs x 8192 dense FLOP/clk at the region's median SM clock
        cp = clock_peak_tflops(num_sms, clocks["sm_mhz"], 2.0 if fp8 else 1.0)
        roofline["clock_peak_tflops"] = cp
        roofline["frac_of_clock_peak"] = achieved / cp
    if k_len is not None:
        ef = effective_flops(w, k_len.tolist())
        roofline["eff_flops"] = ef
        roofline["eff_achieved"] = ef / (kernel_ms * 1e-3) / 1e12
    per_config = None
    if not args.no_per_config and world == 1 and args.workload == DEFAULT_WORKLOAD:
        per_config = measure_per_config(args, local, peaks, num_sms)
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        rate, threads, desc, _ = cpu_oracle_rate(w, q, k, v, k_len, budget_s=15.0)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
        "config": workload_config(w, world, (q.numel() + k.numel() + v.numel()) * q.element_size()),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * (2 if splits > 1 else 1),
        "clocks": clocks,
        "memory": memory_footprint(w, int(ws.numel()) if ws is not None else 0),
    }
    if per_config is not None:
        line["per_config"] = per_config
    print(json.dumps(line), flush=True)


def main():
    args = parse()
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
