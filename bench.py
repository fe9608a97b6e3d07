"""Benchmark: GPTQ-2D INT4 rounding of a 4096 x 4096 attention projection on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (one independent layer per rank)

One step = the whole path on one layer already resident in HBM: factor
preparation of both Kronecker factors (H_L, H_R: 4096 x 4096 fp32) and the
anti-diagonal rounding of W (4096 x 4096 bf16) with INT4 per-row scales.
Metric: weight entries rounded per second (m*n per step, summed over ranks).
Rank 0 prints one JSON line.

Reported beside it:
  roofline      the dominant kernel's algorithmic FLOP/s (CUDA events around
                its launches, on the launching stream) against the FP64
                tensor-core peak measured here (cuBLAS DGEMM 8192^3)
  e2e           the same metric through gptq2d_round_host from pinned host
                buffers: host->device inputs and device->host Q + statistics
                inside the timed region
  cpu_baseline  the fp64 CPU oracle on a bounded sample of the same workload
  clocks        nvidia-smi samples taken during the timed region
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "weight entries rounded/sec at 4096×4096 INT4 (1 B200); % of pipe roofline"
TB = 64


# --------------------------------------------------------------------------- #
# workload and algorithmic work
# --------------------------------------------------------------------------- #
def make_problem(name, seed, device_gram=True):
    import torch
    import workloads as WL

    def gram(X):
        Xt = torch.from_numpy(X).cuda()
        return (Xt.T @ Xt).cpu().numpy()

    mm = gram if device_gram else None
    if name == "attn":
        return WL.attn(seed, matmul=mm)
    if name == "mlp":
        return WL.mlp(seed, matmul=mm)
    if name == "small":
        return WL.small(seed)
    raise ValueError(name)


def far_flops(m, n):
    """Useful flops of the band products to tiles two or more 64-tiles away (far_kernel):
    entry (i, j) feeds 2 * (n - 64 (j//64 + 2)) flops right and 2 * (m - 64 (i//64 + 2)) down."""
    jt = np.arange(n) // TB
    it = np.arange(m) // TB
    right = m * np.sum(2.0 * np.maximum(0, n - TB * (jt + 2)))
    down = n * np.sum(2.0 * np.maximum(0, m - TB * (it + 2)))
    return float(right + down)


def sweep_flops(m, n):
    """Useful flops inside sweep_kernel: the in-tile pushes (entry (a, c) of a rows x cols tile
    pushes (cols-1-c) + (rows-1-a) FMAs) plus the pulled contributions of the neighbouring
    tiles (each entry feeds the next tile to the right and the next tile below)."""
    tot = 0.0
    for r in [min(TB, m - r0) for r0 in range(0, m, TB)]:
        for c in [min(TB, n - c0) for c0 in range(0, n, TB)]:
            tot += 2.0 * (r * c * (c - 1) / 2 + c * r * (r - 1) / 2)
    jt = np.arange(n) // TB
    it = np.arange(m) // TB
    near_r = m * np.sum(2.0 * np.clip(n - TB * (jt + 1), 0, TB))
    near_d = n * np.sum(2.0 * np.clip(m - TB * (it + 1), 0, TB))
    return float(tot + near_r + near_d)


def prep_flops(k):
    return k ** 3 / 3.0


# --------------------------------------------------------------------------- #
# clocks
# --------------------------------------------------------------------------- #
class ClockSampler:
    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        rows = []
        for ln in self.lines:
            p = [x.strip() for x in ln.split(",")]
            if len(p) < 10:
                continue
            if self.bus_id and self.bus_id[-12:] not in p[1].lower():
                continue
            rows.append(p)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[6 + k] == "Active"})
        pw = [float(r[4]) for r in rows if r[4].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "power_w_max": max(pw) if pw else None, "samples": len(rows)}


def bus_id_of(dev):
    import torch
    p = torch.cuda.get_device_properties(dev)
    for attr in ("pci_bus_id",):
        if hasattr(p, attr):
            dom = getattr(p, "pci_domain_id", 0)
            return f"{dom:08x}:{getattr(p, attr):02x}:{getattr(p, 'pci_device_id', 0):02x}.0"
    return ""


# --------------------------------------------------------------------------- #
# ncu traffic figures (profiles/ncu_traffic.txt: kernel, source sha256, bytes per launch, units)
# --------------------------------------------------------------------------- #
def ncu_traffic(kernel_class, src_file):
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(path):
        return None
    sha = hashlib.sha256(open(src_file, "rb").read()).hexdigest()[:16]
    for ln in open(path):
        if ln.startswith("#") or not ln.strip():
            continue
        p = ln.split()
        if len(p) >= 3 and p[0] == kernel_class and p[1] == sha:
            return float(p[2])
    return None


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def measure_dgemm_tflops():
    import torch
    n = 8192
    a = torch.randn(n, n, dtype=torch.float64, device="cuda")
    b = torch.randn(n, n, dtype=torch.float64, device="cuda")
    for _ in range(2):
        torch.matmul(a, b)
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.matmul(a, b)
        e1.record()
        e1.synchronize()
        best = max(best, 2 * n ** 3 / (e0.elapsed_time(e1) * 1e-3) / 1e12)
    del a, b
    torch.cuda.empty_cache()
    return best


def cpu_baseline(pb, sample):
    """The fp64 oracle as it stands on the host cores: LAPACK factors of both full Grams plus
    the anti-diagonal rounding of the leading sample x sample prefix (the prefix is a GPTQ-2D
    problem of its own), scaled to the full layer by the work ratio mn(m+n)."""
    import oracle as O
    m, n = pb.shape
    t0 = time.perf_counter()
    ML = O.reverse_cholesky(pb.H_L)
    MR = O.reverse_cholesky(pb.H_R)
    t_prep = time.perf_counter() - t0
    k = min(sample, m, n)
    t0 = time.perf_counter()
    O.gptq2d_antidiagonal(pb.W[:k, :k].astype(np.float64), ML[:k, :k], MR[:k, :k],
                          pb.scales[:k].astype(np.float64), pb.bits, pb.clamp)
    t_rnd = time.perf_counter() - t0
    t_full = t_prep + t_rnd * (m * n * (m + n)) / (k * k * 2 * k)
    try:
        from threadpoolctl import threadpool_info
        cores = max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        cores = os.cpu_count()
    return {"value": m * n / t_full, "unit": "entries/s", "cores": cores, "kind": "oracle",
            "sample": (f"LAPACK reverse Cholesky of both {m}x{m}/{n}x{n} Grams ({t_prep:.2f} s) + "
                       f"anti-diagonal oracle on the leading {k}x{k} prefix ({t_rnd:.2f} s), "
                       f"rounding time scaled by mn(m+n) to {m}x{n}: {t_full:.1f} s per layer")}


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def lpt_assign(costs, world: int):
    """Longest-processing-time-first assignment of independent layers to ranks: layers in
    descending cost (ties: lower index first), each to the least-loaded rank (ties: lower
    rank).  Every rank computes the same assignment; no collective is needed."""
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    load = [0.0] * world
    owner = [0] * len(costs)
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        owner[i] = r
        load[r] += costs[i]
    return owner


def rank_seed(rank: int) -> int:
    """Each rank rounds its own independent layer: the workload seed is the rank."""
    return rank


def aggregate_value(m: int, n: int, world: int, ms_step_max: float) -> float:
    """Whole-job entries/s: every rank rounds m*n entries per step; time is the slowest rank's."""
    return world * m * n / (ms_step_max * 1e-3)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import two_sided_adaptive_b200 as g
    from two_sided_adaptive_b200 import build as gbuild

    if rank == 0:
        gbuild.build()
    if world > 1:
        dist.barrier()
    g.lib()
    dev = torch.device("cuda", local_rank)
    pb = make_problem(args.workload, seed=rank_seed(rank))
    m, n = pb.shape
    W = torch.from_numpy(pb.W).to(dev).to(torch.bfloat16 if args.workload != "small" else torch.float32)
    H_L = torch.from_numpy(pb.H_L).to(dev)
    H_R = torch.from_numpy(pb.H_R).to(dev)
    s = torch.from_numpy(pb.scales).to(dev)
    M_L = torch.empty((m, m), dtype=torch.float64, device=dev)
    M_R = torch.empty((n, n), dtype=torch.float64, device=dev)
    wsQ = torch.empty(g.quantize_workspace_size(m, n), dtype=torch.uint8, device=dev)
    Q = torch.empty((m, n), dtype=torch.int8, device=dev)
    st = torch.empty(g.STATS_WORDS, dtype=torch.int64, device=dev)

    wsP = torch.empty(512, dtype=torch.uint8, device=dev)

    def step():
        g.prepare_pair(H_L, H_R, out_l=M_L, out_r=M_R, workspace=wsP, check=False)
        g.quantize(W, M_L, M_R, s, pb.bits, pb.clamp, out=Q, stats=st, workspace=wsQ)

    if args.profile_step:
        # one pass of the path and nothing else (for ncu captures of single kernels)
        step()
        torch.cuda.synchronize()
        return None

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    import ctypes
    for off in (0, 256):
        piv = ctypes.c_int64(-1)
        rc = g.lib().gptq2d_prepare_info(wsP.data_ptr() + off, None, ctypes.byref(piv))
        assert rc == 0, f"factor not SPD (pivot {piv.value})"
    stats = g.stats_dict(st)
    assert stats["status"] == 0, stats

    sampler = ClockSampler(bus_id_of(dev)) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    l0 = g.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    launches = g.launch_count() - l0
    clocks = sampler.stop() if sampler else None
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    ms_step = ms / args.steps
    value = aggregate_value(m, n, world, ms_step)

    # per-kernel device time: the same K steps again with a CUDA event pair around every
    # launch on its own stream; per-step figures are the totals / K
    g.profile_reset()
    g.profile_enable(True)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    prof = {k: (v[0] / args.steps, v[1] / args.steps) for k, v in g.profile_read().items()}
    g.profile_enable(False)
    g.profile_reset()

    # the two calls of a step on their own (events on the caller stream)
    def timed(fn, reps):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(reps):
            fn()
        f1.record()
        torch.cuda.synchronize()
        return f0.elapsed_time(f1) / reps
    reps = max(3, min(args.steps, 10))
    phases = {
        "prepare_pair": timed(lambda: g.prepare_pair(H_L, H_R, out_l=M_L, out_r=M_R,
                                                     workspace=wsP, check=False), reps),
        "quantize": timed(lambda: g.quantize(W, M_L, M_R, s, pb.bits, pb.clamp, out=Q, stats=st,
                                             workspace=wsQ), reps),
    }

    # the proxy loss of round-to-nearest on the same factors (the pages' baseline), and of
    # the rounding's own Q as a full quadratic form, outside the timed region
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    rtn_loss = g.proxy_loss(W, M_L, M_R, s, None, pb.bits, pb.clamp)
    f1.record()
    own_loss = g.proxy_loss(W, M_L, M_R, s, Q, pb.bits, pb.clamp)
    torch.cuda.synchronize()
    stats["rtn_loss"] = float(rtn_loss.item())
    stats["proxy_loss_quadratic_form"] = float(own_loss.item())
    stats["proxy_loss_ms"] = f0.elapsed_time(f1)

    # end to end through the C ABI from pinned host memory
    e2e = None
    if not args.no_e2e:
        wdt = torch.bfloat16 if args.workload != "small" else torch.float32
        Wh = torch.from_numpy(pb.W).to(wdt).pin_memory()
        HLh = torch.from_numpy(pb.H_L).pin_memory()
        HRh = torch.from_numpy(pb.H_R).pin_memory()
        sh = torch.from_numpy(pb.scales).pin_memory()
        Qh = torch.empty((m, n), dtype=torch.int8).pin_memory()
        sth = torch.empty(g.STATS_WORDS, dtype=torch.int64).pin_memory()
        wsH = torch.empty(g.round_host_workspace_size(m, n, g._dtype_code(Wh), g.DTYPE_F32),
                          dtype=torch.uint8, device=dev)
        g.round_host(Wh, HLh, HRh, sh, pb.bits, pb.clamp, workspace=wsH, Q_out=Qh, stats_out=sth)
        assert torch.equal(Qh, Q.cpu()), "round_host and device path disagree"
        ke = max(1, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for _ in range(ke):
            g.round_host(Wh, HLh, HRh, sh, pb.bits, pb.clamp, workspace=wsH, Q_out=Qh, stats_out=sth)
        f1.record()
        torch.cuda.synchronize()
        ems = max_over_ranks(f0.elapsed_time(f1) / ke, dev)
        def lower_bytes(k, esz):  # round_host copies each 64-row block of a Gram up to its diagonal
            return sum(min(64, k - r0) * min(k, r0 + 64) for r0 in range(0, k, 64)) * esz
        h2d = (Wh.numel() * Wh.element_size() + lower_bytes(m, HLh.element_size())
               + lower_bytes(n, HRh.element_size()) + sh.numel() * sh.element_size())
        d2h = Qh.numel() + sth.numel() * 8
        e2e = {"value": aggregate_value(m, n, world, ems), "unit": "entries/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ems, "api": "gptq2d_round_host"}

    if rank != 0:
        return None

    peak = measure_dgemm_tflops()
    # library context for the factor preparation: cuSOLVER's Cholesky (torch.linalg.cholesky,
    # fp64) of the same two Grams with their index order reversed (J H J = L L^T gives the
    # reverse factor M = J L^T J), one after the other on one stream, best of 3; the
    # reversals are outside the timing
    Hfl = [torch.flip(H.double(), dims=(0, 1)).contiguous() for H in (H_L, H_R)]
    for Hf in Hfl:
        torch.linalg.cholesky(Hf)
    torch.cuda.synchronize()
    chol_ms = 1e30
    for _ in range(3):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        for Hf in Hfl:
            torch.linalg.cholesky(Hf)
        f1.record()
        torch.cuda.synchronize()
        chol_ms = min(chol_ms, f0.elapsed_time(f1))
    del Hfl
    torch.cuda.empty_cache()
    dom = max(("propagate", "sweep", "prep_trailing", "prep_panel"), key=lambda k: prof[k][1])
    work = {"propagate": far_flops(m, n), "sweep": sweep_flops(m, n),
            "prep_trailing": prep_flops(m) + prep_flops(n), "prep_panel": None}
    nl, tms = prof[dom]
    src = {"propagate": "quantize.cu", "sweep": "quantize.cu", "prep_trailing": "prepare.cu",
           "prep_panel": "prepare.cu"}[dom]
    traffic = ncu_traffic(dom, os.path.join(ROOT, "two_sided_adaptive_b200", "csrc", src))
    achieved = (work[dom] / nl) / (tms / nl * 1e-3) / 1e12 if work[dom] else None
    roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": (achieved / peak) if achieved else None,
                "traffic": traffic, "launches_per_step": nl, "kernel_ms_per_step": tms,
                "algorithmic_flops_per_launch": work[dom] / nl if work[dom] else None,
                "peak_source": "cuBLAS DGEMM 8192^3 (torch.matmul fp64), best of 5, measured in this run",
                "timing": "CUDA events around every launch of this kernel over K profiled steps "
                          "run right after the timed region, averaged per launch"}
    breakdown = {k: {"launches": v[0], "ms": round(v[1], 4)} for k, v in prof.items()}
    phase_out = {k: {"ms": round(v, 4), "entries_per_s": m * n / (v * 1e-3)} for k, v in phases.items()}
    phase_out["quantize"]["fp64_tflops"] = m * n * (m + n) / (phases["quantize"] * 1e-3) / 1e12
    phase_out["quantize"]["frac_of_dgemm"] = phase_out["quantize"]["fp64_tflops"] / peak
    phase_out["prepare_pair"]["cusolver_cholesky_both_ms"] = chol_ms
    total_flops = m * n * (m + n) + prep_flops(m) + prep_flops(n)
    out = {
        "metric": METRIC, "value": value, "unit": "entries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": pb.name.split("_s")[0], "m": m, "n": n, "bits": pb.bits,
                   "w_dtype": str(W.dtype).replace("torch.", ""), "h_dtype": "float32",
                   "step": "prepare_pair(H_L, H_R) + quantize(W), inputs resident in HBM",
                   "l2": "no flush; per-step working set (W, H_L, H_R, factors, 3 fp64 feedback "
                         "buffers) is %.2f GB > 126 MB L2" % (
                             (W.numel() * W.element_size() + 2 * 4 * (m * m + n * n) + 8 * (m * m + n * n)
                              + wsQ_bytes(g, m, n)) / 1e9),
                   "parallelism": "independent layer per rank" if world > 1 else "single GPU"},
        "roofline": roofline,
        "gpu_launches": int(launches),
        "gpu_launches_per_step": launches / args.steps,
        "clocks": clocks,
        "e2e": e2e,
        "stats": stats,
        "breakdown_ms_per_step": breakdown,
        "phases": phase_out,
        "whole_step_fp64_tflops": total_flops / (ms_step * 1e-3) / 1e12,
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(pb, args.cpu_sample)
    return out


def wsQ_bytes(g, m, n):
    return g.quantize_workspace_size(m, n)


# --------------------------------------------------------------------------- #
# reference arm: the fp64 oracle on the host cores
# --------------------------------------------------------------------------- #
def run_reference(args):
    import oracle as O
    pb = make_problem(args.workload, seed=0, device_gram=False) if args.workload == "small" else None
    if pb is None:
        import workloads as WL
        pb = WL.attn(0) if args.workload == "attn" else WL.mlp(0)
    m, n = pb.shape
    k = min(args.ref_sample, m, n)

    def step():
        ML = O.reverse_cholesky(pb.H_L)
        MR = O.reverse_cholesky(pb.H_R)
        t0 = time.perf_counter()
        O.gptq2d_antidiagonal(pb.W[:k, :k].astype(np.float64), ML[:k, :k], MR[:k, :k],
                              pb.scales[:k].astype(np.float64), pb.bits, pb.clamp)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    t_rnd = 0.0
    for _ in range(args.steps):
        t_rnd += step()
    total = time.perf_counter() - t0
    t_prep = (total - t_rnd) / args.steps
    t_full = t_prep + (t_rnd / args.steps) * (m * n * (m + n)) / (k * k * 2 * k)
    try:
        from threadpoolctl import threadpool_info
        cores = max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        cores = os.cpu_count()
    value = m * n / t_full
    sample = (f"per step: LAPACK reverse Cholesky of both full Grams ({t_prep:.2f} s) + "
              f"anti-diagonal oracle on the leading {k}x{k} prefix, scaled by mn(m+n) to {m}x{n}")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "entries/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_full * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": pb.name.split("_s")[0], "m": m, "n": n, "bits": pb.bits},
            "cpu_baseline": {"value": value, "unit": "entries/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "entries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_block70b(args, rank: int = 0, world: int = 1):
    """Seconds per layer and for the whole block: the seven linear layers of one
    70B-class block (q, o: 8192x8192; k, v: 1024x8192; gate, up: 8192x28672; down:
    28672x8192), INT4 per-row absmax scales, W ~ N(0, 0.015^2) in bf16, Grams from
    Student-t(4) activations times U(0.1, 10) column scales with rows = width, plus 1%
    mean-diagonal damping.  The inputs are generated on the GPU (torch, seeded per
    layer) because the largest Gram is 28672^2, and stay resident.  Two schedules,
    each timed with CUDA events on its second pass:
      sequential  prepare_pair + quantize per layer, one after another;
      pipelined   one quantize_block call (the factors of the next layer prepared
                  beside the rounding of the current one), largest layers first.
    Under torchrun the layers are spread over the ranks by LPT on mn(m + n) (no
    collective on the data path); each rank times quantize_block on its share between
    barriers, and the block's time is the slowest rank's (the sequential schedule is
    then not timed)."""
    import torch
    import two_sided_adaptive_b200 as g
    from two_sided_adaptive_b200 import build as gbuild
    import workloads as WL
    gbuild.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    shapes = WL.block70b_shapes()
    owner = lpt_assign([m * n * (m + n) for _, m, n, _ in shapes], world)
    specs, names = [], []
    for li, (name, m, n, _) in enumerate(shapes):
        if owner[li] != rank:
            continue
        torch.manual_seed(1000 + li)

        def gram(width):
            z = torch.randn(width, width, device=dev, dtype=torch.float64)
            chi2 = torch.distributions.Chi2(torch.tensor(4.0, device=dev, dtype=torch.float64))
            X = z / torch.sqrt(chi2.sample((width, width)) / 4.0)
            del z
            X *= torch.empty(width, device=dev, dtype=torch.float64).uniform_(0.1, 10.0)[None, :]
            G = X.T @ X / width
            del X
            G = 0.5 * (G + G.T)
            G.diagonal().add_(0.01 * G.diagonal().mean())
            return G.float()
        HL, HR = gram(m), gram(n)
        W = (torch.randn(m, n, device=dev, dtype=torch.float32) * 0.015).to(torch.bfloat16)
        s = (W.float().abs().amax(dim=1) / 7.0).clamp_min(1e-30).contiguous()
        specs.append({"W": W, "H_L": HL, "H_R": HR, "scales": s, "bits": 4})
        names.append(name)
        torch.cuda.empty_cache()
    # sequential
    layers, total = [], 0.0
    for name, sp in zip(names, specs if world == 1 else []):
        m, n = sp["W"].shape
        ML = torch.empty((m, m), dtype=torch.float64, device=dev)
        MR = torch.empty((n, n), dtype=torch.float64, device=dev)
        wsP = torch.empty(512, dtype=torch.uint8, device=dev)
        wsQ = torch.empty(g.quantize_workspace_size(m, n), dtype=torch.uint8, device=dev)
        Q = torch.empty((m, n), dtype=torch.int8, device=dev)
        st = torch.empty(g.STATS_WORDS, dtype=torch.int64, device=dev)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        for rep in range(2):  # the first pass warms up
            torch.cuda.synchronize()
            e[0].record()
            g.prepare_pair(sp["H_L"], sp["H_R"], out_l=ML, out_r=MR, workspace=wsP, check=False)
            e[1].record()
            g.quantize(sp["W"], ML, MR, sp["scales"], 4, True, out=Q, stats=st, workspace=wsQ)
            e[2].record()
            torch.cuda.synchronize()
        sd = g.stats_dict(st)
        tp, tq = e[0].elapsed_time(e[1]) / 1e3, e[1].elapsed_time(e[2]) / 1e3
        total += tp + tq
        layers.append({"layer": name, "m": m, "n": n, "prepare_s": tp, "quantize_s": tq,
                       "entries_per_s": m * n / (tp + tq),
                       "quantize_fp64_tflops": m * n * (m + n) / tq / 1e12,
                       "status": sd["status"], "n_near_tie": sd["n_near_tie"]})
        del ML, MR, wsP, wsQ, Q, st
        torch.cuda.empty_cache()
    # pipelined: largest layers first
    order = sorted(range(len(specs)), key=lambda i: -(specs[i]["W"].shape[0] * specs[i]["W"].shape[1]
                                                      * sum(specs[i]["W"].shape)))
    bspecs = [specs[i] for i in order]
    ws = torch.empty(g.block_workspace_size(bspecs), dtype=torch.uint8, device=dev)
    tb = None
    import torch.distributed as dist
    multi = world > 1 and dist.is_initialized()
    for rep in range(2):
        if multi:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        Qs, sts = g.quantize_block(bspecs, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        if multi:
            dist.barrier()
        tb = e0.elapsed_time(e1) / 1e3
    tb = max_over_ranks(tb, device=dev)
    bstat = [g.stats_dict(st)["status"] for st in sts]
    return {"metric": "70B-class block: seconds for its 7 linear layers (INT4, %d B200)" % world,
            "value": tb, "unit": "s", "n_gpus": world, "higher_is_better": False,
            "dtype": "f64", "data": "synthetic (generated on the GPU, see run_block70b)",
            "config": {"workload": "block70b",
                       "step": "quantize_block (factors of the next layer beside the rounding "
                               "of the current one), largest first",
                       "order": [names[i] for i in order],
                       "parallelism": "layers by LPT over ranks" if world > 1 else "single GPU",
                       "owner": [shapes[i][0] + ":%d" % owner[i] for i in range(len(shapes))]},
            "sequential_s": total if world == 1 else None, "pipelined_s": tb,
            "pipelined_status": bstat,
            "block_workspace_gb": ws.numel() / 1e9, "layers": layers}


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count()


def run_configs(args):
    """Every workload of the rounding's configuration list, each timed on the GPU
    (prepare_pair + quantize, CUDA events, best of 3 after a warm-up pass) beside the
    fp64 oracle on this host's cores:
      tiny   64 x 64 fp64, unit scales, no clamp: the naive mn x mn Kronecker sweep and
             the anti-diagonal oracle, both in full;
      small  512 x 512, INT4, seeds 0-3: the anti-diagonal oracle in full;
      attn   4096 x 4096 INT4; mlp 4096 x 14336 INT4 and INT3: the oracle's factors in
             full and its rounding on the leading 1024 x 1024 prefix (a problem of its
             own), scaled to the layer by mn(m + n) (the rounding's work; the oracle's
             time grows as about k^3.07 over full k x k runs from 512 to 4096 on 16
             host cores, so the scaled figure is a lower bound);
    and the quantize call's fp64 rate against the cuBLAS DGEMM peak measured here."""
    import torch
    import oracle as O
    import two_sided_adaptive_b200 as g
    import workloads as WL
    from two_sided_adaptive_b200 import build as gbuild
    gbuild.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    peak = measure_dgemm_tflops()
    cores = cpu_cores()

    def gpu_gram(X):
        Xt = torch.from_numpy(X).cuda()
        return (Xt.T @ Xt).cpu().numpy()

    def gpu_time(pb, wdtype):
        m, n = pb.shape
        W = torch.from_numpy(np.ascontiguousarray(pb.W)).to(dev).to(wdtype)
        HL = torch.from_numpy(np.ascontiguousarray(pb.H_L)).to(dev)
        HR = torch.from_numpy(np.ascontiguousarray(pb.H_R)).to(dev)
        sc = torch.from_numpy(pb.scales).to(dev)
        ML = torch.empty((m, m), dtype=torch.float64, device=dev)
        MR = torch.empty((n, n), dtype=torch.float64, device=dev)
        wsP = torch.empty(512, dtype=torch.uint8, device=dev)
        wsQ = torch.empty(g.quantize_workspace_size(m, n), dtype=torch.uint8, device=dev)
        Q = torch.empty((m, n), dtype=torch.int8, device=dev)
        st = torch.empty(g.STATS_WORDS, dtype=torch.int64, device=dev)
        best = None
        for rep in range(4):  # the first pass warms up
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            torch.cuda.synchronize()
            e[0].record()
            g.prepare_pair(HL, HR, out_l=ML, out_r=MR, workspace=wsP, check=False)
            e[1].record()
            g.quantize(W, ML, MR, sc, pb.bits, pb.clamp, out=Q, stats=st, workspace=wsQ)
            e[2].record()
            torch.cuda.synchronize()
            t = (e[0].elapsed_time(e[1]) / 1e3, e[1].elapsed_time(e[2]) / 1e3)
            if rep > 0 and (best is None or sum(t) < sum(best)):
                best = t
        sd = g.stats_dict(st)
        sd["rtn_loss"] = float(g.proxy_loss(W, ML, MR, sc, None, pb.bits, pb.clamp).item())
        Qh = Q.cpu().numpy()
        del W, HL, HR, sc, ML, MR, wsP, wsQ, Q, st
        torch.cuda.empty_cache()
        return best, sd, Qh

    rows = []

    def record(name, pb, wdtype, cpu_s, cpu_how, agree=None):
        m, n = pb.shape
        (tp, tq), sd, _ = gpu_time(pb, wdtype)
        tf = m * n * (m + n) / tq / 1e12
        row = {"config": name, "m": m, "n": n, "bits": pb.bits if pb.clamp else None,
               "w_dtype": str(wdtype).replace("torch.", ""),
               "gpu_s_per_layer": tp + tq, "prepare_s": tp, "quantize_s": tq,
               "entries_per_s": m * n / (tp + tq),
               "quantize_fp64_tflops": tf, "quantize_frac_of_dgemm": tf / peak,
               "status": sd["status"], "n_near_tie": sd["n_near_tie"],
               "proxy_loss": sd["proxy_loss"], "rtn_loss": sd["rtn_loss"],
               "cpu_oracle_s_per_layer": cpu_s, "cpu_cores": cores, "cpu_how": cpu_how}
        if agree is not None:
            row["q_equals_oracle"] = agree
        rows.append(row)
        print(json.dumps(row), file=sys.stderr, flush=True)

    # tiny: both CPU oracles in full
    pb = WL.tiny(0)
    t0 = time.perf_counter()
    Q1, _ = O.babai_kron_sweep(pb.W, pb.H_L, pb.H_R, pb.scales.astype(np.float64), pb.bits,
                               pb.clamp)
    t_naive = time.perf_counter() - t0
    t0 = time.perf_counter()
    r = O.gptq2d(pb.W, pb.H_L, pb.H_R, pb.scales.astype(np.float64), pb.bits, pb.clamp)
    t_o2 = time.perf_counter() - t0
    _, _, Qg = gpu_time(pb, torch.float64)
    record("tiny 64x64 fp64 (s=1, no clamp)", pb, torch.float64, t_o2,
           f"anti-diagonal oracle in full ({t_o2:.3f} s); naive mn x mn Kronecker sweep in full "
           f"({t_naive:.2f} s)", bool(np.array_equal(Qg, r.Q) and np.array_equal(Q1, r.Q)))
    # small, seeds 0-3: the anti-diagonal oracle in full
    for seed in range(4):
        pb = WL.small(seed)
        t0 = time.perf_counter()
        r = O.gptq2d(pb.W.astype(np.float64), pb.H_L, pb.H_R, pb.scales.astype(np.float64),
                     pb.bits, pb.clamp)
        t_o2 = time.perf_counter() - t0
        _, _, Qg = gpu_time(pb, torch.float32)
        record(f"small 512x512 INT4 seed {seed}", pb, torch.float32, t_o2,
               "anti-diagonal oracle in full (LAPACK factors included)",
               bool(np.array_equal(Qg, r.Q)))
    # attn and mlp: factors in full, rounding on a 1024 x 1024 prefix, scaled by mn(m+n)
    k = 1024
    for name, pb in (("attn 4096x4096 INT4", WL.attn(0, matmul=gpu_gram)),
                     ("mlp 4096x14336 INT4", WL.mlp(0, bits=4, matmul=gpu_gram)),
                     ("mlp 4096x14336 INT3", WL.mlp(0, bits=3, matmul=gpu_gram))):
        m, n = pb.shape
        t0 = time.perf_counter()
        ML = O.reverse_cholesky(pb.H_L)
        MR = O.reverse_cholesky(pb.H_R)
        t_f = time.perf_counter() - t0
        W64 = torch.from_numpy(pb.W).to(torch.bfloat16).double().numpy()
        t0 = time.perf_counter()
        O.gptq2d_antidiagonal(W64[:k, :k], ML[:k, :k], MR[:k, :k],
                              pb.scales[:k].astype(np.float64), pb.bits, pb.clamp)
        t_r = time.perf_counter() - t0
        scale = m * n * (m + n) / (k * k * 2 * k)
        record(name, pb, torch.bfloat16, t_f + t_r * scale,
               f"LAPACK factors in full ({t_f:.2f} s) + anti-diagonal rounding of the leading "
               f"{k}x{k} prefix ({t_r:.2f} s) x {scale:.1f} (mn(m+n) ratio): extrapolated")
        del ML, MR
    return {"metric": "seconds per layer and entries/s for every configuration (1 B200), "
                      "beside the fp64 CPU oracle",
            "value": None, "unit": "s", "n_gpus": 1, "higher_is_better": False, "dtype": "f64",
            "data": "synthetic", "dgemm_peak_tflops": peak, "cpu_cores": cores,
            "config": {"workload": "configs"}, "configs": rows}


def run_kron3(args):
    """Hessians with three Kronecker factors.  The line's workload: W is a 4096 x 64 x 64
    tensor (a 4096 x 4096 layer whose input dimension is split into 64 groups of 64, each
    mode with its own factor), H = H_1 kron H_2 kron H_3 with H_1 4096^2 and H_2, H_3
    64^2; beside it a wide case, 1024 x 128 x 64 (n = 8192 columns: the right factor
    dominates).  INT4 per-mode-1 absmax scales, W ~ N(0, 0.02^2) in bf16, Grams from
    Student-t(4) activations times U(0.1, 10) column scales (4096 rows for a factor of
    width >= 1024, else 4 x width) plus 1% mean-diagonal damping, generated on the GPU.
    A third case, 256 x 4096 x 64 (n = 262,144 columns), runs the per-mode route only:
    the dense route's n x n factor would take 550 GB.
    Two routes, each timed with CUDA events over K steps after W warm-up steps, inputs
    resident in HBM:
      per-mode: prepare(H_1), prepare(H_2), prepare(H_3), quantize_kron (the right
                factor kept per mode; the line's value);
      dense:    the same prepares, kron_factor(M_2, M_3) and quantize of the m x n view
                with the n x n right factor."""
    import torch
    import two_sided_adaptive_b200 as g
    from two_sided_adaptive_b200 import build as gbuild
    gbuild.build()
    dev = torch.device("cuda", 0)

    def gram(width, rows):
        z = torch.randn(rows, width, device=dev, dtype=torch.float64)
        chi2 = torch.distributions.Chi2(torch.tensor(4.0, device=dev, dtype=torch.float64))
        X = z / torch.sqrt(chi2.sample((rows, width)) / 4.0)
        X *= torch.empty(width, device=dev, dtype=torch.float64).uniform_(0.1, 10.0)[None, :]
        G = X.T @ X / rows
        G = 0.5 * (G + G.T)
        G.diagonal().add_(0.01 * G.diagonal().mean())
        return G.float()

    def case(dims, seed, dense=True):
        torch.manual_seed(seed)
        Hs = [gram(d, 4096 if d >= 1024 else 4 * d) for d in dims]
        m, n = dims[0], dims[1] * dims[2]
        W = (torch.randn(dims, device=dev, dtype=torch.float32) * 0.02).to(torch.bfloat16)
        W2 = W.reshape(m, n)
        s = (W2.float().abs().amax(dim=1) / 7.0).clamp_min(1e-30).contiguous()
        Ms = [torch.empty((d, d), dtype=torch.float64, device=dev) for d in dims]
        wsP = [torch.empty(max(g.prepare_workspace_size(d), 256), dtype=torch.uint8, device=dev)
               for d in dims]
        wsK = torch.empty(g.quantize_kron_workspace_size(m, dims[1:]), dtype=torch.uint8,
                          device=dev)
        Q = torch.empty((m, n), dtype=torch.int8, device=dev)
        Qd = torch.empty((m, n), dtype=torch.int8, device=dev)
        st = torch.empty(g.STATS_WORDS, dtype=torch.int64, device=dev)
        std = torch.empty(g.STATS_WORDS, dtype=torch.int64, device=dev)
        dense_ws = {}

        def step(dense, ev=None):
            if ev:
                ev[0].record()
            for H, M, ws in zip(Hs, Ms, wsP):
                g.prepare(H, out=M, workspace=ws, check=False)
            if dense:
                g.kron_factor(Ms[1:], out=dense_ws["MR"])
            if ev:
                ev[1].record()
            if dense:
                g.quantize(W2, Ms[0], dense_ws["MR"], s, 4, True, out=Qd, stats=std,
                           workspace=dense_ws["ws"])
            else:
                g.quantize_kron(W2, Ms[0], Ms[1:], s, 4, True, out=Q, stats=st, workspace=wsK)
            if ev:
                ev[2].record()

        def timed(dense):
            for _ in range(args.warmup):
                step(dense)
            torch.cuda.synchronize()
            tp = tq = 0.0
            for _ in range(args.steps):
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                step(dense, ev)
                torch.cuda.synchronize()
                tp += ev[0].elapsed_time(ev[1])
                tq += ev[1].elapsed_time(ev[2])
            return tp / args.steps, tq / args.steps

        tp, tq = timed(False)
        sd = g.stats_dict(st)
        if not dense:  # the dense route's n x n factor would not fit
            out = {"dims": list(dims), "ms_per_step": tp + tq,
                   "entries_per_s": m * n / ((tp + tq) * 1e-3), "prepare_ms": tp,
                   "quantize_kron_ms": tq, "per_mode_workspace_bytes": wsK.numel(),
                   "dense_route": {"n_by_n_factor_bytes": 8 * n * n, "run": False},
                   "status": sd["status"], "n_near_tie": sd["n_near_tie"],
                   "proxy_loss": sd["proxy_loss"]}
            del Hs, Ms, wsP, wsK
            torch.cuda.empty_cache()
            return out
        dense_ws["MR"] = torch.empty((n, n), dtype=torch.float64, device=dev)
        dense_ws["ws"] = torch.empty(g.quantize_workspace_size(m, n), dtype=torch.uint8, device=dev)
        tpd, tqd = timed(True)
        sdd = g.stats_dict(std)
        out = {"dims": list(dims), "ms_per_step": tp + tq, "entries_per_s": m * n / ((tp + tq) * 1e-3),
               "prepare_ms": tp, "quantize_kron_ms": tq,
               "per_mode_workspace_bytes": wsK.numel(),
               "dense_route": {"ms_per_step": tpd + tqd, "prepare_and_kron_ms": tpd,
                               "quantize_ms": tqd,
                               "workspace_bytes": dense_ws["ws"].numel() + dense_ws["MR"].numel() * 8},
               "routes_differ_at": int((Q != Qd).sum()), "status": sd["status"],
               "dense_status": sdd["status"], "n_near_tie": sd["n_near_tie"],
               "proxy_loss": sd["proxy_loss"], "dense_proxy_loss": sdd["proxy_loss"]}
        del dense_ws["MR"], dense_ws["ws"], Hs, Ms, wsP, wsK
        torch.cuda.empty_cache()
        return out

    if args.profile_step:  # one per-mode rounding of the 4096 x 64 x 64 case (ncu input)
        torch.manual_seed(77)
        dims = (4096, 64, 64)
        Hs = [gram(d, 4096 if d >= 1024 else 4 * d) for d in dims]
        W2 = (torch.randn((dims[0], dims[1] * dims[2]), device=dev) * 0.02).to(torch.bfloat16)
        s = (W2.float().abs().amax(dim=1) / 7.0).clamp_min(1e-30).contiguous()
        Ms = [g.prepare(H, check=False) for H in Hs]
        g.quantize_kron(W2, Ms[0], Ms[1:], s, 4, True)
        torch.cuda.synchronize()
        return None
    main = case((4096, 64, 64), 77)
    wide = case((1024, 128, 64), 78)
    huge = case((256, 4096, 64), 79, dense=False)
    return {"metric": "weight entries rounded per second, 3-factor Kronecker Hessian (INT4, 1 B200)",
            "value": main["entries_per_s"], "unit": "entries/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
            "higher_is_better": True, "dtype": "f64",
            "data": "synthetic (generated on the GPU, see run_kron3)",
            "config": {"workload": "kron3", "dims": main["dims"], "bits": 4,
                       "step": "prepare x3 + quantize_kron (per-mode right factor)"},
            "cases": [main, wide, huge]}


def run_grid128(args):
    """The 4096 x 4096 INT4 attention layer of the headline metric on a grid variant:
    128-column groups, asymmetric (integer zero points from each group's min/max, the
    usual GPTQ convention), packed 4-bit output, through gptq2d_quantize_grid.  Inputs as
    for the headline line (workloads.attn, Grams formed on the GPU); one step =
    prepare_pair + quantize_grid, timed with CUDA events over K steps after W warm-ups."""
    import torch
    import two_sided_adaptive_b200 as g
    from two_sided_adaptive_b200 import build as gbuild
    import workloads as WL
    gbuild.build()
    pb = make_problem("attn", seed=0, device_gram=True)
    m, n = pb.W.shape
    dev = torch.device("cuda", 0)
    W = torch.from_numpy(pb.W).to(dev).to(torch.bfloat16)
    S, Z = WL.group_minmax_grid(W.double().cpu().numpy(), 4, 128)
    S, Z = torch.from_numpy(S).to(dev), torch.from_numpy(Z).to(dev)
    HL, HR = torch.from_numpy(pb.H_L).to(dev), torch.from_numpy(pb.H_R).to(dev)
    ML = torch.empty((m, m), dtype=torch.float64, device=dev)
    MR = torch.empty((n, n), dtype=torch.float64, device=dev)
    wsP = torch.empty(512, dtype=torch.uint8, device=dev)
    wsQ = torch.empty(g.quantize_workspace_size(m, n), dtype=torch.uint8, device=dev)
    Q = torch.empty((m, (n + 1) // 2), dtype=torch.uint8, device=dev)
    st = torch.empty(g.STATS_WORDS, dtype=torch.int64, device=dev)

    def step(ev=None):
        if ev:
            ev[0].record()
        g.prepare_pair(HL, HR, out_l=ML, out_r=MR, workspace=wsP, check=False)
        if ev:
            ev[1].record()
        g.quantize_grid(W, ML, MR, S, 4, True, group_size=128, zeros=Z, packed=True, out=Q,
                        stats=st, workspace=wsQ)
        if ev:
            ev[2].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    tp = tq = 0.0
    for _ in range(args.steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        step(ev)
        torch.cuda.synchronize()
        tp += ev[0].elapsed_time(ev[1])
        tq += ev[1].elapsed_time(ev[2])
    tp /= args.steps
    tq /= args.steps
    sd = g.stats_dict(st)
    return {"metric": "weight entries rounded per second, INT4 asymmetric g128 packed (1 B200)",
            "value": m * n / ((tp + tq) * 1e-3), "unit": "entries/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tp + tq,
            "higher_is_better": True, "dtype": "f64", "data": "synthetic (workloads.attn)",
            "config": {"workload": "grid128", "m": m, "n": n, "bits": 4, "group_size": 128,
                       "zero_points": True, "packed": True,
                       "step": "prepare_pair + quantize_grid, inputs resident in HBM"},
            "phases": {"prepare_pair_ms": tp, "quantize_ms": tq,
                       "quantize_fp64_tflops": m * n * (m + n) / (tq * 1e-3) / 1e12},
            "status": sd["status"], "n_near_tie": sd["n_near_tie"], "n_clamped": sd["n_clamped"]}


def run_gram(args):
    """The step before the path: the Kronecker factors from activations on the tensor
    cores (gram_accumulate + gram_finalize, bf16 activations, fp32 accumulation).  For
    each width k the activations are k rows of the workloads recipe (Student-t(4) times
    U(0.1, 10) column scales; the 70B block's recipe uses rows = width), generated on the
    GPU.  Algorithmic work: the lower block triangle, rows * k * (k + 128) flops (the
    128-wide diagonal blocks are computed whole).  Timed with CUDA events, best of K steps
    after W warm-ups, against MEASURED_PEAKS.json's bf16 burst figure; the fp64 matmul that
    forms the same Gram (torch, cuBLAS DGEMM) and cuBLAS's bf16 product X^T X (the whole
    square, twice the triangle's work) are timed beside it for context."""
    import torch
    import two_sided_adaptive_b200 as g
    from two_sided_adaptive_b200 import build as gbuild
    gbuild.build()
    dev = torch.device("cuda", 0)
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) \
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    peak = peaks.get("bf16_tflops", 1590.0)
    out = []
    for k in ((8192,) if args.profile_step else (4096, 8192, 28672)):
        torch.manual_seed(k)
        rows = k
        z = torch.randn(rows, k, device=dev, dtype=torch.float32)
        chi2 = torch.distributions.Chi2(torch.tensor(4.0, device=dev))
        X = (z / torch.sqrt(chi2.sample((rows, k)) / 4.0)) * \
            torch.empty(k, device=dev).uniform_(0.1, 10.0)[None, :]
        del z
        Xb = X.to(torch.bfloat16)
        del X
        H = torch.empty((k, k), dtype=torch.float32, device=dev)
        ws = torch.zeros(256, dtype=torch.uint8, device=dev)

        def step():
            g.gram_accumulate(Xb, H, accumulate=False, workspace=ws)
            g.gram_finalize(H, rows, 0.01, workspace=ws, check=False)

        if args.profile_step:  # one Gram of the 8192-wide case, nothing else (ncu input)
            step()
            torch.cuda.synchronize()
            return None
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        sampler = ClockSampler(bus_id_of(dev))
        sampler.start()
        time.sleep(0.3)
        best = 1e30
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        clocks = sampler.stop()
        best_acc = 1e30  # gram_accumulate alone
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.gram_accumulate(Xb, H, accumulate=False, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            best_acc = min(best_acc, e0.elapsed_time(e1))
        fl = float(rows) * k * (k + 128)
        Xd = Xb.double()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.matmul(Xd.T, Xd)
        torch.cuda.synchronize()
        e0.record()
        torch.matmul(Xd.T, Xd)
        e1.record()
        torch.cuda.synchronize()
        t64 = e0.elapsed_time(e1)
        del Xd
        # cuBLAS on the same bf16 operands (the whole square, fp32 accumulation), for
        # context: best of 5
        torch.matmul(Xb.T, Xb)
        t16 = 1e30
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(Xb.T, Xb)
            e1.record()
            torch.cuda.synchronize()
            t16 = min(t16, e0.elapsed_time(e1))
        del Xb, H
        torch.cuda.empty_cache()
        out.append({"k": k, "rows": rows, "ms": best, "tflops": fl / (best * 1e-3) / 1e12,
                    "frac_of_bf16_peak": fl / (best * 1e-3) / 1e12 / peak,
                    "clocks": clocks,
                    "accumulate_ms": best_acc,
                    "accumulate_tflops": fl / (best_acc * 1e-3) / 1e12,
                    "fp64_matmul_ms": t64,
                    "cublas_bf16_square_ms": t16,
                    "cublas_bf16_square_tflops": 2.0 * rows * k * k / (t16 * 1e-3) / 1e12})
    return {"metric": "Gram X^T X / N + damping from bf16 activations (tensor cores), TFLOP/s",
            "value": out[-1]["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16 operands, f32 accumulation",
            "data": "synthetic (generated on the GPU, see run_gram)",
            "peak": {"bf16_tflops": peak, "source": "MEASURED_PEAKS.json bf16_tflops (burst)"},
            "config": {"workload": "gram", "widths": [o["k"] for o in out]}, "sizes": out}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=80)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("attn", "mlp", "small", "block70b", "kron3", "grid128",
                                           "gram", "configs"),
                    default="attn",
                    help="block70b: seconds per layer for one 70B-class block; kron3: a "
                         "three-factor Kronecker Hessian; grid128: the attention layer on an "
                         "asymmetric 128-column-group packed INT4 grid; gram: the Kronecker "
                         "factors from activations on the tensor cores; configs: every "
                         "configuration with the CPU oracle beside it (reports, not the "
                         "headline metric)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=1024)
    ap.add_argument("--ref-sample", type=int, default=384)
    ap.add_argument("--profile-step", action="store_true",
                    help="run one step of the path only (input for ncu captures); prints nothing")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return

    import torch
    torch.cuda.set_device(local_rank)
    if args.workload == "block70b" and world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
        try:
            res = run_block70b(args, rank, world)
        finally:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    if args.workload in ("block70b", "kron3", "grid128", "gram", "configs"):
        if rank == 0:
            run = {"block70b": run_block70b, "kron3": run_kron3, "grid128": run_grid128,
                   "gram": run_gram, "configs": run_configs}[args.workload]
            res = run(args)
            if res is not None:
                print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
