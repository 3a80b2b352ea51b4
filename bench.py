#!/usr/bin/env python
"""Benchmark: K-interval attention forward + backward on B200.

Default workload: the GPT-2-124M attention shape B8 H12 T1024 d64, causal,
FWM (tau = 6, h = 1.5), Nearest reconstruction with Prob-STE, K = 4, full
calibration gradients -- synthetic inputs with per-head score spans of 8-40
nats.  One step = kiattn_fwd + kiattn_bwd over that batch.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0).  Throughput is algorithmic TFLOP/s: causal
GEMM units U = B*H*T^2*d; forward 3U (+1U for Prob-STE's P_L V), backward 5U.
With N GPUs (torchrun) every rank runs its own batch (weak scaling, no
collective on the data path); value = all ranks' flops / max-over-ranks time.
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# roofline denominators: MEASURED_PEAKS.json (bf16 dense burst) scaled by the
# nominal dense TF32 / BF16 ratio of B200 (1.1 / 2.25 PFLOP/s)
TF32_OVER_BF16 = 1.1 / 2.25
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gpt2_fwm",
                    choices=["gpt2_fwm", "gpt2_heavy", "gpt2_fixed", "gpt2_bf16exp",
                             "gpt2_fp8exp", "tiny"])
    ap.add_argument("--grad", default=None,
                    choices=["full", "detach", "max-only", "min-only", "projection"],
                    help="override the workload's gradient mode")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--diag", default=None, choices=["geometry", "decomposition"],
                    help="time one of the diagnostic row kernels instead of the step")
    ap.add_argument("--matrix", default=None, choices=["variants", "sweep", "one_b"],
                    help="one JSON line per operator variant (every calibration x "
                         "reconstruction x surrogate x gradient mode at the 124M shape), per "
                         "point of the B16 H12 T 1024-4096 throughput sweep, or per gradient "
                         "mode of the 1B-style shape from one shared forward (FWM and MinMax)")
    return ap.parse_args()


GRAD_NAMES = ("full", "detach", "max-only", "min-only", "projection")


def workload(name, grad=None):
    from quantized_softmax_attention_b200 import workloads as W
    if grad is not None:
        w = workload(name)
        return W.Workload(**{**w.__dict__, "grad": GRAD_NAMES.index(grad)})
    return {"gpt2_fwm": W.gpt2_fwm, "gpt2_heavy": W.gpt2_heavy, "gpt2_fixed": W.gpt2_fixed,
            "gpt2_bf16exp": lambda: W.gpt2_rounded_exp(False),
            "gpt2_fp8exp": lambda: W.gpt2_rounded_exp(True), "tiny": W.tiny}[name]()


def lib_config(w, K):
    """The library's operator configuration of workload w (TF32 products)."""
    return K.Config(K=w.K, cal=w.cal, tau=w.tau, rec=w.rec, ste=w.ste, grad=w.grad,
                    causal=w.causal, gemm=K.GEMM_TF32, op=w.operator)


def oracle_config(w, ref):
    """The oracle's configuration of workload w."""
    return ref.RefConfig(K=w.K, cal=w.cal, tau=w.tau, rec=w.rec, ste=w.ste, grad=w.grad,
                         causal=w.causal, softmax=w.operator != 0,
                         exp_round={2: ref.EXP_BF16, 3: ref.EXP_FP8}.get(w.operator, ref.EXP_EXACT))


def gemm_units(w):
    return w.B * w.H * w.T * w.T * w.d


def algorithmic_flops(w):
    """Forward 3U (+1U with Prob-STE) and backward 5U, U = B H T^2 d
    (2 flops per multiply-add over the causal half counts T^2 d per GEMM)."""
    if w.operator == 1:
        return 7 * gemm_units(w)   # exact softmax: one S in the forward (online rescaling)
    prob = w.operator == 0 and w.rec == 1 and w.ste == 1
    return (8 + (1 if prob else 0)) * gemm_units(w)


def config_dict(w, n):
    names = {0: "MinMax", 1: "FWM", 2: "fixed step (untruncated)"}
    if w.operator != 0:
        ops = {1: "softmax", 2: "softmax, bf16-rounded exp", 3: "softmax, FP8-rounded exp"}
        return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d,
                "operator": ops[w.operator], "causal": w.causal, "parallelism": f"dp{n}",
                "l2": "flushed between timed steps (256 MiB write)"}
    return {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "K": w.K,
            "calibration": names[w.cal], "tau": w.tau if w.cal != 0 else None,
            "reconstruction": "LERP" if w.rec == 0 else "Nearest",
            "surrogate": None if w.rec == 0 else ("Prob-STE" if w.ste else "Weight-STE"),
            "grad": GRAD_NAMES[w.grad], "causal": w.causal, "parallelism": f"dp{n}",
            "l2": "flushed between timed steps (256 MiB write)"}


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        return float(mp["bf16_tflops"]), float(mp["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_HBM_GBS, "fallback"


def measure_tf32_peak(n=8192, reps=10):
    """Dense TF32 tensor-core rate of this GPU, measured the way the bf16 peak
    is: torch.matmul of two fp32 n x n matrices with TF32 allowed (cuBLAS),
    best of `reps` CUDA-event timings.  Returns TFLOP/s."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        g = torch.Generator(device="cuda").manual_seed(0)
        a = torch.randn((n, n), device="cuda", generator=g)
        b = torch.randn((n, n), device="cuda", generator=g)
        c = torch.empty((n, n), device="cuda")
        for _ in range(3):
            torch.matmul(a, b, out=c)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b, out=c)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b, c
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def tf32_peak():
    """(TF32 TFLOP/s, source, nominal-ratio figure): the measured TF32 GEMM
    rate, with the bf16 peak of MEASURED_PEAKS.json times the nominal dense
    TF32/BF16 ratio kept beside it."""
    bf16, _, src = peaks()
    nominal = bf16 * TF32_OVER_BF16
    try:
        meas = measure_tf32_peak()
        return meas, ("measured tf32 (torch.matmul fp32 8192^3, allow_tf32, best of 10)",
                      nominal, f"{src} bf16 dense x {TF32_OVER_BF16:.4f} (nominal TF32/BF16)")
    except Exception as e:  # pragma: no cover - only without a usable GPU
        return nominal, (f"{src} bf16 dense x {TF32_OVER_BF16:.4f} (tf32 GEMM not measured: "
                         f"{type(e).__name__})", nominal, "")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, enabled: bool = True):
        self.index = index
        self.proc = None
        self.path = None
        if not enabled:
            return
        fd, self.path = tempfile.mkstemp(prefix="kia_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9 or parts[0] != str(self.index):
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- CPU side

def cpu_oracle_rate(w, target_s=10.0, max_reps=20):
    """fp64 CPU oracle (test infrastructure) on the full workload, repeated
    until ~target_s of work; returns (TFLOP/s, seconds, reps, cores)."""
    import oracle as ref
    from quantized_softmax_attention_b200 import workloads as W
    q, k, v, g = (x.numpy() for x in W.make_inputs(w))
    cfg = oracle_config(w, ref)
    t0 = time.perf_counter()
    reps = 0
    while True:
        ref.attention(q, k, v, g, cfg)
        reps += 1
        el = time.perf_counter() - t0
        if el >= target_s or reps >= max_reps:
            break
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return algorithmic_flops(w) * reps / el / 1e12, el, reps, cores


def reference_arm(args, budget_s=150.0):
    """The oracle timed as the reference implementation: each step is the
    fp64 CPU operator on the whole workload, the oracle running its
    (batch, head) pairs in parallel over the host cores.  The run stops
    early (and says so in `steps`) if the requested steps would take longer
    than about budget_s."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as ref
    from quantized_softmax_attention_b200 import workloads as W
    w = workload(args.workload, args.grad)
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    # the whole workload per step, as the cpu_baseline leg times it (about
    # 0.6 s per step on 16 cores at the 124M shape)
    nb = w.B
    q, k, v, g = (x.numpy() for x in W.make_inputs(w, B=nb))
    cfg = oracle_config(w, ref)
    flops = algorithmic_flops(w) * nb / w.B
    for _ in range(args.warmup):
        ref.attention(q, k, v, g, cfg)
    t0 = time.perf_counter()
    steps = 0
    while steps < args.steps:
        ref.attention(q, k, v, g, cfg)
        steps += 1
        if time.perf_counter() - t0 > budget_s:
            break
    el = time.perf_counter() - t0
    val = flops * steps / el / 1e12
    sample = (f"batches 0..{nb - 1} ({nb * w.H} (b, h) pairs of {w.B * w.H}) of {w.name} "
              f"per step (fp64, OpenMP over (b, h))")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
            "ms_per_step": el / steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, 1),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


METRIC = "K-interval attn fwd+bwd TFLOP/s at B8·H12·T1024·d64; % TF32 roofline"


# sources the three tcgen05 kernels are compiled from (their DRAM traffic
# record is valid while these are unchanged)
TC_SOURCES = ("kia_common.cuh", "kia_elem.cuh", "kia_fast.cuh", "kia_stats.cuh", "kia_tc.cuh",
              "kia_tc_bwd.cuh", "kia_tc_fwd.cuh")


def source_digest():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "quantized_softmax_attention_b200", "csrc")
    for f in TC_SOURCES:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get("kernels", {}).get(kernel)
    if not ent or rec.get("source_digest") != source_digest():
        return None
    return ent.get("bytes_per_launch_full_size")


# ---------------------------------------------------------- multi-rank host

def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank processes its own batch each step; the
    step time is the slowest rank's."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ GPU side

# ------------------------------------------------------ diagnostic kernels

def diag_main(args):
    """One JSON line for a diagnostic row kernel on the benchmark's workload:
    the geometry probe over the scores S = Q K^T, or the fixed-upstream
    decomposition over the backward's dS dump.  Both read each row's visible
    scores once: algorithmic bytes = 4 sum_i L_i + per-row side inputs and
    outputs; HBM-bound by design."""
    import torch
    from quantized_softmax_attention_b200 import kiattn as K
    from quantized_softmax_attention_b200 import workloads as W
    torch.cuda.set_device(0)
    w = workload(args.workload, args.grad)
    cfg = lib_config(w, K)
    host = W.make_inputs(w)
    q, k, v, g = (x.cuda() for x in host)
    B, H, T, d = w.B, w.H, w.T, w.d
    rows = B * H * T
    vis = B * H * (T * (T + 1) // 2 if w.causal else T * T)
    S = torch.empty((B, H, T, T), dtype=torch.float32, device="cuda")
    if args.diag == "geometry":
        K.kiattn_scores(q, k, S, cfg)
        out = torch.empty((B, H, T, K.GEO_FIELD_COUNT), dtype=torch.float32, device="cuda")
        nbytes = 4 * vis + rows * (4 * d + 4 * K.GEO_FIELD_COUNT)

        def run(src, dst, stream=None):
            K.kiattn_geometry(src, dst, cfg, Q=q, stream=stream)
        kname, metric = "geometry_kernel", "geometry probe GB/s (per-row span, width, norm, " \
            "entropies, TV, top-bucket mass) over the scores of B8·H12·T1024"
    else:
        bufs = K.Buffers(B, H, T, d, cfg)
        K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg)
        K.kiattn_bwd(q, k, v, bufs.O, g, bufs.stats, bufs.dQ, bufs.dK, bufs.dV, bufs.work, cfg,
                     dS_dbg=S)
        out = torch.empty((B, H, T, 3), dtype=torch.float64, device="cuda")
        nbytes = 4 * vis + rows * (8 + 24)

        def run(src, dst, stream=None):
            K.kiattn_grad_decomposition(src, bufs.work, dst, cfg, stream=stream)
        kname, metric = "grad_decomp_kernel", "fixed-upstream gradient decomposition GB/s " \
            "over the dS of B8·H12·T1024"
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush.zero_()
        run(S, out)
    torch.cuda.synchronize()
    sampler = ClockSampler(0, enabled=not args.no_clocks)
    time.sleep(0.3 if sampler.proc else 0.0)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        run(S, out)
        ends[i].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    err = K.kiattn_device_error(True)
    if err != 0:
        raise RuntimeError(f"device error word {err}")
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    gbs = nbytes / (ms * 1e-3) / 1e9
    _, hbm, src = peaks()

    # end to end: the step's scores (or dS) copied in from pinned host memory,
    # the kernel, the per-row record copied out
    e2e = None
    if not args.no_e2e:
        hS = S.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        nrep = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(nrep):
            S.copy_(hS, non_blocking=True)
            run(S, out)
            hout.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        te = e0.elapsed_time(e1) / nrep
        e2e = {"value": nbytes / (te * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": hS.numel() * 4,
               "d2h_bytes_per_step": hout.numel() * hout.element_size(), "ms_per_step": te}
    line = {"metric": metric, "value": gbs, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {**config_dict(w, 1), "diagnostic": args.diag,
                       "l2": "flushed between timed launches (256 MiB write)"},
            "roofline": {"bound": "hbm", "kernel": kname, "achieved": gbs, "peak": hbm,
                         "unit": "GB/s", "frac": gbs / hbm, "traffic": None,
                         "bytes_per_launch": nbytes, "peak_source": f"{src} HBM copy"},
            "gpu_launches": args.steps}
    if e2e:
        line["e2e"] = e2e
    if clocks:
        line["clocks"] = clocks
    if not args.no_cpu_baseline:
        import oracle as ref
        rcfg = oracle_config(w, ref)
        Sh = S.cpu().numpy()
        Qh = host[0].numpy()
        ln = np.arange(1, T + 1) if w.causal else np.full(T, T)
        t0, n = time.perf_counter(), 0
        while time.perf_counter() - t0 < 10.0 and n < B * H:
            b, h = divmod(n, H)
            if args.diag == "geometry":
                ref.geometry(Sh[b, h], ln, rcfg, Q=Qh[b, h])
            else:
                ref.grad_decomposition(host[0][b:b + 1, h:h + 1].numpy(),
                                       host[1][b:b + 1, h:h + 1].numpy(),
                                       host[2][b:b + 1, h:h + 1].numpy(),
                                       host[3][b:b + 1, h:h + 1].numpy(), rcfg)
            n += 1
        secs = time.perf_counter() - t0
        per_head = nbytes / (B * H)
        line["cpu_baseline"] = {"value": n * per_head / secs / 1e9, "unit": "GB/s",
                                "cores": int(os.environ.get("OMP_NUM_THREADS",
                                                            os.cpu_count() or 1)),
                                "kind": "oracle",
                                "sample": f"{n} of {B * H} (b, h) pairs ({secs:.1f} s, fp64)"}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------ variant matrices

def one_b_main(args):
    """The 1B-style configuration B4 H16 T2048 d128, LERP K = 32: for FWM and
    for MinMax one forward, timed on its own, then the five backward modes
    from that forward's stats, each timed on its own; one JSON line per
    (calibration, mode) with the step rate (forward + that backward, 8U)."""
    import torch
    from quantized_softmax_attention_b200 import kiattn as K
    from quantized_softmax_attention_b200 import workloads as W
    torch.cuda.set_device(0)
    peak, (src, _, _) = tf32_peak()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(args.warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        err = K.kiattn_device_error(True)
        if err != 0:
            raise RuntimeError(f"device error word {err}")
        return sum(a.elapsed_time(b) for a, b in ev) / args.steps

    for cal in (W.CAL_FWM, W.CAL_MINMAX):
        w = W.one_b(cal=cal)
        q, k, v, g = (x.cuda() for x in W.make_inputs(w))
        cfg = lib_config(w, K)
        bufs = K.Buffers(w.B, w.H, w.T, w.d, cfg)
        t_fwd = timed(lambda: K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg))
        K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg)
        U = gemm_units(w)
        for grad in range(5):
            c = cfg.replace(grad=grad)
            t_bwd = timed(lambda: K.kiattn_bwd(q, k, v, bufs.O, g, bufs.stats, bufs.dQ, bufs.dK,
                                               bufs.dV, bufs.work, c))
            tf = algorithmic_flops(w) / ((t_fwd + t_bwd) * 1e-3) / 1e12
            cd = {**config_dict(W.Workload(**{**w.__dict__, "grad": grad}), 1),
                  "forward": "one forward shared by the five modes"}
            print(json.dumps({"matrix": "one_b", "config": cd, "value": tf, "unit": "TFLOP/s",
                              "ms_fwd": t_fwd, "ms_bwd": t_bwd, "ms_per_step": t_fwd + t_bwd,
                              "fwd_tflops": 3 * U / (t_fwd * 1e-3) / 1e12,
                              "bwd_tflops": 5 * U / (t_bwd * 1e-3) / 1e12,
                              "frac_of_tf32_roofline": tf / peak, "peak": peak,
                              "peak_source": src, "steps": args.steps, "warmup": args.warmup}),
                  flush=True)
        del bufs, q, k, v, g


def matrix_main(args):
    """Fwd+bwd throughput over a matrix of operator variants: `variants` runs
    the 124M span-ladder inputs under every calibration x reconstruction x
    surrogate x gradient mode; `sweep` runs the B16 H12 d64 throughput sweep
    (T in 1024..4096, K in 2..64, both calibrations, three reconstructions,
    plus exact softmax per T).  Same timing rules as the step: warm-up, L2
    flushed between timed steps, CUDA events on the launching stream."""
    import torch
    from quantized_softmax_attention_b200 import kiattn as K
    from quantized_softmax_attention_b200 import workloads as W
    torch.cuda.set_device(0)
    peak, (src, _, _) = tf32_peak()
    recs = [(W.REC_LERP, W.STE_WEIGHT), (W.REC_NEAREST, W.STE_WEIGHT),
            (W.REC_NEAREST, W.STE_PROB)]
    runs = []
    if args.matrix == "variants":
        base = W.gpt2_fwm()
        for cal in (W.CAL_MINMAX, W.CAL_FWM, W.CAL_FIXED):
            for rec, ste in recs:
                for grad in range(5):
                    runs.append(W.Workload(**{**base.__dict__, "cal": cal, "rec": rec, "ste": ste,
                                              "grad": grad, "name": base.name}))
    else:
        for T in (1024, 2048, 4096):
            for Kint in (2, 4, 16, 32, 64):
                for cal in (W.CAL_MINMAX, W.CAL_FWM):
                    for rec, ste in recs:
                        runs.append(W.sweep(T, Kint, cal, rec, ste))
            runs.append(W.Workload(**{**W.sweep(T, 4, W.CAL_MINMAX, W.REC_LERP,
                                                W.STE_WEIGHT).__dict__, "operator": 1}))
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    inputs = {}
    for w in runs:
        key = (w.B, w.H, w.T, w.d, w.seed, w.scores)
        if key not in inputs:
            inputs.clear()
            inputs[key] = [x.cuda() for x in W.make_inputs(w)]
        q, k, v, g = inputs[key]
        cfg = lib_config(w, K)
        bufs = K.Buffers(w.B, w.H, w.T, w.d, cfg)

        def step():
            K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg)
            K.kiattn_bwd(q, k, v, bufs.O, g, bufs.stats, bufs.dQ, bufs.dK, bufs.dV, bufs.work, cfg)

        for _ in range(args.warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        err = K.kiattn_device_error(True)
        if err != 0:
            raise RuntimeError(f"device error word {err}")
        ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
        tf = algorithmic_flops(w) / (ms * 1e-3) / 1e12
        cd = config_dict(w, 1)
        print(json.dumps({"matrix": args.matrix, "config": cd, "value": tf, "unit": "TFLOP/s",
                          "ms_per_step": ms, "frac_of_tf32_roofline": tf / peak,
                          "peak": peak, "peak_source": src,
                          "steps": args.steps, "warmup": args.warmup}), flush=True)
        del bufs


def main():
    args = parse()
    if args.impl == "reference":
        reference_arm(args)
        return
    if args.diag:
        diag_main(args)
        return
    if args.matrix == "one_b":
        one_b_main(args)
        return
    if args.matrix:
        matrix_main(args)
        return
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from quantized_softmax_attention_b200 import kiattn as K
    from quantized_softmax_attention_b200 import workloads as W

    w = workload(args.workload, args.grad)
    cfg = lib_config(w, K)
    w_rank = W.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})
    host = [x.pin_memory() for x in W.make_inputs(w_rank)]
    dev = [x.cuda() for x in host]
    q, k, v, g = dev
    bufs = K.Buffers(w.B, w.H, w.T, w.d, cfg)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        K.kiattn_fwd(q, k, v, bufs.O, bufs.stats, cfg)
        K.kiattn_bwd(q, k, v, bufs.O, g, bufs.stats, bufs.dQ, bufs.dK, bufs.dV, bufs.work, cfg)

    # our kernels per step: the forward, then the tensor-core backward's query
    # and key passes, plus the projection's scan
    launches_per_step = 3 + (1 if w.grad == K.GRAD_PROJECT else 0)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    err = K.kiattn_device_error(True)
    if err != 0:
        raise RuntimeError(f"device error word {err}")

    # timed region: steps queued back to back (no host synchronisation inside),
    # an L2 flush between steps outside each step's pair of events
    sampler = ClockSampler(local, enabled=not args.no_clocks)
    time.sleep(0.3 if sampler.proc else 0.0)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms_step = max_over_ranks(total_ms, device="cuda") / args.steps
    err = K.kiattn_device_error(True)
    if err != 0:
        raise RuntimeError(f"device error word {err}")

    # per-kernel times from the library's own events, on separate steps
    K.kiattn_profile_enable(True)
    phase_tot = {}
    n_prof = max(3, min(args.steps, 20))
    for _ in range(n_prof):
        flush.zero_()
        step()
        for kk, vv in K.kiattn_profile_read().items():   # synchronises on this step
            phase_tot[kk] = phase_tot.get(kk, 0.0) + vv
    K.kiattn_profile_enable(False)
    flops = algorithmic_flops(w)
    value = weak_scaling_value(flops, world, ms_step)

    # end to end through the public API from pinned host memory: every step
    # copies its inputs in, runs forward and backward, and copies O, dQ, dK,
    # dV out, as a pipeline over two buffer sets on three streams (copy in,
    # compute, copy out), so that the copies of one step overlap the compute
    # of its neighbours
    e2e = None
    if not args.no_e2e:
        nrep = max(4, min(args.steps, 50))
        devs = [[torch.empty_like(x) for x in dev] for _ in range(2)]
        bset = [K.Buffers(w.B, w.H, w.T, w.d, cfg) for _ in range(2)]
        hout = [[torch.empty(bufs.O.shape, dtype=torch.float32).pin_memory() for _ in range(4)]
                for _ in range(2)]
        s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_c = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def pipelined(n):
            for i in range(n):
                b = i % 2
                d, bb = devs[b], bset[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_c[b])       # step i-2 no longer reads set b
                    for hd, dd in zip(host, d):
                        dd.copy_(hd, non_blocking=True)
                    ev_in[b].record(s_in)
                s_c.wait_event(ev_in[b])
                if i >= 2:
                    s_c.wait_event(ev_out[b])          # step i-2's outputs copied out
                K.kiattn_fwd(d[0], d[1], d[2], bb.O, bb.stats, cfg, stream=s_c)
                K.kiattn_bwd(d[0], d[1], d[2], bb.O, d[3], bb.stats, bb.dQ, bb.dK, bb.dV, bb.work,
                             cfg, stream=s_c)
                ev_c[b].record(s_c)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_c[b])
                    for ho, dd in zip(hout[b], (bb.O, bb.dQ, bb.dK, bb.dV)):
                        ho.copy_(dd, non_blocking=True)
                    ev_out[b].record(s_out)

        pipelined(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_c.wait_event(e0)
        s_out.wait_event(e0)
        pipelined(nrep)
        s_in.wait_stream(s_c)
        s_in.wait_stream(s_out)
        e1.record(s_in)
        torch.cuda.synchronize()
        err = K.kiattn_device_error(True)
        if err != 0:
            raise RuntimeError(f"device error word {err}")
        te = max_over_ranks(e0.elapsed_time(e1) / nrep, device="cuda")
        nbytes = sum(x.numel() * 4 for x in host)
        e2e = {"value": weak_scaling_value(flops, world, te), "unit": "TFLOP/s",
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": 4 * bufs.O.numel() * 4,
               "ms_per_step": te, "pipeline": "copy-in / compute / copy-out streams, 2 buffer sets"}

    # roofline of the dominant kernel (tensor-core bound: TF32 contraction)
    U = gemm_units(w)
    prob = w.rec == 1 and w.ste == 1
    kernel_flops = {"fwd": (3 + (1 if prob else 0)) * U, "bwd_query_pass": 3 * U,
                    "bwd_key_pass": 4 * U}
    kernel_names = {"fwd": "tc_fwd_kernel", "bwd_query_pass": "tc_bwd_q_kernel",
                    "bwd_key_pass": "tc_bwd_kv_kernel"}
    dom = max(kernel_flops, key=lambda kk: phase_tot.get(kk, 0.0))
    dom_ms = phase_tot[dom] / n_prof
    peak, (src, nominal, nominal_src) = tf32_peak()
    achieved = kernel_flops[dom] / (dom_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "kernel": kernel_names[dom], "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "traffic": ncu_traffic(kernel_names[dom]),
            "peak_source": src, "peak_nominal_ratio": nominal, "peak_nominal_source": nominal_src,
            "flops_per_launch": kernel_flops[dom],
            "phase_ms": {kk: vv / n_prof for kk, vv in phase_tot.items()}}

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "tf32",
            "data": "synthetic", "config": config_dict(w, world), "roofline": roof,
            "frac_of_tf32_roofline": value / world / peak,
            "softmax_equivalent": {"value": value * 7.0 / (flops / gemm_units(w)),
                                   "unit": "TFLOP/s", "flops_per_step": "7U (exact softmax)"},
            "gpu_launches": launches_per_step * args.steps}
    if e2e:
        line["e2e"] = e2e
    if clocks:
        line["clocks"] = clocks
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, secs, reps, cores = cpu_oracle_rate(w)
        line["cpu_baseline"] = {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"full {w.name} batch x{reps} ({secs:.1f} s, fp64)"}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
