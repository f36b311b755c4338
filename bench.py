#!/usr/bin/env python
"""Throughput of incoherence-processed LDLQ for one linear layer on B200.

One step = the whole hot path for one layer on device-resident inputs:
draw (U, V) -> H = X^T X (tensor cores) -> finalise + damp -> W~ = U W V^T,
H~ = V H V^T -> LDL of H~ -> LDLQ rounding -> dequantise -> inverse transform.
Metric: quantized weights per second (m * n / step time), whole job.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config gate70b] [--all-configs]
  python bench.py --impl reference ...    # the FP64 CPU oracle, bounded sample

Multi-GPU (torchrun): each rank quantises its own layer of the same shape
(seed + rank), no data-path collective (weak scaling); the step time is the
max over ranks.  L2 is flushed (256 MB write) before every timed step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quip_synth import CONFIGS, LayerConfig, make_layer  # noqa: E402

METRIC = "quantized weights/s per layer (Hessian+incoherence+LDLQ)"
UNIT = "weights/s"
STAGES = ["transform", "hessian", "finalize", "incoherence_fwd", "ldl", "ldlq", "dequant",
          "incoherence_inv"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# bf16 tensor-core products per fp32-accurate multiply-add in the split GEMMs
# (three bf16 pieces per operand, the six piece products of order <= 2).
SPLIT_PRODUCTS = 6

# FP32 FFMA peak from unit counts and clock: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz.
FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def stage_work(cfg: LayerConfig):
    """Algorithmic work per stage: (kind, amount, bound, engine-note)."""
    m, n, N, b = cfg.m, cfg.n, cfg.N, cfg.block
    xb = 2 if cfg.dtype == "bf16" else 4
    return {
        "transform": ("bytes", 4.0 * (m + n), "hbm"),
        "hessian": ("flops", float(N) * n * (n + 1), "tensor" if cfg.dtype == "bf16" else "alu"),
        "finalize": ("bytes", 8.0 * n * n, "hbm"),
        # W read + W~ write, H read + H~ write (minimum traffic of the transform)
        "incoherence_fwd": ("bytes", (xb + 4.0) * m * n + 8.0 * n * n, "hbm"),
        "ldl": ("flops", n ** 3 / 3.0, "alu"),
        # trailing GEMMs m n (n - b) plus in-block feedback m n b
        "ldlq": ("flops", float(m) * n * n, "alu"),
        "dequant": ("bytes", 5.0 * m * n + 8.0 * m, "hbm"),
        "incoherence_inv": ("bytes", 8.0 * m * n, "hbm"),
    }


def _ldlq_gemm_flops(m: int, n: int, b: int) -> float:
    """Algorithmic flops of LDLQ's trailing GEMMs: the recursive split of the
    columns into halves, 2 m (right width) (left width) per split."""
    def rec(a, c):
        nb = (c - a) // b
        if nb <= 1:
            return 0.0
        mid = a + ((nb + 1) // 2) * b
        return rec(a, mid) + 2.0 * m * (c - mid) * (mid - a) + rec(mid, c)
    return rec(0, n)


def _ldlq_block_flops(m: int, n: int, b: int = 128) -> float:
    """In-block feedback of LDLQ: each b-column block feeds every column's
    error to the block's later columns, m w (w - 1) flops for a w-wide block."""
    return float(sum(m * min(b, n - k0) * (min(b, n - k0) - 1) for k0 in range(0, n, b)))


def kernel_work(cfg: LayerConfig, method: str = "ldlq", passes: int = 1):
    """Algorithmic work per step of the library's kernels, by kernel name:
    (kind, amount, bound).  Flops count multiply-adds as 2; bytes are the
    minimum reads + writes of the kernel's operands.  The tensor-core split
    GEMMs are counted at their fp32 algorithmic flops (2 M N K) although they
    run six bf16 products per multiply-add (the three-piece split).
    ``method`` / ``passes``: the rounding method (LDLQ by default); a greedy
    pass is one full GEMM (E H) plus LDLQ's recursion (block kernel and
    trailing GEMMs)."""
    m, n, N = cfg.m, cfg.n, cfg.N
    greedy = passes if method in ("greedy", "ldlq_rg") else 0
    ldlq_runs = (1 if method in ("ldlq", "ldlq_rg") else 0) + greedy
    has_ldl = method in ("ldlq", "ldlq_rg")
    xb = 2 if cfg.dtype == "bf16" else 4
    PB = 128
    P = (n + PB - 1) // PB
    fac = rows = bulk = 0.0
    for p in range(P - 1, -1, -1):
        c0 = p * PB
        w = min(PB, n - c0)
        fac += w ** 3 / 3.0 + (128.0 * w * w if c0 > 0 else 0.0)
        if c0 > 0:
            rows += c0 * (w * w + 2.0 * w * 128)
        if c0 > PB:
            M = c0 - PB
            bulk += M * (M + 1) * PB            # upper triangle, 2 flops per multiply-add
    kw = {
        "k_syrk_tc": ("flops", float(N) * n * (n + 1), "tensor"),
        "k_row_grid": ("bytes", 4.0 * m * n + 8.0 * m, "hbm"),
        "k_dequant": ("bytes", 5.0 * m * n + 8.0 * m, "hbm"),
        "k_mirror_scale": ("bytes", 8.0 * n * n, "hbm"),
    }
    if has_ldl:
        kw.update({
            "k_ldl_factor": ("flops", fac, "alu"),
            "k_ldl_rows": ("flops", rows, "alu"),
            "k_gemm_split_tc[ldl]": ("flops", bulk, "tensor"),
            "k_split_upper_transposed": ("bytes", 4.0 * n * n / 2 + 10.0 * n * n, "hbm"),
        })
    if ldlq_runs:
        kw["k_gemm_split_tc[ldlq]"] = ("flops", ldlq_runs * _ldlq_gemm_flops(m, n, 128), "tensor")
        kw["k_ldlq_block"] = ("flops", ldlq_runs * _ldlq_block_flops(m, n), "alu")
    if method in ("nearest", "greedy"):
        kw["k_nearest"] = ("bytes", 5.0 * m * n + 8.0 * m, "hbm")
    if greedy:
        kw["k_gemm_split_tc[greedy]"] = ("flops", greedy * 2.0 * m * n * n, "tensor")
        # codes + W in; W^, the accumulator and three bf16 error pieces out
        kw["k_greedy_start"] = ("bytes", greedy * 19.0 * m * n, "hbm")
        # H's upper triangle in; U'^T (fp32 and three pieces) and U' out
        kw["k_greedy_factors"] = ("bytes", 16.0 * n * n, "hbm")
    if cfg.m_side.kind == "kronecker":
        # the m-side Kronecker factors on the tensor cores, forward and inverse:
        # 2 (p + q) m n fp32-algorithmic flops each way (issued as 3 or 6
        # bf16 piece products)
        p_, q_ = cfg.m_side.p, cfg.m_side.q
        kw["k_kron_tc"] = ("flops", 2 * 2.0 * (p_ + q_) * m * n, "tensor")
    if method == "ldlq_rg":
        # H~ gathered twice (8 n^2 each), W~ once (8 m n), the codes back (2 m n)
        kw["k_permute"] = ("bytes", 16.0 * n * n + 10.0 * m * n, "hbm")
    # Hadamard passes: rows read their input (W once as bf16/f32, H and W^
    # in fp32) and write fp32; column passes read and write fp32.
    had = lambda s: s.kind == "hadamard"
    fr = fc = 0.0
    if had(cfg.n_side):
        fr += (xb + 4.0) * m * n + 8.0 * n * n + 8.0 * m * n    # W, H (fwd), W^ (inv)
        fc += 8.0 * n * n                                       # H columns (fwd)
    if had(cfg.m_side):
        fc += 2 * 8.0 * m * n                                   # W~ (fwd), W^ (inv)
    if fr:
        kw["k_fwht_rows"] = ("bytes", fr, "hbm")
    if fc:
        kw["k_fwht_cols"] = ("bytes", fc, "hbm")
    return kw


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
# the gate70b layer, with the first 12 hex digits of the SHA-1 of the source
# file the kernel was built from: a figure is reported only while that file
# is unchanged and only for that workload.  The counters were taken on the
# layer's first 7168 of 28672 rows and 8192 of 32768 tokens (one capture
# stays a few GB): the LDL depends on n alone, so its split GEMMs' average is
# the full layer's; the LDLQ GEMMs' A operand and accumulator and the
# row-wise kernels' bytes grow with the rows, so their figures are the
# slice's times 28672 / 7168 = 4.  Writes still in L2 when a kernel ends are
# not counted (the LDLQ block kernel's codes and error pieces).  The
# dequantisation and row-grid figures were taken on a build of ldlq.cuh that
# differs from this one only in the block kernel.
KERNEL_TRAFFIC = {
    "k_gemm_split_tc[ldlq]": ("gemm_tc.cuh", "07f39ed17af3", 172632584),
    "k_gemm_split_tc[ldl]": ("gemm_tc.cuh", "07f39ed17af3", 61238127),
    "k_ldlq_block": ("ldlq.cuh", "294f51797099", 45038592),
    "k_dequant": ("ldlq.cuh", "294f51797099", 941438976),
    "k_row_grid": ("ldlq.cuh", "294f51797099", 970614784),
}
TRAFFIC_WORKLOAD = "gate70b"


def kernel_traffic(name: str, workload: str):
    import hashlib
    ent = KERNEL_TRAFFIC.get(name)
    if ent is None or workload != TRAFFIC_WORKLOAD:
        return None
    src = os.path.join(ROOT, "post_weight_quantization_09_b200", "csrc", ent[0])
    try:
        h = hashlib.sha1(open(src, "rb").read()).hexdigest()[:12]
    except OSError:
        return None
    return ent[2] if h == ent[1] else None


def roofline_entry(kind, amount, bound, ms, pk, split=False):
    """achieved / peak for one kernel or stage.  split: the flops are fp32
    multiply-adds carried out as six bf16 tensor-core products each (the
    three-piece split), so the peak is the measured bf16 peak / 6."""
    note = None
    if kind == "bytes":
        achieved = amount / (ms * 1e-3) / 1e9
        peak, unit = pk["hbm_gbs"], "GB/s"
    else:
        achieved = amount / (ms * 1e-3) / 1e12
        if bound == "tensor" and split:
            peak, unit = pk["bf16_tflops"] / SPLIT_PRODUCTS, "TFLOP/s"
            note = f"fp32-accurate flops; peak = measured bf16 peak / {SPLIT_PRODUCTS} (bf16 piece products per multiply-add)"
        elif bound == "tensor":
            peak, unit = pk["bf16_tflops"], "TFLOP/s"
        else:
            peak, unit = FFMA_TFLOPS, "TFLOP/s"
    out = {"bound": bound, "achieved": round(achieved, 3), "peak": round(peak, 1), "unit": unit,
           "frac": round(achieved / peak, 4), "traffic": None}
    if note:
        out["peak_note"] = note
    return out


def is_split(name: str) -> bool:
    """Kernels whose tensor-core flops are fp32 multiply-adds as bf16 piece products."""
    return name.startswith("k_gemm_split_tc") or name == "k_kron_tc"


# Stages whose flops the library runs on the tensor cores as split-bf16
# products have their fp32-algorithmic floor at the bf16 peak / 6; the rest
# of their work (the LDL's diagonal chain, LDLQ's in-block rounding) runs on
# the FP32 pipes.


def pipeline_floor(cfg: LayerConfig, pk) -> dict:
    """Speed-of-light time per stage: its work over the engine it runs on:
    the bf16 Hessian at the bf16 tensor peak (an fp32 one at the FP32 FFMA
    peak), the LDL and LDLQ flops at the fp32-accurate split-bf16 rate (bf16
    peak / 6), every byte-counted stage at the measured HBM bandwidth.
    Returns {stage: floor ms}."""
    floors = {}
    for name, (kind, amount, bound) in stage_work(cfg).items():
        if kind == "bytes":
            floors[name] = amount / (pk["hbm_gbs"] * 1e9) * 1e3
        elif bound == "tensor":
            floors[name] = amount / (pk["bf16_tflops"] * 1e12) * 1e3
        elif name in ("ldl", "ldlq"):
            floors[name] = amount / (pk["bf16_tflops"] / SPLIT_PRODUCTS * 1e12) * 1e3
        else:                                           # fp32 inputs: FP32 pipes
            floors[name] = amount / (FFMA_TFLOPS * 1e12) * 1e3
    return floors


def pipeline_entry(cfg: LayerConfig, pk, ms_per_step: float) -> dict:
    """The pipeline fraction: the sum of the stages' floors / the measured step."""
    floors = pipeline_floor(cfg, pk)
    total = sum(floors.values())
    return {"floor_ms": round(total, 4), "frac": round(total / ms_per_step, 4),
            "stage_floor_ms": {k: round(v, 4) for k, v in floors.items()},
            "denominators": f"HBM {pk['hbm_gbs']} GB/s; bf16 {pk['bf16_tflops']} TFLOP/s for the Hessian; "
                            f"bf16 / {SPLIT_PRODUCTS} for the LDL and LDLQ flops (split-bf16 fp32-accurate "
                            f"products); {pk['source']} peaks"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle timing


class OracleSample:
    """The FP64 oracle's own stage functions on a bounded sample of one layer,
    each stage timed on its own and extrapolated to the whole layer.

    Row-separable stages (the forward and inverse transforms of W's rows,
    grid and LDLQ, dequantisation) run on sampled rows, the Hessian on the
    first tokens, the Hessian's transform on sampled rows of H~, each at two
    sample sizes s1 < s2; a stage's whole-layer time is the straight line
    through the two timings at the full size (a fixed part, e.g. building a
    transform matrix or the per-column loop of LDLQ, plus a part per row),
    t(S) = t1 + (t2 - t1) (S - s1) / (s2 - s1), neither part below zero.
    The transforms' draw, the damping and the LDL run at full size.  Stages
    whose input would need a previous full-size stage take a stand-in of the
    same shape (the LDL factors the damped token-sample Hessian, LDLQ uses
    that factor; the inverse transform reads W in place of the dequantised
    W~), which changes no stage's work.  ``items`` lists (stage, size index);
    ``run(item)`` times one stage once at one size and returns seconds."""

    ROWS = (64, 256)
    TOKENS = (512, 2048)
    HROWS = (128, 512)

    def __init__(self, cfg: LayerConfig, d):
        import oracle as O
        self.O, self.cfg = O, cfg
        m, n, N = cfg.m, cfg.n, cfg.N
        rng = np.random.default_rng(7)
        self.rows = np.sort(rng.choice(m, min(self.ROWS[1], m), replace=False))
        self.hrows = np.sort(rng.choice(n, min(self.HROWS[1], n), replace=False))
        self.X = d["X"][:min(self.TOKENS[1], N)]
        self.W = d["W"]
        # untimed set-up: the inputs each timed stage reads
        self.U = O.make_side(cfg.seed, "m", cfg.m_side.kind, m, cfg.m_side.p, cfg.m_side.q)
        self.V = O.make_side(cfg.seed, "n", cfg.n_side.kind, n, cfg.n_side.p, cfg.n_side.q)
        self.H = O.damp(O.hessian(self.X), cfg.damp)
        self.Uf, _ = O.udu(self.H)
        self.Wt = O.incoherence_rows(self.W, self.U, self.V, self.rows)
        self.lo, self.s = O.row_grid(self.Wt, cfg.bits)
        self.codes, _, _ = O.ldlq(self.Wt, self.Uf, self.lo, self.s, cfg.bits)
        # stage -> (sample sizes, full size); None: full size only
        self.scale = {"transform": None, "hessian": (self.TOKENS, N), "finalize": None,
                      "incoherence_fwd_h": (self.HROWS, n), "incoherence_fwd_w": (self.ROWS, m),
                      "ldl": None, "ldlq": (self.ROWS, m), "dequant": (self.ROWS, m),
                      "incoherence_inv": (self.ROWS, m)}
        self.items = []
        for nm, sc in self.scale.items():
            self.items += [(nm, 0)] if sc is None else [(nm, 0), (nm, 1)]

    def size(self, name: str, k: int) -> int:
        sc = self.scale[name]
        return 0 if sc is None else min(sc[0][k], sc[1])

    def run(self, item) -> float:
        O, cfg = self.O, self.cfg
        name, k = item
        sz = self.size(name, k)
        t0 = time.perf_counter()
        if name == "transform":
            O.make_side(cfg.seed, "m", cfg.m_side.kind, cfg.m, cfg.m_side.p, cfg.m_side.q)
            O.make_side(cfg.seed, "n", cfg.n_side.kind, cfg.n, cfg.n_side.p, cfg.n_side.q)
        elif name == "hessian":
            O.hessian(self.X[:sz])
        elif name == "finalize":
            O.damp(self.H, cfg.damp)
        elif name == "incoherence_fwd_h":
            O.incoherence_hessian_rows(self.H, self.V, self.hrows[:sz])
        elif name == "incoherence_fwd_w":
            O.incoherence_rows(self.W, self.U, self.V, self.rows[:sz])
        elif name == "ldl":
            O.udu(self.H)
        elif name == "ldlq":
            lo, s = O.row_grid(self.Wt[:sz], cfg.bits)
            O.ldlq(self.Wt[:sz], self.Uf, lo, s, cfg.bits)
        elif name == "dequant":
            O.dequantize(self.codes[:sz], self.lo[:sz], self.s[:sz])
        elif name == "incoherence_inv":
            O.incoherence_inverse_rows(self.W, self.U, self.V, self.rows[:sz])
        else:
            raise KeyError(name)
        return time.perf_counter() - t0

    def stage_seconds(self, times) -> dict:
        """Whole-layer seconds per stage from {item: [seconds, ...]} (means)."""
        out = {}
        for nm, sc in self.scale.items():
            t1 = statistics.mean(times[(nm, 0)])
            if sc is None:
                out[nm] = t1
                continue
            t2 = statistics.mean(times[(nm, 1)])
            s1, s2, full = self.size(nm, 0), self.size(nm, 1), sc[1]
            if s2 <= s1:
                out[nm] = t1 * full / max(s1, 1)
                continue
            per = max(0.0, (t2 - t1) / (s2 - s1))
            fixed = max(0.0, t1 - per * s1)
            out[nm] = fixed + per * full
        return out

    def estimate(self, times) -> float:
        return sum(self.stage_seconds(times).values())

    def describe(self) -> str:
        c = self.cfg
        r, t, h = (self.size("ldlq", 0), self.size("ldlq", 1)), self.TOKENS, self.HROWS
        return (f"FP64 oracle stage functions on {c.name}: Hessian on {t[0]} and {t[1]} of {c.N} tokens, H~ on "
                f"{h[0]} and {h[1]} of {c.n} rows, W~, grid, LDLQ, dequantisation and inverse transform on "
                f"{r[0]} and {r[1]} of {c.m} rows, each extrapolated to the whole layer along the line through "
                f"its two timings (fixed + per-row part); transform draw, damping and LDL at full size")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return sum(i.get("num_threads", 0) for i in info if i.get("user_api") == "blas") or os.cpu_count()
    except Exception:
        return os.cpu_count()


# ----------------------------------------------------------------------------- arms


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_config(cfg: LayerConfig, rank: int) -> LayerConfig:
    """Each rank quantises its own layer of the same shape (seed + rank)."""
    return LayerConfig(**{**cfg.__dict__, "seed": cfg.seed + rank})


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over the ranks (the job's step time); no-op at N = 1."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(cfg: LayerConfig, world: int, ms_per_step: float) -> float:
    """Whole-job quantized weights per second: every rank's layer over the
    slowest rank's step time (weak scaling)."""
    return world * cfg.m * cfg.n / (ms_per_step * 1e-3)


def stage_schedule(names, steps: int):
    """Stages of each of `steps` steps: one stage per step in rotation when
    there are at least as many steps as stages, else every stage once, split
    over the steps."""
    S = len(names)
    if steps >= S:
        return [[names[i % S]] for i in range(steps)]
    return [[names[j] for j in range(S) if j % steps == i] for i in range(steps)]


def cpu_baseline_entry(cfg: LayerConfig, d) -> dict:
    """The oracle on its bounded sample: one untimed call to start the BLAS
    threads, then every (stage, size) item twice, the faster timing kept (a
    single short timing is noisy); the whole-layer estimate from those."""
    smp = OracleSample(cfg, d)
    smp.run(("hessian", 0))
    times = {it: [min(smp.run(it), smp.run(it))] for it in smp.items}
    sec = smp.estimate(times)
    return {"value": cfg.m * cfg.n / sec, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": smp.describe() + f"; whole layer estimated at {sec:.1f} s",
            "stage_seconds": {nm: round(v, 4) for nm, v in smp.stage_seconds(times).items()}}


def run_reference(args, cfg: LayerConfig):
    """The FP64 oracle (this problem's reference: the pages ship no code) on
    the host cores.  Each step times a bounded part of the oracle's sample of
    the layer ((stage, size) items in rotation, see OracleSample); value is
    the layer's weights over the whole-layer time those timings give."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    d = make_layer(cfg)
    smp = OracleSample(cfg, d)
    items = smp.items
    for step in stage_schedule(items, max(args.warmup, 1)):
        for it in step:
            smp.run(it)
    times = {it: [] for it in items}
    step_s = []
    for step in stage_schedule(items, args.steps):
        t0 = time.perf_counter()
        for it in step:
            times[it].append(smp.run(it))
        step_s.append(time.perf_counter() - t0)
    sec = smp.estimate(times)
    value = cfg.m * cfg.n / sec
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(step_s) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_desc(cfg, args),
        "layer_seconds_estimated": sec,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": smp.describe() + f"; the {len(items)} (stage, size) timings in rotation, "
                                   f"one or more per step; ms_per_step is the measured wall time of one step, "
                                   f"value the layer's weights over the {sec:.1f} s whole-layer estimate"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_desc(cfg: LayerConfig, args):
    side = lambda s: (s.kind if s.kind != "kronecker" else f"kronecker {s.p}x{s.q}") + \
        (" with random permutation" if getattr(s, "permute", False) else "")
    method = getattr(args, "method", "ldlq")
    passes = getattr(args, "passes", 1)
    rounding = {"ldlq": f"LDLQ block {cfg.block}", "nearest": "nearest rounding",
                "greedy": f"Greedy ({passes} passes)",
                "ldlq_rg": f"LDLQ-RG (block {cfg.block}, {passes} greedy passes)"}[method]
    return {
        "workload": f"{cfg.name}: W {cfg.m}x{cfg.n} {cfg.dtype}, X {cfg.N}x{cfg.n} {cfg.dtype}, "
                    f"U {side(cfg.m_side)}, V {side(cfg.n_side)}, {rounding}, {cfg.bits}-bit",
        "m": cfg.m, "n": cfg.n, "tokens": cfg.N, "bits": cfg.bits, "block": cfg.block,
        "damp": cfg.damp, "l2": "flushed before every timed step (256 MB write)",
        "parallelism": f"replicas x{args.gpus} (one layer per GPU)",
    }


def run_ours(args, cfg: LayerConfig):
    import torch
    import torch.distributed as dist
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    import post_weight_quantization_09_b200 as Q
    from post_weight_quantization_09_b200 import _lib as L
    lib = Q.load()
    rcfg = rank_config(cfg, rank)
    d = make_layer(rcfg)
    as_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
        else torch.from_numpy(a)
    W_h = as_t(d["W_bf16"] if cfg.dtype == "bf16" else d["W"]).pin_memory()
    X_h = as_t(d["X_bf16"] if cfg.dtype == "bf16" else d["X"]).pin_memory()
    W = W_h.cuda()
    X = X_h.cuda()
    q = Q.LayerQuantizer(cfg.m, cfg.n, cfg.m_side, cfg.n_side, cfg.bits, cfg.block, cfg.damp,
                         rcfg.seed, method=args.method, passes=args.passes)
    stream = torch.cuda.current_stream()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")   # 256 MB > L2

    def step(ev=None):
        mark = (lambda i: ev[i].record(stream)) if ev else (lambda i: None)
        mark(0)
        q.new_transform()
        mark(1)
        Q.quip_hessian_accumulate(X, q.H, False)
        mark(2)
        Q.quip_hessian_finalize(q.H, cfg.N, cfg.damp)
        mark(3)
        Q.quip_incoherence_forward(q.tf, W, q.W_t, q.H, q.ws)
        mark(4)
        if args.method == "ldlq":
            Q.quip_ldl(q.H, q.D, q.ws)
            mark(5)
            Q.quip_ldlq_quantize(q.W_t, q.H, cfg.bits, cfg.block, q.codes, q.lo, q.scale, q.ws)
        else:
            q.prepare_hessian()
            mark(5)
            q.round_weights()
        mark(6)
        Q.quip_dequantize(q.codes, q.lo, q.scale, q.W_hat)
        mark(7)
        Q.quip_incoherence_inverse(q.tf, q.W_hat, q.W_hat, q.ws)
        mark(8)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    st = Q.quip_sync_status()
    if st != L.QUIP_OK:
        raise RuntimeError(f"device status after warm-up: {L.status_string(st)}")

    # the timed step: for LDLQ the library's whole-layer call on the
    # device-resident W and X (quip_quantize_layer), else the method's calls
    def whole_step():
        if args.method == "ldlq":
            q.run(W, X)
        else:
            step()

    for _ in range(max(3, args.warmup)):
        whole_step()
    torch.cuda.synchronize()
    nev = len(STAGES) + 1
    step_ms, stage_ms = [], [[] for _ in STAGES]
    launches0 = lib.quip_kernel_launches()
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            flush.zero_()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            whole_step()
            e1.record(stream)
            torch.cuda.synchronize()
            step_ms.append(e0.elapsed_time(e1))
            if world > 1:
                dist.barrier()
    launches = lib.quip_kernel_launches() - launches0
    st = Q.quip_sync_status()
    if st != L.QUIP_OK:
        raise RuntimeError(f"device status after timing: {L.status_string(st)}")

    # stage breakdown: the same path as one call per stage, events in between
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
        step(ev)
        torch.cuda.synchronize()
        for i in range(len(STAGES)):
            stage_ms[i].append(ev[i].elapsed_time(ev[i + 1]))

    # ---- per-kernel device time: the same steps again, each launch bracketed
    # by CUDA events on its own stream (kept out of the timed region above)
    Q.quip_timing_begin()
    for _ in range(args.steps):
        flush.zero_()
        torch.cuda.synchronize()
        step()
    torch.cuda.synchronize()
    per_kernel = Q.quip_timing_end()

    total_ms = max_over_ranks(float(sum(step_ms)), world, "cuda")
    ms_per_step = total_ms / args.steps
    value = job_throughput(cfg, world, ms_per_step)

    # ---- end to end through the public API: pinned host inputs in, codes + grid
    # out (LDLQ: one library call, quip_quantize_layer_host, copies included)
    codes_h = torch.empty(cfg.m, cfg.n, dtype=torch.uint8).pin_memory()
    lo_h = torch.empty(cfg.m, dtype=torch.float32).pin_memory()
    sc_h = torch.empty(cfg.m, dtype=torch.float32).pin_memory()
    e2e_ms = []
    for i in range(max(1, args.e2e_steps) + 1):
        flush.zero_()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        q.run_host(W_h, X_h, codes_h, lo_h, sc_h)
        e1.record(stream)
        torch.cuda.synchronize()
        if i > 0:                      # the first one is a warm-up
            e2e_ms.append(e0.elapsed_time(e1))
    e2e = max_over_ranks(statistics.mean(e2e_ms), world, "cuda")
    h2d = W_h.numel() * W_h.element_size() + X_h.numel() * X_h.element_size()
    d2h = codes_h.numel() + 4 * (lo_h.numel() + sc_h.numel())

    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    pk = peaks()
    work = stage_work(cfg)
    stages = {}
    for i, name in enumerate(STAGES):
        ms = statistics.mean(stage_ms[i])
        kind, amount, bound = work[name]
        if args.method != "ldlq" and name in ("ldl", "ldlq"):
            stages[name] = {"ms": round(ms, 4)}      # the method's own kernels: see "kernels"
            continue
        stages[name] = {"ms": round(ms, 4), **roofline_entry(kind, amount, bound, ms, pk)}
    kwork = kernel_work(cfg, args.method, args.passes)
    kernels = {}
    for name, (cnt, tot_ms) in per_kernel.items():
        ent = {"launches_per_step": cnt / args.steps, "ms_per_step": round(tot_ms / args.steps, 4)}
        if name in kwork:
            kind, amount, bound = kwork[name]
            ent.update(roofline_entry(kind, amount, bound, tot_ms / args.steps, pk, split=is_split(name)))
            ent["traffic"] = kernel_traffic(name, cfg.name)
        kernels[name] = ent
    ranked = sorted((k for k in kernels if "frac" in kernels[k]), key=lambda k: -kernels[k]["ms_per_step"])
    dominant = ranked[0]
    dk = kernels[dominant]
    roof = {"bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"], "unit": dk["unit"],
            "frac": dk["frac"], "traffic": kernel_traffic(dominant, cfg.name), "kernel": dominant,
            **({"peak_note": dk["peak_note"]} if "peak_note" in dk else {}),
            "launches_per_step": dk["launches_per_step"],
            "avg_launch_ms": round(dk["ms_per_step"] / max(dk["launches_per_step"], 1e-9), 5),
            "peak_source": pk["source"]}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded Gaussian W / X with outliers, bf16; no weights or C4 in the box)",
        "config": config_desc(cfg, args),
        "roofline": roof,
        "stages": stages,
        # speed of light of the LDLQ pipeline's stages over the measured step
        **({"pipeline": pipeline_entry(cfg, pk, ms_per_step)} if args.method == "ldlq" else {}),
        "kernels": kernels,
        "e2e": {"value": job_throughput(cfg, world, e2e), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_entry(cfg, d)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_decode(args):
    """Inference: one decode step of a batch of B tokens through every linear
    layer of a Llama-2-7B decoder stack (32 blocks x q, k, v, o 4096x4096,
    gate, up 11008x4096, down 4096x11008), each a QuantizedLinear on packed
    b-bit codes with its incoherence transform applied around the product
    (Hadamard on 4096-wide sides, Kronecker 86x128 on 11008-wide ones).
    Codes, grids and transforms are seeded and synthetic (the product's time
    does not depend on the code values).  The 224 products of a step are
    captured in one CUDA graph, with the block's data dependencies: q, k and
    v (and gate and up) read the same input and run on parallel branches.
    The packed codes (1.6 GB at 2 bits) exceed L2, so every step streams them
    from HBM.  Attention and the activations between layers are not part of
    the step: o reads v's product and down reads up's in their place."""
    import torch
    import post_weight_quantization_09_b200 as Q
    from post_weight_quantization_09_b200 import _lib as L
    from quip_synth import Side
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    lib = Q.load()
    bits, B, blocks = args.bits, args.decode_batch, args.decode_blocks
    had, kron = Side("hadamard"), Side("kronecker", 86, 128)
    shapes = [("q", 4096, 4096, had, had), ("k", 4096, 4096, had, had), ("v", 4096, 4096, had, had),
              ("o", 4096, 4096, had, had), ("gate", 11008, 4096, kron, had),
              ("up", 11008, 4096, kron, had), ("down", 4096, 11008, had, kron)]
    g = torch.Generator(device="cuda").manual_seed(1234 + rank)
    layers = []
    for blk in range(blocks):
        for i, (name, m, n, ms, ns) in enumerate(shapes):
            seed = 1000 * blk + i + 7919 * rank
            tf = Q.Transform(seed, m, n, ms, ns)
            codes = torch.randint(0, 2 ** bits, (m, n), generator=g, device="cuda", dtype=torch.uint8)
            lo = torch.rand(m, generator=g, device="cuda") * -0.05
            sc = torch.rand(m, generator=g, device="cuda") * 0.01 + 0.001
            layers.append(Q.QuantizedLinear(tf, codes, lo, sc, bits, max_batch=B))
            del codes
    torch.cuda.synchronize()
    x0 = torch.randn(B, 4096, device="cuda", generator=g)
    outs = [torch.empty(B, ql.m, device="cuda") for ql in layers]
    side = [torch.cuda.Stream() for _ in range(2)]

    def parallel(main, jobs):
        """Run (layer, input, output) jobs that read the same input on the
        main stream and the side streams, then join them into the main one."""
        streams = [main] + side[:len(jobs) - 1]
        for s_ in streams[1:]:
            s_.wait_stream(main)
        for s_, (ql, inp, out) in zip(streams, jobs):
            with torch.cuda.stream(s_):
                ql(inp, out)
        for s_ in streams[1:]:
            main.wait_stream(s_)

    def step():
        # one decoder block: q, k, v read the block's input; o reads the
        # attention output (here v's product stands in for it); gate and up
        # read o's; down reads up's (in place of act(gate) * up); the next
        # block reads down's
        main = torch.cuda.current_stream()
        x = x0
        for blk in range(blocks):
            i = 7 * blk
            parallel(main, [(layers[i + t], x, outs[i + t]) for t in range(3)])
            parallel(main, [(layers[i + 3], outs[i + 2], outs[i + 3])])
            parallel(main, [(layers[i + 4], outs[i + 3], outs[i + 4]), (layers[i + 5], outs[i + 3], outs[i + 5])])
            parallel(main, [(layers[i + 6], outs[i + 5], outs[i + 6])])
            x = outs[i + 6]

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    torch.cuda.synchronize()
    st = Q.quip_sync_status()
    if st != L.QUIP_OK:
        raise RuntimeError(f"device status after warm-up: {L.status_string(st)}")
    graph = torch.cuda.CUDAGraph()
    launches0 = lib.quip_kernel_launches()
    with torch.cuda.graph(graph, stream=stream):
        step()
    per_step_launches = lib.quip_kernel_launches() - launches0
    torch.cuda.synchronize()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    ms = []
    main = torch.cuda.current_stream()
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(main)
            graph.replay()
            e1.record(main)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
    # per-kernel device time of the same step, eager, each launch bracketed by events
    Q.quip_timing_begin()
    with torch.cuda.stream(stream):
        for _ in range(min(args.steps, 20)):
            step()
    torch.cuda.synchronize()
    per_kernel = Q.quip_timing_end()
    nrep = min(args.steps, 20)
    st = Q.quip_sync_status()
    if st != L.QUIP_OK:
        raise RuntimeError(f"device status after timing: {L.status_string(st)}")
    ms_step = max_over_ranks(statistics.mean(ms), world, "cuda")
    code_bytes = sum(ql.packed.numel() * 4 for ql in layers)
    grid_bytes = sum(8 * ql.m for ql in layers)
    weights = sum(ql.m * ql.n for ql in layers)
    pk = peaks()
    qk = per_kernel.get("k_qmatvec", (0, 0.0))
    qms = qk[1] / nrep
    # algorithmic bytes of the products: packed codes, grids, x' in and z out
    qbytes = code_bytes + grid_bytes + 4.0 * B * sum(ql.m + ql.n for ql in layers)
    kernels = {k: {"launches_per_step": c / nrep, "ms_per_step": round(t / nrep, 4)}
               for k, (c, t) in per_kernel.items()}
    ach = qbytes / (qms * 1e-3) / 1e9 if qms > 0 else None
    line = {
        "metric": f"decode tokens/s through the quantized linear layers of a Llama-2-7B stack "
                  f"({bits}-bit, batch {B})",
        "value": world * B * 1e3 / ms_step, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded random codes, grids, transforms)",
        "config": {"workload": f"{blocks} blocks x (q, k, v, o 4096x4096; gate, up 11008x4096; down "
                               f"4096x11008), {bits}-bit packed codes ({code_bytes / 1e9:.2f} GB), "
                               f"batch {B}, one CUDA graph per step (q / k / v and gate / up on "
                               f"parallel branches)",
                   "weights": weights, "l2": "not flushed: the packed codes exceed L2 (126 MB)"},
        "roofline": {"bound": "hbm", "achieved": round(ach, 1) if ach else None, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": round(ach / pk["hbm_gbs"], 4) if ach else None,
                     "traffic": None, "kernel": "k_qmatvec",
                     "step_gbs": round(qbytes / (ms_step * 1e-3) / 1e9, 1),
                     "peak_source": pk["source"]},
        "kernels": kernels,
        "gpu_launches": int(per_step_launches * args.steps),
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph


def run_group(args, cfg: LayerConfig):
    """G layers of cfg's shape reading the same input X (q / k / v of an
    attention block, up / gate of an MLP): one Hessian, one transform of it
    and one LDL for the group, LDLQ on the stacked rows.  value = G m n /
    step time (quantized weights per second)."""
    import torch
    import post_weight_quantization_09_b200 as Q
    from post_weight_quantization_09_b200 import _lib as L
    world, rank, local = dist_setup()
    if world > 1:
        raise SystemExit("--group runs on one GPU")
    torch.cuda.set_device(local)
    lib = Q.load()
    G = args.group
    as_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 \
        else torch.from_numpy(a)
    Ws, X = [], None
    for g in range(G):
        d = make_layer(rank_config(cfg, g))           # seed + g: G different weight matrices
        Ws.append(as_t(d["W_bf16"] if cfg.dtype == "bf16" else d["W"]).cuda())
        if X is None:
            X = as_t(d["X_bf16"] if cfg.dtype == "bf16" else d["X"]).cuda()
    q = Q.LayerGroupQuantizer(G, cfg.m, cfg.n, cfg.m_side, cfg.n_side, cfg.bits, cfg.block, cfg.damp,
                              cfg.seed)
    stream = torch.cuda.current_stream()
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")   # 256 MB > L2
    for _ in range(max(3, args.warmup)):
        q.run(Ws, X)
    torch.cuda.synchronize()
    st = Q.quip_sync_status()
    if st != L.QUIP_OK:
        raise RuntimeError(f"device status after warm-up: {L.status_string(st)}")
    step_ms = []
    launches0 = lib.quip_kernel_launches()
    with ClockSampler(local) as clk:
        for _ in range(args.steps):
            flush.zero_()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            q.run(Ws, X)
            b.record(stream)
            torch.cuda.synchronize()
            step_ms.append(a.elapsed_time(b))
    launches = (lib.quip_kernel_launches() - launches0) // max(1, args.steps)
    ms = statistics.mean(step_ms)
    desc = config_desc(cfg, args)
    desc["workload"] = f"{G} layers sharing one input, each " + desc["workload"]
    desc["group"] = G
    line = {"metric": METRIC, "value": G * cfg.m * cfg.n / (ms * 1e-3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded Gaussian W / X with outliers, bf16; no weights or C4 in the box)",
            "config": desc, "gpu_launches_per_step": launches, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="gate70b", choices=sorted(CONFIGS),
                    help="workload (default: the largest single-GPU layer, the 70B-shaped MLP gate)")
    ap.add_argument("--all-configs", action="store_true",
                    help="one JSON line per workload (tiny, attn7b, up7b, down7b, gate70b)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--group", type=int, default=1,
                    help="layers of the config's shape sharing one input (one Hessian and LDL)")
    ap.add_argument("--permute", action="store_true",
                    help="random permutation within both sides' orthogonal transforms")
    ap.add_argument("--method", default="ldlq", choices=["ldlq", "nearest", "greedy", "ldlq_rg"],
                    help="rounding method (QuIP, Experiments, Methods)")
    ap.add_argument("--passes", type=int, default=1, help="greedy passes of greedy / ldlq_rg")
    ap.add_argument("--decode", action="store_true",
                    help="inference: quantized products of a Llama-2-7B linear stack per decode step")
    ap.add_argument("--decode-batch", type=int, default=1)
    ap.add_argument("--decode-blocks", type=int, default=32)
    ap.add_argument("--bits", type=int, default=2, help="code width of --decode")
    ap.add_argument("--rows", type=int, default=0,
                    help="a slice of the workload with this many rows of W (its n, sides and bits kept; "
                         "a Kronecker m side keeps q and takes p = rows / q): for profiling at a size "
                         "a capture can hold")
    ap.add_argument("--tokens", type=int, default=0, help="calibration tokens of the slice (default: the workload's)")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]
    if args.rows or args.tokens:
        from dataclasses import replace as _rep
        ms = cfg.m_side
        if args.rows:
            if ms.kind == "kronecker":
                if args.rows % ms.q:
                    raise SystemExit(f"--rows must be a multiple of q = {ms.q}")
                ms = _rep(ms, p=args.rows // ms.q)
            elif ms.kind == "hadamard" and args.rows & (args.rows - 1):
                raise SystemExit("--rows must be a power of two for a Hadamard m side")
        cfg = _rep(cfg, name=f"{cfg.name}[slice]", m=args.rows or cfg.m, N=args.tokens or cfg.N, m_side=ms)
    if args.permute:
        from dataclasses import replace
        cfg = replace(cfg, m_side=replace(cfg.m_side, permute=True),
                      n_side=replace(cfg.n_side, permute=True))
    if args.decode:
        run_decode(args)
        return
    if args.all_configs:
        from dataclasses import replace as _rep
        for name in ("tiny", "attn7b", "up7b", "down7b", "gate70b"):
            c = CONFIGS[name]
            if args.permute:
                c = _rep(c, m_side=_rep(c.m_side, permute=True), n_side=_rep(c.n_side, permute=True))
            (run_reference if args.impl == "reference" else run_ours)(args, c)
        return
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        if args.group > 1:
            if args.method != "ldlq":
                raise SystemExit("--group runs LDLQ only")
            run_group(args, cfg)
        else:
            run_ours(args, cfg)


if __name__ == "__main__":
    main()
