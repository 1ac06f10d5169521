#!/usr/bin/env python
"""Benchmark of the FP8 linear layer with per-tensor delayed scaling on B200.

One *step* is the whole hot path over one batch: the forward and backward (dX, dW, bias
gradient) of every linear of a 12-layer, dim-1024 transformer trained at batch 4 x 512
tokens (M = 2048 rows); per layer the (K, N) = (1024, 3072), (1024, 1024), (1024, 4096),
(4096, 1024) projections.  HYBRID formats (E4M3 forward, E5M2 backward), delayed scaling with
history 16 and margin 0, bias fused into the forward GEMM.  Per linear and step (default
``--path rowmajor``): one row-major quantize launch (x and w, each written in E4M3 for the
forward and in E5M2 with the forward's steps for the backward, from the same products) + one
GEMM launch forward (the GEMM also folds the two rings), one quantize launch (g row-major with
per-tile column sums) + one GEMM launch backward (dX = g8 . w8 and dW = g8^T . x8 with the
operands read in place as MN-major tiles, grad_b reduced by its epilogue warps, the g ring
folded).  ``--path saved`` writes x^T / w^T in the forward instead and quantizes g in both
orientations; ``--path requant`` runs the pages' own split of the same work (the forward
quantizes x, w row-major; the backward re-quantizes x^T, w^T beside g).  All three give the
same numbers (the pages' HYBRID backward), and the line reports the other two as variants.

Timing: every layer has its own weights, activations and gradients (about 3 GB, far above
the 126 MB L2).  The step is captured as CUDA graphs (one per history-ring slot, since the
slot index is a host-side argument) and replayed; device time from CUDA events with a
synchronize on both sides, max over ranks.  Per-kernel durations for the roofline come from
the library's own CUDA-event profiler over instrumented replays of the same step.  Beside the
headline the line reports the other compositions and the mixed-format backward (variants), and
the sweeps of single GEMMs and quantizes.

``--impl reference`` times the CPU oracle (the plain restatement of the method, on the host
cores) on a bounded sample of the same workload: one training linear per step.

Launch: ``python bench.py [--gpus N --steps K --warmup W]``; N > 1 under torchrun runs the
step data parallel: every rank its own batch (weak scaling) and, after each step, one
all-reduce (MAX) of every history ring's amax so that all ranks fold the same rings.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FP8 GEMM TFLOP/s (fwd/dX/dW) + quantize GB/s, % of B200 roofline"
UNIT = "TFLOP/s"
HIST = 16
WORKLOAD = ("training linears of a 12-layer dim-1024 transformer at B4xT512 (M=2048), HYBRID "
            "(E4M3 fwd, E5M2 bwd), delayed scaling history 16 margin 0, bias, fwd+dX+dW+grad_b")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=600)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-sweeps", action="store_true")
    p.add_argument("--no-variants", action="store_true", help="skip the variant steps")
    p.add_argument("--path", default=STEP_PATH[0], choices=PATHS,
                   help="headline step: the backward's copies of x / w saved row-major or transposed by the "
                        "forward's quantize launch, or re-quantized by the backward's (identical numbers)")
    p.add_argument("--dp-fold", action="store_true",
                   help="fold the rings once per step after an amax all-reduce (always on with several GPUs)")
    p.add_argument("--kernel", default=None, choices=["gemm", "quantize", "linear"],
                   help="time one kernel on one shape instead of the step (small cases for ncu)")
    p.add_argument("--shape", default="4096,4096,4096", help="gemm: M,N,K; quantize: ROWS,COLS; linear: M,K,N")
    p.add_argument("--qmode", default="dual", choices=["row", "t", "dual"])
    p.add_argument("--gemm-split-k", type=int, default=None,
                   help="GEMM split-K mode: 0 automatic, 1 never, 2..4 forced (library default if omitted)")
    p.add_argument("--tiled-persist-threshold", type=int, default=None,
                   help="tile count above which transposed / dual quantize runs persistent "
                        "(library default if omitted)")
    return p.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


# ---------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------------------
def oracle_linear_step(k, n, seed, shrink=1):
    """The oracle's forward + backward of one training linear (M = 2048 rows), every dimension
    divided by `shrink` for a bounded sample; returns (seconds, flops)."""
    import numpy as np
    import workloads as W
    from oracle import linear as L
    from oracle import scaling as S

    m, k, n = W.TRAINING_TOKENS // shrink, k // shrink, n // shrink
    t = W.training_linear(m, k, n, seed)
    bits = {key: W.bf16_bits(t[key]) for key in ("x", "w", "b", "g")}
    rx, rw, rg = S.Ring(HIST, "e4m3"), S.Ring(HIST, "e4m3"), S.Ring(HIST, "e5m2")
    f32 = {key: t[key].float().numpy() for key in ("x", "w", "g")}
    rx.seed(f32["x"])
    rw.seed(f32["w"])
    rg.seed(f32["g"])
    t0 = time.perf_counter()
    f = L.forward(bits["x"], bits["w"], bits["b"], "e4m3", rx, rw)
    L.backward(bits["g"], bits["x"], bits["w"], "e5m2", f["sx"], f["sw"], rg)
    dt = time.perf_counter() - t0
    del np
    return dt, 3 * 2.0 * m * k * n


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline():
    import workloads as W
    total_t, total_f = 0.0, 0.0
    for i, (k, n) in enumerate(W.TRAINING_LINEARS):
        dt, fl = oracle_linear_step(k, n, seed=7000 + i)
        total_t += dt
        total_f += fl
    return {"value": total_f / total_t / 1e12, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": "one transformer layer (its 4 training linears, M=2048) forward + backward through the "
                      f"numpy oracle (fp64 GEMMs): {total_f / 1e9:.1f} GFLOP in {total_t:.1f} s"}


REFERENCE_BUDGET_S = 150.0  # wall-clock budget of a whole --impl reference run


def reference_shrink(steps, warmup):
    """The factor (a power of two, at most 32) every dimension of the reference steps' training
    linear is divided by, so that warm-up plus timed steps stay within REFERENCE_BUDGET_S.  The
    oracle's wall-clock cost (input generation included) is calibrated on one step shrunk 16x
    and taken to grow with the square of the factor it saves (a conservative bound: its GEMMs
    grow with the cube)."""
    oracle_linear_step(1024, 3072, seed=7998, shrink=32)  # first-call overheads out of the way
    t0 = time.perf_counter()
    for k, n in ((1024, 3072), (1024, 1024), (1024, 4096), (4096, 1024)):
        oracle_linear_step(k, n, seed=7999, shrink=16)
    cal = max((time.perf_counter() - t0) / 4, 1e-4)
    per_step = REFERENCE_BUDGET_S / max(1, steps + warmup)
    for shrink in (1, 2, 4, 8, 16):
        if cal * (16 / shrink) ** 2 <= per_step:
            return shrink
    return 32


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import workloads as W
    shrink = reference_shrink(args.steps, args.warmup)
    for i in range(args.warmup):
        k, n = W.TRAINING_LINEARS[i % 4]
        oracle_linear_step(k, n, seed=8000 + i, shrink=shrink)
    total_t, total_f = 0.0, 0.0
    for i in range(args.steps):
        k, n = W.TRAINING_LINEARS[i % 4]
        dt, fl = oracle_linear_step(k, n, seed=9000 + i, shrink=shrink)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    sample = (f"one training linear per step ((M,K,N) = (2048,K,N) / {shrink}, (K,N) cycling over the 4 "
              f"shapes; sized so the run stays within about {REFERENCE_BUDGET_S:.0f} s) forward + backward "
              f"through the numpy oracle; {args.steps} steps, {total_t:.1f} s timed")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_t * 1e3 / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": f"one linear per step, every dimension / {shrink}"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------
# GPU workload
# ---------------------------------------------------------------------------------------
class Linear:
    def __init__(self, F, W, torch, m, k, n, seed, dev):
        self.F, self.m, self.k, self.n = F, m, k, n
        t = W.training_linear(m, k, n, seed, device=dev)
        self.x, self.w, self.b, self.g = t["x"], t["w"], t["b"], t["g"]
        bf = torch.bfloat16
        self.y = torch.empty((m, n), dtype=bf, device=dev)
        self.gx = torch.empty((m, k), dtype=bf, device=dev)
        self.gw = torch.empty((n, k), dtype=bf, device=dev)
        self.gb = torch.empty((n,), dtype=bf, device=dev)
        self.fws_n = F.linear_forward_fp8_workspace_size(m, k, n)
        self.bws_n = F.linear_backward_fp8_workspace_size(m, k, n)
        self.fws = torch.empty(self.fws_n, dtype=torch.uint8, device=dev)
        self.bws = torch.empty(self.bws_n, dtype=torch.uint8, device=dev)
        self.state = torch.zeros((3, HIST + 4), dtype=torch.float32, device=dev)
        self.steps = torch.zeros(4, dtype=torch.float32, device=dev)  # sx, sw, sg
        for i in range(3):
            F.fp8_scale_ring_init(self.state[i], HIST)
        self.rx = F.Ring(self.state[0], HIST, F.FP8_E4M3)
        self.rw = F.Ring(self.state[1], HIST, F.FP8_E4M3)
        self.rg = F.Ring(self.state[2], HIST, F.FP8_E5M2)
        F.fp8_scale_ring_seed(self.rx, self.x, F.FP8_IN_BF16, self.x.numel())
        F.fp8_scale_ring_seed(self.rw, self.w, F.FP8_IN_BF16, self.w.numel())
        F.fp8_scale_ring_seed(self.rg, self.g, F.FP8_IN_BF16, self.g.numel())

    def set_slot(self, idx):
        self.rx.hist_idx = self.rw.hist_idx = self.rg.hist_idx = idx

    def fwd(self):
        F = self.F
        F.linear_forward_fp8(self.x, self.w, 0, None, self.b, None, self.m, self.k, self.n, F.FP8_E4M3, self.rx,
                             self.rw, 1.0, self.steps[0:1], self.steps[1:2], self.fws, self.fws_n, self.y)

    def bwd(self):
        F = self.F
        F.linear_backward_fp8(self.g, self.x, self.w, self.m, self.k, self.n, F.FP8_E5M2, 1, 1, 1,
                              self.steps[0:1], self.steps[1:2], self.rg, 1.0, self.steps[2:3], self.bws,
                              self.bws_n, self.gx, self.gw, self.gb)

    def fwd_keep(self):
        """Forward that keeps x8 / w8 for the mixed-format backward."""
        F = self.F
        if not hasattr(self, "x8k"):
            import torch
            self.x8k = torch.empty((self.m, self.k), dtype=torch.uint8, device=self.x.device)
            self.w8k = torch.empty((self.n, self.k), dtype=torch.uint8, device=self.x.device)
            self.mws_n = F.linear_backward_fp8_mixed_workspace_size(self.m, self.k, self.n)
            self.mws = torch.empty(self.mws_n, dtype=torch.uint8, device=self.x.device)
        F.linear_forward_fp8_keep(self.x, self.w, 0, None, self.b, None, self.m, self.k, self.n, F.FP8_E4M3, self.rx,
                                  self.rw, 1.0, self.steps[0:1], self.steps[1:2], self.x8k, self.w8k, self.fws,
                                  self.fws_n, self.y)

    def bwd_mixed(self):
        """Backward that quantizes only g (E5M2) and reuses the forward's E4M3 x8 / w8."""
        F = self.F
        F.linear_backward_fp8_mixed(self.g, self.x8k, self.w8k, self.m, self.k, self.n, F.FP8_E5M2, F.FP8_E4M3,
                                    F.FP8_E4M3, 1, 1, 1, self.steps[0:1], self.steps[1:2], self.rg, 1.0,
                                    self.steps[2:3], self.mws, self.mws_n, self.gx, self.gw, self.gb)

    def fwd_save(self):
        """Forward whose quantize launch also writes x^T / w^T (E5M2, the forward's steps)."""
        F = self.F
        if not hasattr(self, "x8t"):
            import torch
            self.x8t = torch.empty((self.k, self.m), dtype=torch.uint8, device=self.x.device)
            self.w8t = torch.empty((self.k, self.n), dtype=torch.uint8, device=self.x.device)
            self.sws_n = F.linear_backward_fp8_saved_t_workspace_size(self.m, self.k, self.n)
            self.sws = torch.empty(self.sws_n, dtype=torch.uint8, device=self.x.device)
        F.linear_forward_fp8_save_t(self.x, self.w, self.b, None, self.m, self.k, self.n, F.FP8_E4M3, F.FP8_E5M2,
                                    self.rx, self.rw, self.steps[0:1], self.steps[1:2], self.x8t, self.w8t, self.fws,
                                    self.fws_n, self.y)

    def bwd_saved(self):
        """Backward that quantizes only g and reads the forward's saved x^T / w^T."""
        F = self.F
        F.linear_backward_fp8_saved_t(self.g, self.x8t, self.w8t, self.m, self.k, self.n, F.FP8_E5M2, F.FP8_E5M2,
                                      1, 1, 1, self.steps[0:1], self.steps[1:2], self.rg, 1.0, self.steps[2:3],
                                      self.sws, self.sws_n, self.gx, self.gw, self.gb)

    def fwd_save_rm(self):
        """Forward whose row-major quantize launch also writes x and w in E5M2 (the forward's
        steps), row-major, for the backward."""
        F = self.F
        if not hasattr(self, "x8b"):
            import torch
            self.x8b = torch.empty((self.m, self.k), dtype=torch.uint8, device=self.x.device)
            self.w8b = torch.empty((self.n, self.k), dtype=torch.uint8, device=self.x.device)
            self.rws_n = F.linear_backward_fp8_mixed_workspace_size(self.m, self.k, self.n)
            self.rws = torch.empty(self.rws_n, dtype=torch.uint8, device=self.x.device)
        F.linear_forward_fp8_save_rm(self.x, self.w, self.b, None, self.m, self.k, self.n, F.FP8_E4M3, F.FP8_E5M2,
                                     self.rx, self.rw, self.steps[0:1], self.steps[1:2], self.x8b, self.w8b, self.fws,
                                     self.fws_n, self.y)

    def bwd_saved_rm(self):
        """Backward that quantizes only g (row-major) and reads the forward's E5M2 x / w in place."""
        F = self.F
        F.linear_backward_fp8_mixed(self.g, self.x8b, self.w8b, self.m, self.k, self.n, F.FP8_E5M2, F.FP8_E5M2,
                                    F.FP8_E5M2, 1, 1, 1, self.steps[0:1], self.steps[1:2], self.rg, 1.0,
                                    self.steps[2:3], self.rws, self.rws_n, self.gx, self.gw, self.gb)

    @property
    def quant_bytes_saved_rm(self):
        m, k, n = self.m, self.k, self.n
        # fwd: x, w row-major in two formats (2 B in, 1 + 1 B out); bwd: g row-major (2 + 1)
        return 4 * (m * k + n * k) + 3 * m * n

    @property
    def quant_bytes_saved(self):
        m, k, n = self.m, self.k, self.n
        # fwd: x, w in both orientations (2 B in, 1 + 1 B out); bwd: g dual (2 + 1 + 1)
        return 4 * (m * k + n * k) + 4 * m * n

    @property
    def quant_bytes_mixed(self):
        m, k, n = self.m, self.k, self.n
        # fwd: x, w row-major (2 B in, 1 B out); bwd: g row-major (2 B in, 1 B out)
        return 3 * (m * k + n * k) + 3 * m * n

    @property
    def gemm_flops(self):
        return 3 * 2.0 * self.m * self.k * self.n

    @property
    def quant_bytes(self):
        m, k, n = self.m, self.k, self.n
        # fwd: x, w row-major (2 B in, 1 B out); bwd: g dual (2 + 1 + 1), x^T, w^T (2 + 1)
        return 3 * (m * k + n * k) + 4 * m * n + 3 * (m * k + n * k)


def build_workload(F, W, torch, dev, seed_base):
    lins = []
    for layer in range(W.TRAINING_LAYERS):
        for j, (k, n) in enumerate(W.TRAINING_LINEARS):
            lins.append(Linear(F, W, torch, W.TRAINING_TOKENS, k, n, seed_base + 100 * layer + 10 * j, dev))
    return lins


PATHS = ("rowmajor", "saved", "requant")
PATH_WHAT = {
    "rowmajor": "x and w also written in E5M2 (the forward's steps), row-major, by the forward's quantize "
                "launch; the backward quantizes only g (row-major) and its GEMMs read g8, x8 and w8 in place "
                "(MN-major operands)",
    "saved": "x^T / w^T (E5M2, the forward's steps) written by the forward's quantize launch; the backward "
             "quantizes only g",
    "requant": "the backward's quantize launch re-quantizes x^T / w^T (E5M2, the forward's steps) beside g",
}
STEP_PATH = ["rowmajor"]  # the headline step's composition (--path)


def quant_bytes_of(lin, path):
    return {"rowmajor": lin.quant_bytes_saved_rm, "saved": lin.quant_bytes_saved, "requant": lin.quant_bytes}[path]


def run_step(lins, slot, mixed=False, path=None):
    """One training step: every linear's forward, then every backward in reverse order.
    path "saved": the forward's quantize launch also writes x^T / w^T for the backward (same
    bytes as re-quantizing them there); "requant": the backward re-quantizes x^T / w^T.
    mixed=True: the forward keeps x8 / w8 and the backward reuses them (E5M2 g only)."""
    path = path or STEP_PATH[0]
    for lin in lins:
        lin.set_slot(slot)
    for lin in lins:
        if mixed:
            lin.fwd_keep()
        elif path == "rowmajor":
            lin.fwd_save_rm()
        elif path == "saved":
            lin.fwd_save()
        else:
            lin.fwd()
    for lin in reversed(lins):
        if mixed:
            lin.bwd_mixed()
        elif path == "rowmajor":
            lin.bwd_saved_rm()
        elif path == "saved":
            lin.bwd_saved()
        else:
            lin.bwd()


# ---------------------------------------------------------------------------------------
# Clocks and peaks
# ---------------------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def start_clock_sampler(torch, dev):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    ids = [v.strip() for v in vis.split(",") if v.strip()] if vis else []
    target = ids[dev.index] if dev.index is not None and dev.index < len(ids) else str(dev.index or 0)
    cmd = ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
    if target:
        cmd += ["-i", target]
    try:
        return subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
    except Exception:
        return None


def stop_clock_sampler(proc):
    if proc is None:
        return None
    proc.terminate()
    try:
        out, _ = proc.communicate(timeout=10)
    except Exception:
        proc.kill()
        return None
    sm, mx, reasons = [], [], set()
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    for line in out.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx.append(float(parts[2]))
        except ValueError:
            continue
        for name, val in zip(names, parts[5:9]):
            if val.lower().startswith("active"):
                reasons.add(name)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def gemm_traffic_per_launch():
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was taken on the
    current GEMM source (its hash is recorded there); otherwise None."""
    import hashlib
    summary = os.path.join(ROOT, "profiles", "fp8_gemm_training_linears_traffic.txt")
    src = os.path.join(ROOT, "fp8_delayed_scaling_amax_b200", "csrc", "gemm.cu")
    try:
        with open(src, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
        vals = {}
        with open(summary) as f:
            for line in f:
                if "=" in line and not line.lstrip().startswith("#"):
                    key, v = line.split("=", 1)
                    vals[key.strip()] = v.strip()
        if vals.get("gemm_source_sha256_16") != h:
            return None
        return float(vals["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------------------
# Single-kernel timing: rotate enough input sets that the bytes touched exceed twice the L2,
# so every launch reads its operands from HBM.
# ---------------------------------------------------------------------------------------
L2_BYTES = 126 * 1024 * 1024


def _graph_time(torch, launch, iters, warmup, slots=1):
    """Capture `iters` back-to-back launches in CUDA graphs and time their replay, so host
    launch cost does not show up in the device time.  `slots` > 1 captures one graph per
    history-ring slot (the slot index is a host argument baked into the capture)."""
    cap = torch.cuda.Stream()
    for i in range(warmup):
        launch(i)
    torch.cuda.synchronize()
    graphs = []
    for sl in range(slots):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for i in range(iters):
                launch(i)
        graphs.append(g)
    graphs[0].replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for g in graphs:
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / (iters * slots)


def time_gemm(F, W, torch, dev, m, n, k, iters=20, warmup=5, batch=1, bcast_b=False, hot=False):
    """hot=False: enough operand sets rotated that each launch reads from HBM; hot=True: one
    set, so operands smaller than L2 stay resident (the pages time their GEMMs this way)."""
    per_set = batch * m * k + (1 if bcast_b else batch) * n * k + batch * m * n * 2
    nsets = 1 if hot else max(1, min(16, (2 * L2_BYTES) // max(per_set, 1) + 1))
    sets = []
    for i in range(nsets):
        a = W.fp8_bytes((batch, m, k), seed=31 + i, device=dev)
        b = W.fp8_bytes((1 if bcast_b else batch, n, k), seed=57 + i, device=dev)
        out = torch.empty((batch, m, n), dtype=torch.bfloat16, device=dev)
        sets.append((a, b, out))
    sa = torch.tensor([0.75], device=dev)
    sb = torch.tensor([1.5], device=dev)
    bias = W.normal_bf16((n,), 0.1, seed=5, device=dev)

    def launch(i):
        a, b, out = sets[i % nsets]
        F.fp8_gemm(a, b, 0, 0, F.FP8_LAYOUT_NT, m, n, k, k, k, n, batch, m * k if batch > 1 else 0,
                   0 if (bcast_b or batch == 1) else n * k, m * n, sa, sb, bias, None, out)

    ms = _graph_time(torch, launch, iters, warmup)
    return {"ms": ms, "tflops": 2.0 * batch * m * n * k / (ms * 1e-3) / 1e12, "sets": nsets}


def time_fp8_output(F, W, torch, dev, m, n, k, fused, iters=20, warmup=5):
    """The producer-side quantize of a GEMM output: fused (fp8_gemm_fp8out writing only the fp8
    bytes, amax into a ring slot) or as two launches (fp8_gemm to bf16, then fp8_quantize of that
    output folding a ring)."""
    per_set = m * k + n * k + m * n * 3
    nsets = max(1, min(16, (2 * L2_BYTES) // max(per_set, 1) + 1))
    sets = []
    for i in range(nsets):
        a = W.fp8_bytes((m, k), seed=131 + i, device=dev)
        b = W.fp8_bytes((n, k), seed=157 + i, device=dev)
        out = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        out8 = torch.empty((m, n), dtype=torch.uint8, device=dev)
        st = torch.zeros(HIST + 4, dtype=torch.float32, device=dev)
        F.fp8_scale_ring_init(st, HIST)
        st[HIST] = 1.0 / 64
        sets.append((a, b, out, out8, st, F.Ring(st, HIST, F.FP8_E4M3)))
    sa = torch.tensor([0.75], device=dev)
    sb = torch.tensor([1.5], device=dev)
    bias = W.normal_bf16((n,), 0.1, seed=5, device=dev)
    used = torch.zeros(1, device=dev)

    def launch(i):
        a, b, out, out8, st, ring = sets[i % nsets]
        if fused:
            F.fp8_gemm_fp8out(a, b, 0, 0, F.FP8_LAYOUT_NT, m, n, k, k, k, n, 1, 0, 0, 0, sa, sb, bias, None, None,
                              F.FP8_E4M3, st[HIST:HIST + 1], out8, st[HIST + 2:HIST + 3], used)
        else:
            F.fp8_gemm(a, b, 0, 0, F.FP8_LAYOUT_NT, m, n, k, k, k, n, 1, 0, 0, 0, sa, sb, bias, None, out)
            F.fp8_quantize(out, F.FP8_IN_BF16, m, n, st[HIST:HIST + 1], F.FP8_E4M3, 0, out8, None, ring)

    ms = _graph_time(torch, launch, iters, warmup)
    return {"ms": ms, "tflops": 2.0 * m * n * k / (ms * 1e-3) / 1e12}


def time_quantize(F, W, torch, dev, rows, cols, mode, iters=20, warmup=5, fmt=None):
    fmt = F.FP8_E4M3 if fmt is None else fmt
    per_set = rows * cols * (2 + (2 if mode == "dual" else 1))
    nsets = max(1, min(16, (2 * L2_BYTES) // max(per_set, 1) + 1))
    sets = []
    for i in range(nsets):
        x = W.normal_bf16((rows, cols), 1.0, seed=80 + i, device=dev)
        out = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
        out_t = torch.empty((cols, rows), dtype=torch.uint8, device=dev)
        st = torch.zeros(HIST + 4, dtype=torch.float32, device=dev)
        F.fp8_scale_ring_init(st, HIST)
        ring = F.Ring(st, HIST, fmt)
        F.fp8_scale_ring_seed(ring, x, F.FP8_IN_BF16, x.numel())
        sets.append((x, out, out_t, ring))

    def launch(i):
        x, out, out_t, ring = sets[i % nsets]
        step = ring.state[HIST:HIST + 1]
        if mode == "row":
            F.fp8_quantize(x, F.FP8_IN_BF16, rows, cols, step, fmt, 0, out, None, ring)
        elif mode == "t":
            F.fp8_quantize(x, F.FP8_IN_BF16, rows, cols, step, fmt, 1, out_t, None, ring)
        else:
            F.fp8_quantize_dual(x, F.FP8_IN_BF16, rows, cols, step, fmt, out, out_t, None, ring)
        ring.advance()

    ms = _graph_time(torch, launch, iters, warmup)
    nbytes = rows * cols * (2 + (2 if mode == "dual" else 1))
    return {"ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9, "sets": nsets}


def run_kernel_mode(args):
    import torch
    import fp8_delayed_scaling_amax_b200 as F
    import workloads as W
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.tiled_persist_threshold is not None:
        F.fp8_set_tiled_persist_threshold(args.tiled_persist_threshold)
    dims = [int(v) for v in args.shape.split(",")]
    peaks = measured_peaks()
    if args.kernel == "gemm":
        m, n, k = dims
        r = time_gemm(F, W, torch, dev, m, n, k, iters=args.steps, warmup=args.warmup)
        r.update(kernel="fp8_gemm", shape=[m, n, k], frac=r["tflops"] / (2 * peaks["bf16_tflops"]))
    elif args.kernel == "linear":
        # one training linear, forward + backward, in the step's composition (--path), in a
        # CUDA graph: 4 launches per iteration
        m, k, n = dims
        STEP_PATH[0] = args.path
        lin = Linear(F, W, torch, m, k, n, 7, dev)

        def launch(i):
            run_step([lin], i % HIST)

        ms = _graph_time(torch, launch, args.steps, args.warmup)
        r = {"ms": ms, "tflops": lin.gemm_flops / (ms * 1e-3) / 1e12, "kernel": f"linear_{args.path}",
             "shape": [m, k, n]}
    else:
        rows, cols = dims
        r = time_quantize(F, W, torch, dev, rows, cols, args.qmode, iters=args.steps, warmup=args.warmup)
        r.update(kernel=f"fp8_quantize_{args.qmode}", shape=[rows, cols], frac=r["gbs"] / peaks["hbm_gbs"])
    r["status"] = F.fp8_get_device_status()
    print(json.dumps(r), flush=True)
    return 0


def run_sweeps(F, W, torch, dev):
    """Square NT GEMMs (pre-quantized E4M3, bias on), the skinny / batched shapes, and the
    quantize bandwidth sweep, each timed alone with operands rotated through HBM."""
    peaks = measured_peaks()
    burst_fp8 = 2.0 * peaks["bf16_tflops"]
    out = {"gemm_square": {}, "gemm_skinny_batched": {}, "quantize": {}, "gemm_fp8_output": {}}
    def gemm_entry(m, n, k, batch=1, bcast_b=False, iters=20):
        r = time_gemm(F, W, torch, dev, m, n, k, iters=iters, batch=batch, bcast_b=bcast_b)
        e = {"tflops": round(r["tflops"], 1), "us": round(r["ms"] * 1e3, 2), "frac": round(r["tflops"] / burst_fp8, 4)}
        # operands that fit in L2 are also timed hot (one operand set, as the pages time them)
        per_set = batch * m * k + (1 if bcast_b else batch) * n * k + batch * m * n * 2
        if per_set < L2_BYTES // 2:
            h = time_gemm(F, W, torch, dev, m, n, k, iters=iters, batch=batch, bcast_b=bcast_b, hot=True)
            e.update(hot_tflops=round(h["tflops"], 1), hot_us=round(h["ms"] * 1e3, 2))
        return e

    for s in W.SQUARE_SIZES:
        out["gemm_square"][str(s)] = gemm_entry(s, s, s, iters=20 if s < 8192 else 10)
    for ba, bb, m, n, k in W.SKINNY_BATCHED:
        batch = max(ba, bb)
        key = f"{batch}x{m}x{n}x{k}" + ("(B bcast)" if bb == 1 and batch > 1 else "")
        out["gemm_skinny_batched"][key] = gemm_entry(m, n, k, batch=batch, bcast_b=(bb == 1 and batch > 1))
    # bf16 inputs of 2^24 .. 2^28 elements with a ring; E5M2 beside E4M3 at the two larger sizes
    for rows, cols, fmts in ((8192, 2048, ("e4m3",)), (4096, 4096, ("e4m3",)), (8192, 8192, ("e4m3", "e5m2")),
                             (16384, 16384, ("e4m3", "e5m2"))):
        for fname in fmts:
            for mode in ("row", "t", "dual"):
                r = time_quantize(F, W, torch, dev, rows, cols, mode,
                                  fmt=F.FP8_E4M3 if fname == "e4m3" else F.FP8_E5M2)
                key = f"{mode}_{rows}x{cols}" + ("" if fname == "e4m3" else "_e5m2")
                out["quantize"][key] = {"gbs": round(r["gbs"], 1), "us": round(r["ms"] * 1e3, 2),
                                        "frac": round(r["gbs"] / peaks["hbm_gbs"], 4)}
    for m, n, k in ((2048, 3072, 1024), (2048, 4096, 1024), (4096, 4096, 4096)):
        fused = time_fp8_output(F, W, torch, dev, m, n, k, True)
        split = time_fp8_output(F, W, torch, dev, m, n, k, False)
        out["gemm_fp8_output"][f"{m}x{n}x{k}"] = {"fused_us": round(fused["ms"] * 1e3, 2),
                                                  "gemm_then_quantize_us": round(split["ms"] * 1e3, 2),
                                                  "fused_tflops": round(fused["tflops"], 1)}
    out["peaks"] = {"fp8_tflops_burst": burst_fp8, "hbm_gbs": peaks["hbm_gbs"], "source": peaks["source"]}
    return out


# ---------------------------------------------------------------------------------------
def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.kernel is not None:
        return run_kernel_mode(args) if rank == 0 else 0

    import torch
    import torch.distributed as dist

    import fp8_delayed_scaling_amax_b200 as F
    import workloads as W

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    F.lib()
    if args.tiled_persist_threshold is not None:
        F.fp8_set_tiled_persist_threshold(args.tiled_persist_threshold)
    if args.gemm_split_k is not None:
        F.fp8_set_gemm_split_k(args.gemm_split_k)

    STEP_PATH[0] = args.path
    lins = build_workload(F, W, torch, dev, seed_base=100000 * rank)
    flops_step = sum(l.gemm_flops for l in lins)
    qbytes_step = sum(quant_bytes_of(l, args.path) for l in lins)

    # Data parallel over several GPUs: the linears leave each ring's amax in its slot and, after
    # every step, the ranks reduce all rings' amax (one all-reduce MAX) and fold them, so every
    # rank keeps the same rings.  One GPU folds inside the calls.
    dp_rings, dp_buf = [], None
    use_dp = world > 1 or args.dp_fold
    if use_dp:
        from fp8_delayed_scaling_amax_b200 import dp as DP
        F.fp8_set_ring_fold_mode(1)
        dp_rings = [r for l in lins for r in (l.rx, l.rw, l.rg)]
        dp_buf = torch.zeros(len(dp_rings), dtype=torch.float32, device=dev)

    def end_of_step(slot):
        if use_dp:
            for l in lins:
                l.set_slot(slot)
            DP.fold_rings_data_parallel(dp_rings, dp_buf)

    # eager warm step (module load, attributes), then one graph per ring slot
    run_step(lins, 0)
    end_of_step(0)
    torch.cuda.synchronize()
    assert F.fp8_get_device_status() == 0
    cap = torch.cuda.Stream()
    graphs = []
    for slot in range(HIST):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            run_step(lins, slot)
        graphs.append(g)
    torch.cuda.synchronize()

    counter = [1]  # the eager warm step used slot 0

    def replay():
        slot = counter[0] % HIST
        graphs[slot].replay()
        end_of_step(slot)
        counter[0] += 1

    for t in range(args.warmup):
        replay()
    torch.cuda.synchronize()
    sampler = start_clock_sampler(torch, dev) if rank == 0 or world == 1 else None
    time.sleep(0.6)  # let the sampler start before the timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for t in range(args.steps):
        replay()
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = stop_clock_sampler(sampler)
    ms = start.elapsed_time(end)
    ms_t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(ms_t, op=dist.ReduceOp.MAX)
    ms_max = float(ms_t.item())
    status = F.fp8_get_device_status()

    # variants of the step, each with its own graphs, warm-up and timed replays, reported beside
    # the headline: the other composition of the same numbers, and the mixed-format backward
    def time_variant(mixed_v, path_v):
        run_step(lins, counter[0] % HIST, mixed=mixed_v, path=path_v)
        end_of_step(counter[0] % HIST)
        counter[0] += 1
        torch.cuda.synchronize()
        vgraphs = []
        for slot in range(HIST):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                run_step(lins, slot, mixed=mixed_v, path=path_v)
            vgraphs.append(g)
        torch.cuda.synchronize()
        for t in range(args.warmup):
            vgraphs[counter[0] % HIST].replay()
            end_of_step(counter[0] % HIST)
            counter[0] += 1
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        vsteps = max(3, args.steps // 2)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for t in range(vsteps):
            vgraphs[counter[0] % HIST].replay()
            end_of_step(counter[0] % HIST)
            counter[0] += 1
        s1.record()
        torch.cuda.synchronize()
        vt = torch.tensor([s0.elapsed_time(s1)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(vt, op=dist.ReduceOp.MAX)
        vms = float(vt.item())
        del vgraphs
        return {"ms_per_step": vms / vsteps, "value": flops_step * vsteps * world / (vms * 1e-3) / 1e12,
                "unit": UNIT, "steps": vsteps, "device_status": F.fp8_get_device_status()}

    variants = {}
    if not args.no_variants:
        for other in PATHS:
            if other == args.path:
                continue
            v = time_variant(False, other)
            v["quantize_bytes_per_step"] = sum(quant_bytes_of(l, other) for l in lins)
            v["what"] = PATH_WHAT[other] + " (the same numbers as the headline step)"
            variants[f"path_{other}"] = v
        v = time_variant(True, None)
        v["quantize_bytes_per_step"] = sum(l.quant_bytes_mixed for l in lins)
        v["what"] = ("forward keeps its E4M3 x8 / w8; backward quantizes only g (E5M2, row-major + column sums) "
                     "and reads x8 / w8 in place (mixed-format GEMMs); not the pages' HYBRID numerics")
        variants["mixed_backward"] = v

    # per-kernel durations: the same step captured again with the library's profiler on
    # (an event-record node on each side of every kernel), each of the 16 slot graphs
    # replayed once, then every event pair read back
    F.fp8_profiler_read(0), F.fp8_profiler_read(1), F.fp8_profiler_read(2)
    F.fp8_profiler_enable(True)
    timed_graphs = []
    for slot in range(HIST):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            run_step(lins, slot)
        timed_graphs.append(g)
    F.fp8_profiler_enable(False)
    for t in range(HIST):
        timed_graphs[counter[0] % HIST].replay()
        end_of_step(counter[0] % HIST)
        counter[0] += 1
    torch.cuda.synchronize()
    n_instr = HIST
    q_ms, q_n, q_bytes = F.fp8_profiler_read(0)
    gp_ms, gp_n, gp_flops = F.fp8_profiler_read(3)  # GEMM launches on CTA-pair tiles
    gs_ms, gs_n, gs_flops = F.fp8_profiler_read(4)  # GEMM launches on single-CTA tiles
    o_ms, o_n, _ = F.fp8_profiler_read(2)
    g_ms, g_n, g_flops = gp_ms + gs_ms, gp_n + gs_n, gp_flops + gs_flops
    launches_per_step = (q_n + g_n + o_n) / n_instr

    # end to end through the public API: every step's activations and gradients copied in from
    # pinned host memory and its bias gradients and used steps read back.  The inputs are double
    # buffered: while step t runs on one device copy of every x and g, a copy stream brings step
    # t+1's into the other (the copies of every step stay inside the timed region).
    e2e = None
    if not args.no_e2e:
        sets = [[(l.x, l.g) for l in lins], [(torch.empty_like(l.x), torch.empty_like(l.g)) for l in lins]]

        def bind(si):
            for l, (x, g) in zip(lins, sets[si]):
                l.x, l.g = x, g

        bind(1)
        graphs_b = []
        for slot in range(HIST):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                run_step(lins, slot)
            graphs_b.append(g)
        bind(0)
        gsets = [graphs, graphs_b]
        host_in = [(torch.empty_like(l.x, device="cpu").pin_memory(), torch.empty_like(l.g, device="cpu").pin_memory())
                   for l in lins]
        for (hx, hg), l in zip(host_in, lins):
            hx.copy_(l.x)
            hg.copy_(l.g)
        host_out = [(l.gb, torch.empty_like(l.gb, device="cpu").pin_memory(), l.steps,
                     torch.empty_like(l.steps, device="cpu").pin_memory()) for l in lins]
        h2d = sum(l.x.numel() * 2 + l.g.numel() * 2 for l in lins)
        d2h = sum(l.gb.numel() * 2 + l.steps.numel() * 4 for l in lins)
        comp = torch.cuda.current_stream()
        copy_stream = torch.cuda.Stream()
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        freed = [torch.cuda.Event(), torch.cuda.Event()]

        def copy_in(si):
            with torch.cuda.stream(copy_stream):
                for (dx, dg), (hx, hg) in zip(sets[si], host_in):
                    dx.copy_(hx, non_blocking=True)
                    dg.copy_(hg, non_blocking=True)
            copied[si].record(copy_stream)

        def run_e2e(nsteps):
            begin = torch.cuda.Event()
            begin.record(comp)
            copy_stream.wait_event(begin)
            copy_in(0)
            for t in range(nsteps):
                si = t % 2
                if t + 1 < nsteps:
                    if t >= 1:
                        copy_stream.wait_event(freed[1 - si])  # step t-1 is done with that copy
                    copy_in(1 - si)
                comp.wait_event(copied[si])
                slot = counter[0] % HIST
                gsets[si][slot].replay()
                end_of_step(slot)
                counter[0] += 1
                freed[si].record(comp)
                for dgb, hgb, dst, hst in host_out:
                    hgb.copy_(dgb, non_blocking=True)
                    hst.copy_(dst, non_blocking=True)

        run_e2e(4)  # warm-up of both graph sets
        torch.cuda.synchronize()
        e2e_steps = max(3, min(args.steps, 40))
        if world > 1:
            dist.barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        run_e2e(e2e_steps)
        e2.record()
        torch.cuda.synchronize()
        e_ms = torch.tensor([s2.elapsed_time(e2)], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(e_ms, op=dist.ReduceOp.MAX)
        e2e = {"value": flops_step * e2e_steps * world / (float(e_ms.item()) * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
               "overlap": "inputs double-buffered: step t+1's host-to-device copies run beside step t"}
        del gsets, graphs_b

    if world > 1:
        dist.barrier()
    del graphs, timed_graphs
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = measured_peaks()
    # fp8 dense = 2 x bf16 (nominal 4.5 / 2.25 PF); the burst figure, since the timed region is
    # well under a second and runs at full clock (the sustained one is for seconds-long loops)
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    tflops = lambda fl, ms: fl / (ms * 1e-3) / 1e12 if ms > 0 else 0.0  # noqa: E731
    gemm_tflops = tflops(g_flops, g_ms)
    pair_tflops, single_tflops = tflops(gp_flops, gp_ms), tflops(gs_flops, gs_ms)
    quant_gbs = q_bytes / (q_ms * 1e-3) / 1e9 if q_ms > 0 else 0.0
    traffic = gemm_traffic_per_launch()
    value = flops_step * args.steps * world / (ms_max * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers": W.TRAINING_LAYERS, "tokens": W.TRAINING_TOKENS,
                   "linears_kn": [list(kn) for kn in W.TRAINING_LINEARS],
                   "l2": "inputs larger than L2: every layer has its own x, w, g (about 3 GB working set)",
                   "graphs": f"one CUDA graph per history slot ({HIST})",
                   "path": PATH_WHAT[args.path],
                   "parallelism": (f"data parallel over {world} GPU(s): each rank its own batch, one all-reduce "
                                   f"(MAX) of every ring's amax per step" if use_dp else "single GPU")},
        "gemm_flops_per_step": flops_step, "quantize_bytes_per_step": qbytes_step,
        "kernels": {"gemm_tflops": gemm_tflops, "gemm_ms_per_step": g_ms / n_instr,
                    "gemm_pair": {"launches_per_step": gp_n / n_instr, "us_per_launch": 1e3 * gp_ms / max(gp_n, 1),
                                  "gflop_per_launch": gp_flops / max(gp_n, 1) / 1e9, "tflops": pair_tflops,
                                  "frac": pair_tflops / fp8_peak},
                    "gemm_single_cta": {"launches_per_step": gs_n / n_instr,
                                        "us_per_launch": 1e3 * gs_ms / max(gs_n, 1),
                                        "gflop_per_launch": gs_flops / max(gs_n, 1) / 1e9, "tflops": single_tflops,
                                        "frac": single_tflops / fp8_peak},
                    "quantize_gbs": quant_gbs, "quantize_ms_per_step": q_ms / n_instr,
                    "other_ms_per_step": o_ms / n_instr,
                    "quantize_frac_of_hbm": quant_gbs / peaks["hbm_gbs"],
                    "timing": "CUDA events around every library launch in an instrumented replay of the step "
                              "(the event nodes stop each launch from overlapping its predecessor, so these "
                              "are per-launch durations including the prologue)"},
        "roofline": {"bound": "tensor", "kernel": "fp8_gemm_kernel, 256 x 256 tiles on CTA pairs (the step's "
                                                  "dominant launches: forward N >= 3072 and every dX + dW)",
                     "achieved": pair_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": pair_tflops / fp8_peak,
                     "traffic": traffic,
                     "peak_note": f"fp8 dense = 2 x {peaks['source']} burst bf16 ({peaks['bf16_tflops']} "
                                  f"TFLOP/s), of {peaks['source']}: the timed region is {ms_max / 1e3:.3f} s"},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "device_status": status,
    }
    if clocks:
        line["clocks"] = clocks
    if variants:
        line["variants"] = variants
    if e2e:
        line["e2e"] = e2e
    if world == 1 and not args.no_sweeps:
        line["sweeps"] = run_sweeps(F, W, torch, dev)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
