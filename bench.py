#!/usr/bin/env python
"""Benchmark of the batched Shampoo preconditioner inverse root on one B200.

Workload (one "step"): A^(-1/4) of 64 SPD blocks of 1024 x 1024, each
Q diag(lambda) Q^T with lambda log-uniform on [1e-6, 1] (cond 1e6), by two
coupled Newton-Schulz passes with PRISM alpha (d = 2, Gaussian sketch p = 8,
alpha in [3/8, 1], residual tol 1e-3 per pass), on the fp64-grade path:
fp64 iterates, every product by the Ozaki scheme on the int8 tensor cores
(five digit slices per operand, exact int32 accumulation).  fp32 storage
cannot hold this spectrum: TF32 rounding of A/||A||_F makes the blocks
indefinite and the 3xTF32 split ends about 4e-2 from eigh; both are reported
beside the headline as context.

Metric: algorithmic TFLOP/s (2 n^3 per n x n product actually executed,
summed over blocks) and preconditioners/s, with the fraction of the int8
tensor peak that the dominant kernel reaches (15 int8 digit products per
fp64-grade product).  Under torchrun each rank runs its own independent batch
(replicas, weak scaling); the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "inv-root/polar TFLOP/s & preconditioners/s at 1024², % of B200 tensor peak"
N, BATCH, LAM_LO, D, P, TOL, MAX_ITER = 1024, 64, 1e-6, 2, 8, 1e-3, 24
SEED_A, SEED_S = 103, 1003
PREC = "ozaki"
OZ_SLICES = 5
OZ_PRODUCTS = OZ_SLICES * (OZ_SLICES + 1) // 2  # int8 digit products per fp64-grade product
# blocks whose accuracy the bench reports (the two where the float64 oracle,
# stopped at residual 1e-3 per pass, is farthest from eigh, and two others)
ACC_BLOCKS = (0, 5, 37, 63)
# tensor peak ratios (nominal dense), used only where a peak is not measured
TF32_OVER_BF16 = 1.1 / 2.25
# dram__bytes_read.sum + dram__bytes_write.sum of one 3xTF32 persistent GEMM
# launch (64 x 1024^3): an ncu capture of 16 blocks scaled x4 by the blocks
GEMM_TRAFFIC_PER_LAUNCH = 4 * (290.093e6 + 43.367e6)
# ... of one k_gemm_oz launch with the accumulate (C <- C + A B) epilogue,
# 64 x 1024^3: an ncu capture of 16 products (302.37 MB read, 93.54 MB
# written) scaled x4 by the products
OZ_GEMM_TRAFFIC_PER_LAUNCH = 4 * (302.37e6 + 93.54e6)
# dram__bytes_read.sum + dram__bytes_write.sum of one k_sketch_tma<8> launch
# over 48 x 1024^2 (201.393 MB read, 4.646 MB written), scaled x 64/48 by the
# rows processed and x 5 for the passes of one alpha fit (d = 2)
SKETCH_TRAFFIC_PER_FIT = 5 * 64 / 48 * (201.393e6 + 4.646e6)


def workload_config(world):
    return {
        "workload": f"inv4_root_{BATCH}x1024sq_spd_cond1e6_prism_d2_p8",
        "n": N, "batch_per_gpu": BATCH, "d": D, "p": P, "tol": TOL, "max_iter": MAX_ITER,
        "alpha_interval": [0.375, 1.0], "prec": "ozaki (fp64 iterates, int8 x5 digit products)",
        "lambda": "log-uniform [1e-6, 1]",
        "l2": "inputs larger than L2 (256 MiB of A plus 4.6 GB of iterates and slices per GPU)",
        "parallelism": f"replicas x{world}",
    }


def gemm_count(iters):
    """Products of one block: pass with k updates costs 4k - 1 (d = 2)."""
    return sum(max(4 * int(k) - 1, 0) for k in iters)


def pass_flops(k, n):
    """Algorithmic flops of one coupled pass with k updates (d = 2): 4k - 1
    full n x n x n products (2n^3 each).  Z_k Y_k, R_k^2 and the updates are
    symmetric only in exact arithmetic and are formed in full."""
    return gemm_count([k]) * 2.0 * n ** 3


def block_flops(iters, n):
    return sum(pass_flops(k, n) for k in iters)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def measure_tensor_peaks(dev):
    """Burst tensor-core peaks of this GPU, measured the way the BF16 figure
    of MEASURED_PEAKS.json is: the best of 10 library GEMMs of 8192^3 (cuBLAS
    through torch) in TF32 (fp32 inputs, TF32 allowed), BF16, and int8
    (int32 accumulation)."""
    import torch
    n = 8192

    def best(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        t = 1e9
        for _ in range(10):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            t = min(t, e0.elapsed_time(e1))
        return 2.0 * n ** 3 / (t / 1e3) / 1e12

    g = torch.Generator(device=dev).manual_seed(1)
    a = torch.randn(n, n, device=dev, generator=g)
    b = torch.randn(n, n, device=dev, generator=g)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    tf32 = best(lambda: a @ b)
    torch.backends.cuda.matmul.allow_tf32 = prev
    ab, bb = a.bfloat16(), b.bfloat16()
    bf16 = best(lambda: ab @ bb)
    ai = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8, generator=g)
    bi = torch.randint(-127, 128, (n, n), device=dev, dtype=torch.int8, generator=g).t().contiguous().t()
    i8 = best(lambda: torch._int_mm(ai, bi))
    del a, b, ab, bb, ai, bi
    torch.cuda.empty_cache()
    return {"tf32_tflops": tf32, "bf16_tflops": bf16, "int8_tops": i8,
            "how": "best of 10 cuBLAS 8192^3 GEMMs via torch (burst)"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_timing(local_ms, local_units, local_flops, local_launches, world):
    """Max over ranks of the time, sums of the work.  Works with any
    initialised process group (nccl on the GPUs, gloo in the CPU tests)."""
    if world == 1:
        return local_ms, local_units, local_flops, local_launches
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([local_ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    s = torch.tensor([local_units, local_flops, local_launches], dtype=torch.float64, device=dev)
    dist.all_reduce(s, op=dist.ReduceOp.SUM)
    return float(t.item()), float(s[0].item()), float(s[1].item()), int(s[2].item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ oracle leg
def oracle_sample(A_block, S_np, seconds_hint=None):
    """Time the float64 oracle on one block; returns (seconds, flops)."""
    from oracle import prism_ref as o
    opts = o.PrismOpts(d=D, p=P, lo=0.375, hi=1.0, tol=TOL, max_iter=MAX_ITER)
    t0 = time.perf_counter()
    _, infos = o.inv_root_ref(A_block, o.POW_INV4, opts, S_np)
    dt = time.perf_counter() - t0
    return dt, block_flops([i.iters for i in infos], N)


def eigh_sample(A_block):
    """Time the eigendecomposition route to A^(-1/4) (float64 LAPACK eigh) on
    one block: the direct method the iteration replaces; returns seconds."""
    from oracle import prism_ref as o
    t0 = time.perf_counter()
    o.spd_power_eigh(A_block, -0.25)
    return time.perf_counter() - t0


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    from second_order_optimizer_shampoo_b200 import synth
    S_np = synth.sketch_stack(2 * MAX_ITER, N, P, SEED_S)
    blocks = [synth.spd_block(N, LAM_LO, 1.0, SEED_A, i) for i in range(max(1, args.steps + args.warmup))]
    for i in range(args.warmup):
        oracle_sample(blocks[i], S_np)
    tot_t, tot_f = 0.0, 0.0
    for i in range(args.steps):
        t, f = oracle_sample(blocks[args.warmup + i], S_np)
        tot_t += t
        tot_f += f
    value = tot_f / tot_t / 1e12
    cores = os.cpu_count()
    t_eigh = eigh_sample(blocks[0])
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "one 1024x1024 block of the 64-block batch per step "
                                   "(float64 NumPy/LAPACK oracle, same recurrence and sketch)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "eigh_reference": {"ms_per_block": 1e3 * t_eigh, "cores": cores,
                           "kind": "float64 LAPACK eigh route to A^(-1/4), one 1024x1024 block"},
    }
    print(json.dumps(line))
    return 0


def step_only(args):
    """One config-3 step alone (profiling aid): --batch blocks of 1024^2 at
    cond 1e6, every kernel launched from the host loop so that profilers see
    each launch; --prec selects the product path."""
    import torch

    from second_order_optimizer_shampoo_b200 import prism, synth
    dev = torch.device("cuda", 0)
    A = torch.from_numpy(synth.spd_batch(N, args.batch, LAM_LO, 1.0, SEED_A)).to(dev)
    S = torch.from_numpy(synth.sketch_stack(2 * MAX_ITER, N, P, SEED_S)).to(dev)
    opts = prism.make_opts(d=D, p=P, tol=TOL, max_iter=MAX_ITER, prec=args.prec, host_loop=True)
    X = torch.empty_like(A)
    rep = prism.make_report(args.batch, MAX_ITER, dev)
    for _ in range(max(args.warmup, 1) + args.steps):
        prism.matfn_inv_root(A, "inv4", opts, S, out=X, report=rep)
    torch.cuda.synchronize()
    ok = int((rep["status"].cpu().numpy() == 0).sum())
    print(json.dumps({"kernel": "step", "prec": args.prec, "batch": args.batch, "status_ok": ok,
                      "iters": rep["iters"].cpu().numpy()[0].tolist()}))
    return 0


def ozgemm_only(args):
    """The Ozaki-scheme GEMM alone (profiling aid), as the bench's roofline
    times it: --batch products of 1024^2 fp64 matrices through
    shp_matmul_f64; the first call slices both operands, every later one
    reuses the slices and accumulates (C <- C + A B, the step's epilogue), so
    it is one k_gemm_oz launch."""
    import torch

    from second_order_optimizer_shampoo_b200 import _abi, prism
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(5)
    X = torch.randn(args.batch, N, N, device=dev, generator=g, dtype=torch.float64)
    Y = torch.randn(args.batch, N, N, device=dev, generator=g, dtype=torch.float64)
    out = torch.zeros_like(X)
    ws = torch.empty(int(_abi.lib().shp_matmul_f64_workspace_bytes(N, N, N, args.batch)),
                     dtype=torch.uint8, device=dev)
    prism.shp_matmul_f64(X, Y, out=out, ws=ws)
    for _ in range(max(args.warmup, 1)):
        prism.shp_matmul_f64(X, Y, out=out, ws=ws, reuse_a=True, reuse_b=True, accumulate=True)
    stream = torch.cuda.current_stream()
    ms = _time(lambda: prism.shp_matmul_f64(X, Y, out=out, ws=ws, reuse_a=True, reuse_b=True,
                                            accumulate=True), stream, args.steps)
    flops = 2.0 * args.batch * N ** 3
    print(json.dumps({"kernel": "ozgemm", "batch": args.batch, "ms_per_launch": ms,
                      "fp64_tflops": flops / (ms / 1e3) / 1e12,
                      "int8_tops": 15 * flops / (ms / 1e3) / 1e12,
                      "launches": args.steps + max(args.warmup, 1)}))
    return 0


def gemm_only(args):
    """The dominant kernel alone: batched 1024^3 3xTF32 products (profiling aid)."""
    import torch

    from second_order_optimizer_shampoo_b200 import prism
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(5)
    X = torch.randn(args.batch, N, N, device=dev, generator=g)
    Y = torch.randn(args.batch, N, N, device=dev, generator=g)
    Xh, Xl = prism.shp_split_tf32(X)
    Yh, Yl = prism.shp_split_tf32(Y)
    out = torch.empty_like(X)
    for _ in range(max(args.warmup, 1) + args.steps):
        prism.shp_matmul(Xh, Yh, "3xtf32", A_lo=Xl, B_lo=Yl, out=out)
    torch.cuda.synchronize()
    print(json.dumps({"kernel": "gemm", "batch": args.batch, "launches": args.steps + max(args.warmup, 1)}))
    return 0


SB_N, SB_BATCH, SB_P, SB_MAX_ITER = 64, 16384, 4, 50
FP32_LANES_PER_SM, SMS = 128, 148
# dram__bytes_read.sum + dram__bytes_write.sum of one full-size small-block
# launch (16384 x 64^2, ncu capture of the current kernel)
SMALL_TRAFFIC_PER_LAUNCH = 276.44e6 + 238.29e6


def small_block_leg(args, dev, stream, sm_max_mhz):
    """Many small blocks: 16384 independent 64 x 64 SPD blocks (lambda
    log-uniform on [1e-3, 1]), A^(-1/4) by PRISM d = 1, p = 4, tol 1e-6, one
    CTA per block iterating on chip (products and sketch powers on the
    tensor cores, 3xTF32 warp-level MMA).  The block's iteration is a chain of
    dependent steps and block barriers, so the figure is latency-bound; the
    fraction is given against the 3xTF32 tensor rate and, for continuity, the
    fp32 FMA rate."""
    import torch

    from second_order_optimizer_shampoo_b200 import _abi, prism, synth
    A = torch.from_numpy(synth.spd_batch(SB_N, SB_BATCH, 1e-3, 1.0, 101)).to(dev)
    S = torch.from_numpy(synth.sketch_stack(2 * SB_MAX_ITER, SB_N, SB_P, 1001)).to(dev)
    opts = prism.make_opts(d=1, p=SB_P, lo=0.5, tol=1e-6, max_iter=SB_MAX_ITER, prec="3xtf32")
    ws = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, SB_N, SB_N, SB_BATCH, opts),
                     dtype=torch.uint8, device=dev)
    X = torch.empty_like(A)
    rep = prism.make_report(SB_BATCH, SB_MAX_ITER, dev)
    for _ in range(3):
        prism.matfn_inv_root(A, "inv4", opts, S, out=X, ws=ws, report=rep)
    torch.cuda.synchronize()
    iters = rep["iters"].cpu().numpy()
    ok = int((rep["status"].cpu().numpy() == 0).sum())
    products = float(sum(max(3 * int(k) - 1, 0) for blk in iters for k in blk))  # d = 1
    flops = products * 2.0 * SB_N ** 3
    reps = 10
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        prism.matfn_inv_root(A, "inv4", opts, S, out=X, ws=ws, report=rep)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    # compulsory HBM bytes: the block in, the root out (the sketch slices are
    # shared by the batch and stay in L2)
    hbm_bytes = SB_BATCH * 2 * SB_N * SB_N * 4
    peaks, _ = load_peaks()
    tf = flops / (ms / 1e3) / 1e12
    fma_peak = SMS * FP32_LANES_PER_SM * 2 * sm_max_mhz * 1e6 / 1e12
    tf32 = peaks.get("tf32_tflops", peaks["bf16_tflops"] * TF32_OVER_BF16)
    return {"workload": "inv4_root_16384x64sq_spd_cond1e3_prism_d1_p4_tol1e-6_onchip",
            "ms_per_call": ms, "roots_per_s": SB_BATCH / (ms / 1e3), "value": tf,
            "unit": "TFLOP/s", "products": products, "status_ok": ok,
            "median_iters_per_pass": [int(x) for x in np.median(iters, axis=0)],
            "hbm_gbs": hbm_bytes / (ms / 1e3) / 1e9, "hbm_peak_gbs": peaks["hbm_gbs"],
            "fma_frac": tf / fma_peak,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": tf32 / 3, "unit": "TFLOP/s",
                         "frac": tf / (tf32 / 3), "traffic": SMALL_TRAFFIC_PER_LAUNCH,
                         "traffic_unit": "bytes per launch", "algorithmic_bytes": hbm_bytes,
                         "peak_note": "3xTF32 products: the measured TF32 peak / 3; the "
                                      "iteration is latency-bound (a chain of dependent steps "
                                      "per block), fma_frac against the fp32 FMA rate "
                                      f"({SMS} SMs x {FP32_LANES_PER_SM} lanes x 2 flop x "
                                      f"{sm_max_mhz:.0f} MHz)"}}


def small_only(args):
    """The small-block kernel alone (profiling aid): --batch blocks of 64 x 64."""
    import torch

    from second_order_optimizer_shampoo_b200 import prism, synth
    dev = torch.device("cuda", 0)
    batch = args.batch if args.batch != BATCH else SB_BATCH
    A = torch.from_numpy(synth.spd_batch(SB_N, batch, 1e-3, 1.0, 101)).to(dev)
    S = torch.from_numpy(synth.sketch_stack(2 * SB_MAX_ITER, SB_N, SB_P, 1001)).to(dev)
    opts = prism.make_opts(d=1, p=SB_P, lo=0.5, tol=1e-6, max_iter=SB_MAX_ITER, prec="3xtf32")
    X = torch.empty_like(A)
    rep = prism.make_report(batch, SB_MAX_ITER, dev)
    for _ in range(max(args.warmup, 1)):
        prism.matfn_inv_root(A, "inv4", opts, S, out=X, report=rep)
    ms = _time(lambda: prism.matfn_inv_root(A, "inv4", opts, S, out=X, report=rep),
               torch.cuda.current_stream(), args.steps)
    ok = int((rep["status"].cpu().numpy() == 0).sum())
    print(json.dumps({"kernel": "small", "batch": batch, "status_ok": ok, "ms_per_call": ms,
                      "roots_per_s": batch / (ms / 1e3),
                      "iters": rep["iters"].cpu().numpy()[0].tolist(),
                      "launches": args.steps + max(args.warmup, 1)}))
    return 0


def _time(fn, stream, reps):
    import torch
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def shampoo_only(args):
    """One config-2 Shampoo step alone (profiling aid), the inverse roots
    with the host loop so that profilers see each launch."""
    import torch
    dev = torch.device("cuda", 0)
    out = shampoo_step_leg(args, dev, torch.cuda.current_stream(), host_loop=True,
                           reps=args.steps)
    print(json.dumps({"kernel": "shampoo", "ms_per_step": out["ms_per_step"]}))
    return 0


def shampoo_step_leg(args, dev, stream, host_loop=False, reps=10):
    """One Shampoo step on a 1024 x 1024 weight: 10 EMA steps of L and R with
    fresh G (TF32), L^(-1/4) and R^(-1/4) by PRISM (d = 2, p = 8, tol 1e-3,
    TF32) as one batch of two, and W -= 1e-3 L^(-1/4) G R^(-1/4).  The ten
    gradients are all given, so the EMA steps go through one
    shampoo_gram_ema_steps call; the ten one-step calls are timed beside it."""
    import torch

    from second_order_optimizer_shampoo_b200 import _abi, prism, synth
    n, beta, eps, lr, mi = 1024, 0.95, 1e-6, 1e-3, 30
    W0 = torch.from_numpy(synth.gaussian((1, n, n), 0.02, 102, index=0)).to(dev)
    Gs = [torch.from_numpy(synth.gaussian((1, n, n), 0.02, 102, index=t + 1)).to(dev)
          for t in range(10)]
    S = torch.from_numpy(synth.sketch_stack(2 * mi, n, 8, 1002)).to(dev)
    opts = prism.make_opts(d=2, p=8, tol=1e-3, max_iter=mi, prec="tf32", host_loop=host_loop)
    LR = torch.zeros(2, n, n, device=dev)
    W = W0.clone()
    roots = torch.empty_like(LR)
    rep = prism.make_report(2, mi, dev)
    ws = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, n, n, 2, opts),
                     dtype=torch.uint8, device=dev)
    eye = torch.eye(n, device=dev) * eps
    Gst = torch.stack(Gs)  # [10][1][n][n]
    ws_ema = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_GRAM_EMA_STEPS, n, n, 10,
                                                   prism.make_opts(prec="tf32")),
                         dtype=torch.uint8, device=dev)

    def ema_steps():
        prism.shampoo_gram_ema_steps(Gst, LR[0:1], LR[1:2], beta, eps, "tf32", ws=ws_ema)

    ws_one = torch.empty(max(prism.shp_workspace_bytes(_abi.SHP_OP_GRAM_EMA, n, n, 1,
                                                       prism.make_opts(prec="tf32")), 16),
                         dtype=torch.uint8, device=dev)

    def ema_one_step_calls():
        for G in Gs:
            prism.shampoo_gram_ema(G, LR[0:1], LR[1:2], beta, eps, "tf32", ws=ws_one)

    def step():
        LR.copy_(eye.expand(2, n, n))
        W.copy_(W0)
        ema_steps()
        prism.matfn_inv_root(LR, "inv4", opts, S, out=roots, ws=ws, report=rep)
        prism.shampoo_apply(W, Gs[-1], roots[0:1], roots[1:2], lr, "tf32")

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    iters = rep["iters"].cpu().numpy()
    ms = _time(step, stream, reps)
    ms_ema_steps = _time(ema_steps, stream, reps)
    ms_ema_calls = _time(ema_one_step_calls, stream, reps)
    flops = 10 * 2 * n * (n + 1) * n + sum(block_flops(blk, n) for blk in iters) + 2 * 2.0 * n ** 3
    return {"workload": "shampoo_step_1024sq_ema10_inv4_d2_p8_tf32_apply", "ms_per_step": ms,
            "value": flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s",
            "preconditioners_per_s": 2 / (ms / 1e3),
            "ema10_steps_call_ms": ms_ema_steps, "ema10_one_step_calls_ms": ms_ema_calls,
            "iters_per_pass": [[int(k) for k in blk] for blk in iters],
            "status": [int(x) for x in rep["status"].cpu().numpy()],
            "note": "EMA products counted n(n+1)n (symmetric results, formed on their "
                    "upper-triangle tiles); inverse-root products and the apply at 2n^3"}


def gemm_count_leg(args, dev, stream, A):
    """GEMMs to residual 1e-3 per pass on the config-3 batch (the headline
    path): PRISM d = 2 against the fixed-coefficient (Taylor) iterations
    d = 2 and d = 1."""
    import torch

    from second_order_optimizer_shampoo_b200 import prism, synth
    mi = 40
    S = torch.from_numpy(synth.sketch_stack(2 * mi, N, P, SEED_S)).to(dev)
    out = {}
    for name, d, fixed in (("prism_d2", 2, False), ("taylor_d2", 2, True),
                           ("taylor_d1", 1, True)):
        opts = prism.make_opts(d=d, p=P, tol=TOL, max_iter=mi, prec=PREC, fixed_alpha=fixed)
        X, rep = prism.matfn_inv_root(A, "inv4", opts, S)
        torch.cuda.synchronize()
        it = rep["iters"].cpu().numpy()
        per = (3 if d == 1 else 4)
        counts = [sum(max(per * int(k) - 1, 0) for k in blk) for blk in it]
        out[name] = {"median_iters_per_pass": [int(x) for x in np.median(it, axis=0)],
                     "median_gemms_per_block": float(np.median(counts)),
                     "status_ok": int((rep["status"].cpu().numpy() == 0).sum())}
    return out


SWEEP_SIGMA_MIN = (1e-1, 1e-2, 1e-3, 1e-4)


def sigma_sweep_leg(args, dev, stream):
    """Polar factor of 8 matrices 1024 x 1024 with singular values log-uniform
    on [sigma_min, 1], to ||I - X^T X||_F / sqrt(n) <= 1e-6 (split path):
    iterations and GEMMs of PRISM d = 2 against the fixed-coefficient d = 2
    and d = 1 iterations, per sigma_min."""
    import torch

    from second_order_optimizer_shampoo_b200 import prism, synth
    n, batch, mi = 1024, 8, 60
    S = torch.from_numpy(synth.sketch_stack(mi, n, 8, 1006)).to(dev)
    out = {"workload": "polar_8x1024sq_sigma_min_sweep_tol1e-6_3xtf32", "rows": []}
    for smin in SWEEP_SIGMA_MIN:
        G = torch.from_numpy(synth.singular_spectrum(n, n, smin, batch, 106)).to(dev)
        row = {"sigma_min": smin}
        for name, d, fixed in (("prism_d2", 2, False), ("taylor_d2", 2, True),
                               ("taylor_d1", 1, True)):
            opts = prism.make_opts(d=d, p=8, tol=1e-6, max_iter=mi, prec="3xtf32",
                                   fixed_alpha=fixed)
            _, rep = prism.matfn_polar(G, opts, S)
            torch.cuda.synchronize()
            it = rep["iters"][:, 0].cpu().numpy()
            # per update: X^T X, R R (d = 2 only), X Delta; plus the final residual
            gem = [int(k) * (2 if d == 1 else 3) + 1 for k in it]
            row[name] = {"median_iters": float(np.median(it)),
                         "median_gemms": float(np.median(gem)),
                         "status_ok": int((rep["status"].cpu().numpy() == 0).sum())}
        out["rows"].append(row)
    return out


def single_block_leg(args, dev, stream):
    """Config 1 as single calls: one 64 x 64 A^(-1/4) (d = 1, p = 4, tol 1e-6)
    and one 64 x 32 polar factor, microseconds per call."""
    import torch

    from second_order_optimizer_shampoo_b200 import _abi, prism, synth
    A = torch.from_numpy(synth.spd_batch(64, 1, 1e-3, 1.0, 101)).to(dev)
    S = torch.from_numpy(synth.sketch_stack(100, 64, 4, 1001)).to(dev)
    opts = prism.make_opts(d=1, p=4, lo=0.5, tol=1e-6, max_iter=50, prec="3xtf32")
    X = torch.empty_like(A)
    rep = prism.make_report(1, 50, dev)
    ws = torch.empty(256, dtype=torch.uint8, device=dev)
    G = torch.from_numpy(synth.gaussian((1, 64, 32), 1.0, 101)).to(dev)
    Sp = torch.from_numpy(synth.sketch_stack(50, 32, 4, 1001)).to(dev)
    Xp = torch.empty_like(G)
    repp = prism.make_report(1, 50, dev)

    def root():
        prism.matfn_inv_root(A, "inv4", opts, S, out=X, ws=ws, report=rep)

    def polar():
        prism.matfn_polar(G, opts, Sp, out=Xp, ws=ws, report=repp)

    for _ in range(5):
        root()
        polar()
    torch.cuda.synchronize()
    return {"workload": "inv4_root_64sq_cond1e3_d1_p4_tol1e-6 + polar_64x32_d1_p4",
            "us_per_inv_root": 1e3 * _time(root, stream, 50),
            "us_per_polar": 1e3 * _time(polar, stream, 50),
            "iters_inv_root": [int(k) for k in rep["iters"].cpu().numpy()[0]],
            "iters_polar": int(repp["iters"].cpu().numpy()[0][0])}


def large_sqrt_leg(args, dev, stream):
    """A^(1/2) of one 10240 x 10240 Marchenko-Pastur matrix (A = X X^T / 20480 +
    1e-4 I), PRISM d = 2, p = 16, tol 1e-6, on the fp64-grade path (the one
    that reaches 1e-5 against eigh at this size); GEMMs to the residual
    against the fixed-coefficient iterations d = 2 and d = 1; the 3xTF32
    split timed beside it."""
    import torch

    from second_order_optimizer_shampoo_b200 import _abi, prism, synth
    n, mi = 10240, 40
    A = torch.from_numpy(synth.mp_spd(n, 2 * n, 1e-4, 105)[None]).to(dev)
    S = torch.from_numpy(synth.sketch_stack(mi, n, 16, 1005)).to(dev)
    out = {"workload": "sqrt_10240sq_marchenko_pastur_prism_d2_p16_tol1e-6_ozaki"}
    for name, d, fixed, pr in (("prism_d2", 2, False, "ozaki"), ("taylor_d2", 2, True, "ozaki"),
                               ("taylor_d1", 1, True, "ozaki"), ("prism_d2_3xtf32", 2, False, "3xtf32")):
        opts = prism.make_opts(d=d, p=16, tol=1e-6, max_iter=mi, prec=pr, fixed_alpha=fixed)
        ws = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, n, n, 1, opts),
                         dtype=torch.uint8, device=dev)
        X = torch.empty_like(A)
        rep = prism.make_report(1, mi, dev)

        def call():
            prism.matfn_inv_root(A, "sqrt", opts, S, out=X, ws=ws, report=rep)

        call()
        torch.cuda.synchronize()
        k = int(rep["iters"].cpu().numpy()[0][0])
        gemms = max((3 if d == 1 else 4) * k - 1, 0)
        entry = {"iters": k, "gemms": gemms, "status": int(rep["status"].cpu().numpy()[0])}
        if not fixed:
            ms = _time(call, stream, 3)
            tf = gemms * 2.0 * n ** 3 / (ms / 1e3) / 1e12
            entry.update({"ms": ms, "value": tf, "unit": "TFLOP/s"})
        out[name] = entry
        del ws, X
        torch.cuda.empty_cache()
    return out


def tf32_batched_leg(args, dev, stream, tp):
    """The TF32 path where it applies: 64 SPD blocks 1024^2 in the Shampoo
    statistics regime (lambda log-uniform on [1e-2, 1], cond 1e2), A^(-1/4),
    d = 2, p = 8, tol 1e-3, against the measured TF32 tensor peak; accuracy
    of two blocks against eigh."""
    import torch

    from oracle import prism_ref as o
    from second_order_optimizer_shampoo_b200 import _abi, prism, synth
    mi = 30
    A_np = synth.spd_batch(N, BATCH, 1e-2, 1.0, 107)
    A = torch.from_numpy(A_np).to(dev)
    S = torch.from_numpy(synth.sketch_stack(2 * mi, N, P, 1007)).to(dev)
    opts = prism.make_opts(d=D, p=P, tol=1e-3, max_iter=mi, prec="tf32")
    ws = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, N, N, BATCH, opts),
                     dtype=torch.uint8, device=dev)
    X = torch.empty_like(A)
    rep = prism.make_report(BATCH, mi, dev)
    call = lambda: prism.matfn_inv_root(A, "inv4", opts, S, out=X, ws=ws, report=rep)  # noqa: E731
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ms = _time(call, stream, 10)
    it = rep["iters"].cpu().numpy()
    tf = float(sum(block_flops(k, N) for k in it)) / (ms / 1e3) / 1e12
    Xh = X.cpu().numpy()
    errs = []
    for b in (0, BATCH - 1):
        r = o.spd_power_eigh(A_np[b], -0.25)
        errs.append(float(np.linalg.norm(Xh[b] - r) / np.linalg.norm(r)))
    st = rep["status"].cpu().numpy()
    return {"workload": "inv4_root_64x1024sq_spd_cond1e2_prism_d2_p8_tol1e-3_tf32",
            "ms": ms, "value": tf, "unit": "TFLOP/s", "frac_of_tf32_peak": tf / tp["tf32_tflops"],
            "median_iters_per_pass": [int(x) for x in np.median(it, axis=0)],
            "ok_or_stall_blocks": int(((st == 0) | (st == 17)).sum()), "max_vs_eigh": max(errs),
            "peak_note": "measured TF32 burst (cuBLAS 8192^3)"}


PM, PN, PBATCH, PRANK = 4096, 1024, 96, 64


def polar_flops(iters):
    """Algorithmic flops of one polar factor with k updates: per update the
    symmetric X^T X (n(n+1)m) and R^2 (n(n+1)n) and X Delta (2mn^2), plus the
    final residual."""
    k = int(iters)
    sym = PN * (PN + 1) * PM
    return k * (sym + PN * (PN + 1) * PN + 2 * PM * PN * PN) + sym


def polar_leg(args, dev, stream, peaks=None, batch=PBATCH, host_loop=False):
    """The Muon-style polar batch: 96 matrices 4096 x 1024, rank-64 signal plus
    0.01 noise, bf16 storage, d = 2, p = 8, until ||I - X^T X||_F / sqrt(n) <= 1e-2.
    `batch` and `host_loop` serve profiling (fewer matrices; every launch
    issued from the host, where profilers see it)."""
    import torch

    from second_order_optimizer_shampoo_b200 import _abi, prism, synth
    bits, _ = synth.lowrank_noise_batch(PM, PN, PRANK, 0.01, batch, 104)
    G = torch.from_numpy(bits.view("int16")).to(dev).view(torch.bfloat16)
    S = torch.from_numpy(synth.sketch_stack(40, PN, 8, 1004)).to(dev)
    opts = prism.make_opts(d=2, p=8, tol=1e-2, max_iter=40, prec="bf16", host_loop=host_loop)
    o2 = _abi.PrismOpts.from_buffer_copy(opts)
    o2.prec = _abi.SHP_BF16
    ws = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_POLAR, PM, PN, batch, o2),
                     dtype=torch.uint8, device=dev)
    X = torch.empty_like(G)
    rep = prism.make_report(batch, 40, dev)
    for _ in range(2):
        prism.matfn_polar(G, opts, S, out=X, ws=ws, report=rep)
    torch.cuda.synchronize()
    iters = rep["iters"][:, 0].cpu().numpy()
    ok = int((rep["status"].cpu().numpy() == 0).sum())
    flops = float(sum(polar_flops(k) for k in iters))
    reps = 3
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        prism.matfn_polar(G, opts, S, out=X, ws=ws, report=rep)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    peaks, src = load_peaks() if peaks is None else (peaks, "given")
    bf16_sust = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": f"polar_{batch}x4096x1024_bf16_lowrank64_prism_d2_p8_tol1e-2",
            "value": tf, "unit": "TFLOP/s", "ms_per_step": ms,
            "matrices_per_s": batch / (ms / 1e3), "median_iters": float(np.median(iters)),
            "status_ok": ok, "frac_of_bf16_peak": tf / bf16_sust,
            "note": "symmetric products (X^T X, R R) formed on their upper-triangle tiles "
                    "and counted n(n+1)K; peak: sustained BF16"}


def sketch_leg(R, S0, stream, peaks, peak_src):
    """Roofline of the sketch kernel (HBM bound): the alpha fit of d = 2 on a
    stack of n x n fp32 residuals, 5 passes V_j = R V_{j-1} (R read once per
    pass; 256 MiB at the config-3 size, larger than L2) plus the per-block
    Gram/argmin, replayed from a CUDA graph as inside the step (no host gaps)."""
    import torch

    from second_order_optimizer_shampoo_b200 import prism
    batch, n = R.shape[0], R.shape[-1]
    p = S0.shape[-1]
    v_dim = 2 * D + 1
    for _ in range(3):
        prism.prism_alpha_fit(R, S0, D, 0.375, 1.0)
    torch.cuda.synchronize()
    fit_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(fit_graph):
        prism.prism_alpha_fit(R, S0, D, 0.375, 1.0)
    for _ in range(3):
        fit_graph.replay()
    torch.cuda.synchronize()
    reps = 20
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    k0.record(stream)
    for _ in range(reps):
        fit_graph.replay()
    k1.record(stream)
    torch.cuda.synchronize()
    fit_ms = k0.elapsed_time(k1) / reps
    del fit_graph
    sk_bytes = v_dim * (batch * n * n * 4 + 2 * batch * n * p * 4)  # R once, V in and out
    sk_gbs = sk_bytes / (fit_ms / 1e3) / 1e9
    hbm = peaks.get("hbm_gbs", 6650.0)
    full = batch == BATCH and n == N and p == P
    return {
        "kernel": f"k_sketch_tma<8> x 5 + k_alpha (alpha fit, d = 2, {batch} x {n}^2, p = {p})",
        "bound": "hbm", "achieved": sk_gbs, "peak": hbm, "unit": "GB/s", "frac": sk_gbs / hbm,
        "traffic": SKETCH_TRAFFIC_PER_FIT if full else None, "algorithmic_bytes": sk_bytes,
        "ms_per_fit": fit_ms,
        "peak_note": f"{peak_src} STREAM-style copy bandwidth; the alpha kernel's time is included",
    }


def sketch_only(args):
    """The sketch leg alone on --batch seeded N(0, 0.01^2) symmetric residuals
    1024 x 1024 (for profiling k_sketch_tma)."""
    import torch

    from second_order_optimizer_shampoo_b200 import synth
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    R = torch.randn(args.batch, N, N, device=dev, generator=g) * 0.01
    R = (R + R.transpose(1, 2)).contiguous()
    S0 = torch.from_numpy(synth.sketch_stack(1, N, P, SEED_S)[0]).to(dev)
    peaks, src = load_peaks()
    print(json.dumps(sketch_leg(R, S0, torch.cuda.current_stream(), peaks, src)))
    return 0


# ------------------------------------------------------------------ our leg
def main():
    global BATCH
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-polar", action="store_true", help="skip the polar-factor leg")
    ap.add_argument("--no-small", action="store_true", help="skip the small-block leg")
    ap.add_argument("--no-large", action="store_true",
                    help="skip the 10240^2 square-root leg (it builds a 10240 x 20480 product "
                         "on the host first)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the Shampoo-step, GEMM-count and single-block legs")
    ap.add_argument("--prec", default="ozaki", choices=["ozaki", "3xtf32", "tf32"],
                    help="product path of --kernel step")
    ap.add_argument("--kernel", default=None, choices=["gemm", "small", "polar", "sketch", "step", "ozgemm",
                             "shampoo"],
                    help="run one piece alone for profiling: the batched 3xTF32 GEMM, the "
                         "small-block kernel, the polar leg (host-launched loop), the sketch "
                         "leg, the inverse-root step, the Ozaki GEMM or the Shampoo step "
                         "(--batch sets the GEMM/small/sketch/polar/step batch)")
    ap.add_argument("--batch", type=int, default=BATCH)
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.kernel == "gemm":
        return gemm_only(args)
    if args.kernel == "step":
        return step_only(args)
    if args.kernel == "ozgemm":
        return ozgemm_only(args)
    if args.kernel == "shampoo":
        return shampoo_only(args)
    if args.kernel == "small":
        return small_only(args)
    if args.kernel == "sketch":
        return sketch_only(args)
    if args.kernel == "polar":
        import torch
        print(json.dumps(polar_leg(args, torch.device("cuda", 0), torch.cuda.current_stream(),
                                   batch=args.batch, host_loop=True)))
        return 0
    BATCH = args.batch  # blocks per GPU of the main workload (64 unless profiling)

    import numpy as np
    import torch

    from second_order_optimizer_shampoo_b200 import _abi, prism, synth

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    # ---- inputs: each rank its own BATCH blocks (seeded by global block index)
    idx = list(range(rank * BATCH, (rank + 1) * BATCH))
    A_np = synth.spd_batch(N, BATCH, LAM_LO, 1.0, SEED_A, indices=idx)
    S_np = synth.sketch_stack(2 * MAX_ITER, N, P, SEED_S)
    A = torch.from_numpy(A_np).to(dev)
    S = torch.from_numpy(S_np).to(dev)
    opts = prism.make_opts(d=D, p=P, tol=TOL, max_iter=MAX_ITER, prec=PREC)
    ws = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, N, N, BATCH, opts),
                     dtype=torch.uint8, device=dev)
    X = torch.empty_like(A)
    rep_buf = prism.make_report(BATCH, MAX_ITER, dev)

    def step():
        return prism.matfn_inv_root(A, "inv4", opts, S, out=X, ws=ws, report=rep_buf)

    for _ in range(max(args.warmup, 3)):
        _, rep = step()
    torch.cuda.synchronize()
    iters = rep["iters"].cpu().numpy()
    status = rep["status"].cpu().numpy()
    flops_step = float(sum(block_flops(it, N) for it in iters))

    # ---- timed region (device time, CUDA events on the launching stream)
    stream = torch.cuda.current_stream()
    try:  # nvidia-smi -i takes the UUID, which survives CUDA_VISIBLE_DEVICES remapping
        clk = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    except Exception:
        clk = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clk.start()
    time.sleep(0.3)
    l0 = prism.kernel_launches()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = prism.kernel_launches() - l0
    clocks = clk.stop()
    barrier(world)
    ms = e0.elapsed_time(e1)
    ms_max, units, flops, launches_all = reduce_timing(ms, BATCH * args.steps, flops_step * args.steps,
                                                       launches, world)
    value = flops / (ms_max / 1e3) / 1e12
    precond_s = units / (ms_max / 1e3)
    X_host_res = X.cpu().numpy()

    # ---- end to end through the public API with host buffers.  Every step
    # copies its input from pinned host memory and its result and statuses
    # back; with two device buffer sets and separate copy streams the copies
    # of step i+1 (in) and i-1 (out) run while step i computes.
    A_host = torch.from_numpy(A_np).pin_memory()
    S_host = torch.from_numpy(S_np).pin_memory()
    X_host = [torch.empty_like(A_host).pin_memory() for _ in range(2)]
    st_host = [torch.empty(BATCH, dtype=torch.int32).pin_memory() for _ in range(2)]
    A2 = [torch.empty_like(A) for _ in range(2)]
    S2 = [torch.empty_like(S) for _ in range(2)]
    X2 = [torch.empty_like(A) for _ in range(2)]
    rep2 = [prism.make_report(BATCH, MAX_ITER, dev) for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731
    for b in range(2):  # record both buffer sets' graphs outside the timed region
        prism.matfn_inv_root(A, "inv4", opts, S, out=X2[b], ws=ws, report=rep2[b])
    barrier(world)
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    h2d_s.wait_stream(stream)
    d2h_s.wait_stream(stream)
    in_ready, computed, out_read = [None, None], [None, None], [None, None]
    for i in range(args.steps):
        b = i % 2
        with torch.cuda.stream(h2d_s):
            if computed[b] is not None:  # step i-2 has finished reading A2[b]
                h2d_s.wait_event(computed[b])
            A2[b].copy_(A_host, non_blocking=True)
            S2[b].copy_(S_host, non_blocking=True)
            in_ready[b] = ev()
            in_ready[b].record(h2d_s)
        stream.wait_event(in_ready[b])
        if out_read[b] is not None:  # step i-2's result has been copied out
            stream.wait_event(out_read[b])
        prism.matfn_inv_root(A2[b], "inv4", opts, S2[b], out=X2[b], ws=ws, report=rep2[b])
        computed[b] = ev()
        computed[b].record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(computed[b])
            X_host[b].copy_(X2[b], non_blocking=True)
            st_host[b].copy_(rep2[b]["status"], non_blocking=True)
            out_read[b] = ev()
            out_read[b].record(d2h_s)
    stream.wait_stream(d2h_s)
    f1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms, _, _, _ = reduce_timing(f0.elapsed_time(f1), 0, 0, 0, world)
    e2e_value = flops / (e2e_ms / 1e3) / 1e12
    h2d = A_host.numel() * 4 + S_host.numel() * 4
    d2h = X_host[0].numel() * 4 + st_host[0].numel() * 4
    e2e_ok = bool(all(int((h.numpy() == 0).sum()) == BATCH for h in st_host))
    del A2, S2, X2, rep2

    peaks, peak_src = load_peaks()
    tp = measure_tensor_peaks(dev)

    # ---- roofline of the dominant kernel: k_gemm_oz in the step's launch
    # shape (64 x 1024^3) and its in-step epilogue (C <- C + A B, fp64 read,
    # combine, write, maxima), timed alone with the operands' slices reused
    g = torch.Generator(device=dev).manual_seed(9)
    Xa = torch.randn(BATCH, N, N, device=dev, dtype=torch.float64, generator=g)
    Xb = torch.randn(BATCH, N, N, device=dev, dtype=torch.float64, generator=g)
    Cc = torch.zeros_like(Xa)
    mws = torch.empty(int(_abi.lib().shp_matmul_f64_workspace_bytes(N, N, N, BATCH)),
                      dtype=torch.uint8, device=dev)
    prism.shp_matmul_f64(Xa, Xb, out=Cc, ws=mws)
    for _ in range(3):
        prism.shp_matmul_f64(Xa, Xb, out=Cc, ws=mws, reuse_a=True, reuse_b=True, accumulate=True)
    torch.cuda.synchronize()
    reps = 20
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(reps):
        prism.shp_matmul_f64(Xa, Xb, out=Cc, ws=mws, reuse_a=True, reuse_b=True, accumulate=True)
    g1.record(stream)
    torch.cuda.synchronize()
    gemm_ms = g0.elapsed_time(g1) / reps
    del Xa, Xb, Cc, mws
    torch.cuda.empty_cache()
    int8_ops = OZ_PRODUCTS * 2.0 * N ** 3 * BATCH
    int8_rate = int8_ops / (gemm_ms / 1e3) / 1e12
    step_ms = ms_max / args.steps
    roofline = {
        "kernel": "k_gemm_oz (Ozaki int8 x5, persistent CTA pairs, 64 x 1024^3, C += A B)",
        "bound": "tensor", "achieved": int8_rate, "peak": tp["int8_tops"], "unit": "TOP/s int8",
        "frac": int8_rate / tp["int8_tops"], "traffic": OZ_GEMM_TRAFFIC_PER_LAUNCH,
        "traffic_unit": "bytes per launch",
        "algorithmic_bytes": BATCH * N * N * (2 * OZ_SLICES + 16),
        "peak_note": "measured here: best cuBLAS int8 8192^3 (burst)",
        "ms_per_launch": gemm_ms, "fp64_equiv_tflops": 2.0 * N ** 3 * BATCH / (gemm_ms / 1e3) / 1e12,
        # the step's products at this kernel's rate, as a share of the step time
        "step_share_est": flops_step / (2.0 * N ** 3 * BATCH / (gemm_ms / 1e3)) / (step_ms / 1e3),
    }

    # ---- accuracy of the headline result and the fp32-storage paths
    from oracle import prism_ref as o
    acc_blocks = [b for b in ACC_BLOCKS if b < BATCH]
    refs = {b: o.spd_power_eigh(A_np[b], -0.25) for b in acc_blocks}

    def rel(x, r):
        return float(np.linalg.norm(x - r) / np.linalg.norm(r))

    acc = {"blocks": acc_blocks,
           "ozaki_vs_eigh": [rel(X_host_res[b], refs[b]) for b in acc_blocks]}
    fp32_paths = {}
    if world == 1 and not args.no_extra:
        for name, pr in (("split_3xtf32", "3xtf32"), ("tf32", "tf32")):
            o3 = prism.make_opts(d=D, p=P, tol=TOL, max_iter=MAX_ITER, prec=pr)
            ws3 = torch.empty(prism.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, N, N, BATCH, o3),
                              dtype=torch.uint8, device=dev)
            X3 = torch.empty_like(A)
            r3 = prism.make_report(BATCH, MAX_ITER, dev)
            call = lambda: prism.matfn_inv_root(A, "inv4", o3, S, out=X3, ws=ws3, report=r3)  # noqa: E731
            call()
            torch.cuda.synchronize()
            t3 = _time(call, stream, 5)
            it3 = r3["iters"].cpu().numpy()
            st3 = r3["status"].cpu().numpy()
            X3h = X3.cpu().numpy()
            errs = [rel(X3h[b], refs[b]) for b in acc_blocks]
            fp32_paths[name] = {
                "ms": t3, "tflops": float(sum(block_flops(k, N) for k in it3)) / (t3 / 1e3) / 1e12,
                "ok_blocks": int((st3 == 0).sum()), "max_vs_eigh": max(errs) if np.all(np.isfinite(errs)) else None}
            acc[name + "_vs_eigh"] = errs
            del ws3, X3
            torch.cuda.empty_cache()

    sketch_roof = sketch_leg(A, S[0], stream, peaks, peak_src)

    polar = None if args.no_polar else polar_leg(args, dev, stream, peaks)
    extra = not args.no_extra and world == 1
    step2 = shampoo_step_leg(args, dev, stream) if extra else None
    counts = gemm_count_leg(args, dev, stream, A) if extra else None
    single = single_block_leg(args, dev, stream) if extra else None
    sweep = sigma_sweep_leg(args, dev, stream) if extra else None
    tf32b = tf32_batched_leg(args, dev, stream, tp) if extra else None
    small = None if args.no_small else small_block_leg(args, dev, stream,
                                                        peaks.get("sm_max_mhz", 1965.0))
    large = large_sqrt_leg(args, dev, stream) if extra and not args.no_large else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_tot, f_tot, nb = 0.0, 0.0, 0
        for b in range(BATCH):
            t, f = oracle_sample(A_np[b], S_np)
            t_tot += t
            f_tot += f
            nb += 1
            if t_tot > 10.0:
                break
        cpu = {"value": f_tot / t_tot / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
               "kind": "oracle",
               "sample": f"{nb} of the {BATCH} blocks, float64 NumPy/LAPACK oracle (same recurrence)",
               "ms_per_block": 1e3 * t_tot / nb,
               "eigh_ms_per_block": 1e3 * eigh_sample(A_np[0])}
        # the oracle's own distance from eigh on the reported blocks
        oo = o.PrismOpts(d=D, p=P, lo=0.375, hi=1.0, tol=TOL, max_iter=MAX_ITER)
        oxs = {b: o.inv_root_ref(A_np[b], o.POW_INV4, oo, S_np,
                                 force_iters=iters[b])[0] for b in acc_blocks}
        acc["oracle_vs_eigh"] = [rel(oxs[b], refs[b]) for b in acc_blocks]
        acc["ozaki_vs_oracle"] = [rel(X_host_res[b], oxs[b]) for b in acc_blocks]

    def r4(x):
        if isinstance(x, float):
            return float(f"{x:.4g}")
        if isinstance(x, dict):
            return {k: r4(v) for k, v in x.items()}
        if isinstance(x, list):
            return [r4(v) for v in x]
        return x

    if rank == 0:
        # the detailed legs first and the headline keys last: the end of the
        # line is what a truncated log keeps
        line = {
            "polar_sigma_sweep": sweep,
            "gemms_to_residual": counts,
            "single_64": single,
            "small_blocks": small,
            "shampoo_step_1024": step2,
            "tf32_batched": tf32b,
            "sqrt_10240": large,
            "polar": polar,
            "roofline_sketch": sketch_roof,
            "cpu_baseline": cpu,
            "clocks": clocks,
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(world),
            "preconditioners_per_s": precond_s,
            "iters_per_pass": [int(x) for x in np.median(iters, axis=0)],
            "status_ok_blocks": int((status == 0).sum()), "blocks": int(len(status)),
            "gpu_launches": int(launches_all),
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "status_ok": e2e_ok},
            "peaks": tp,
            "fp32_paths": fp32_paths,
            "polar_tflops": polar["value"] if polar else None,
            "polar_frac_bf16": polar["frac_of_bf16_peak"] if polar else None,
            "sqrt10240_ms": large["prism_d2"]["ms"] if large else None,
            "sqrt10240_gemms": {k: large[k]["gemms"] for k in ("prism_d2", "taylor_d2", "taylor_d1")} if large else None,
            "tf32_1024_tflops": tf32b["value"] if tf32b else None,
            "tf32_1024_frac": tf32b["frac_of_tf32_peak"] if tf32b else None,
            "sketch_frac_hbm": sketch_roof["frac"],
            "accuracy": acc,
            "roofline": roofline,
        }
        print(json.dumps(r4(line), separators=(",", ":")))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
