#!/usr/bin/env python
"""Benchmark of the MPQ row solve on B200.

One step = one whole solve of a layer (init, T_vamp VAMP iterations, marginal
MAP, <= 3 CD sweeps, energies) through the C ABI with W already resident in
HBM.  Default workload: the 4096x4096 q_proj-shaped layer, 4-bit scalar grid,
T_vamp = 16, 3 CD sweeps, X 8192x4096 (synthetic, seeded).  Setup (the
compact SVD of X on the device) is timed separately and not part of a step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mpq|reference]

With N > 1 (torchrun, one rank per GPU) every rank solves its own rows of a
layer with N*m_out rows (weak scaling, no data-path collective); the time is
the max over ranks.  `--impl reference` times the float64 CPU oracle on a
bounded sample of the same workload on the host cores.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MPQ solve weights/sec (VAMP+3 CD sweeps) per layer; % of roofline"
UNIT = "weights/s"
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # FMA lanes x 2 x max SM clock


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mpq", choices=["mpq", "reference"])
    ap.add_argument("--config", default="q4096")
    ap.add_argument("--cpu-rows", type=int, default=0,
                    help="oracle sample size in rows (0: 8 for scalar grids, 1 for the 65536-word "
                         "E8 codebook, whose oracle denoiser enumerates every codeword per block)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--rows", type=int, default=0,
                    help="solve only the first ROWS rows (small cases for ncu captures; "
                         "the line then names the reduced workload)")
    ap.add_argument("--cd-panel", type=int, default=0,
                    help="columns per CD panel (multiple of 128; 0 = automatic)")
    ap.add_argument("--group-size", type=int, default=0,
                    help="scalar workloads: one min-max grid per group of this many columns "
                         "(0 = one per row)")
    ap.add_argument("--greedy", action="store_true",
                    help="the greedy baseline (LDLQ init, T_vamp = 0) with the same CD sweeps "
                         "instead of MPQ")
    ap.add_argument("--tau", type=float, default=0.2,
                    help="prior anchor scale in codebook units (the pages' default 0.2; "
                         "inf = the unanchored form)")
    ap.add_argument("--spectrum-cache", default=None,
                    help="npz file: reuse the spectrum a previous run computed on the device")
    ap.add_argument("--gram-rows", type=int, default=262144,
                    help="also time the streamed fp64 Gram accumulation of this many calibration "
                         "rows (chunks of 16384 through mpq_gram_accumulate; 0 = skip)")
    ap.add_argument("--rht-rows", type=int, default=32768,
                    help="also time the random Hadamard rotation (mpq_rht, in place) of this "
                         "many rows of the config's width (0 = skip)")
    return ap.parse_args()


def rht_timing(n, rows, dev, reps=5):
    """Average milliseconds (CUDA events on the current stream) of one
    in-place random Hadamard rotation of a rows x n fp32 matrix, after one
    warm-up.  At 32768 x 4096 the matrix is 512 MiB, four times L2, so every
    rotation reads and writes HBM."""
    import torch
    import post_weight_quantization_row_b200 as mpq
    g = torch.Generator(device=dev)
    g.manual_seed(20261300)
    X = torch.randn(rows, n, generator=g, device=dev, dtype=torch.float32)
    signs = torch.where(torch.rand(n, generator=g, device=dev) < 0.5, -1.0, 1.0).to(torch.float32)
    mpq.rht(X, signs)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        mpq.rht(X, signs)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def gram_timing(n, rows, dev):
    """Seconds (CUDA events) to accumulate X^T X over `rows` synthetic rows
    of width n in chunks of 16384 through the streamed Gram handle; two
    device-resident chunks take turns, so the time is the accumulation's."""
    import torch
    import post_weight_quantization_row_b200 as mpq
    chunk = min(16384, rows)
    g = torch.Generator(device=dev)
    g.manual_seed(20261299)
    xs = [torch.randn(chunk, n, generator=g, device=dev, dtype=torch.float32) for _ in range(2)]
    gram = mpq.Gram(n)
    gram.accumulate(xs[0])  # warm-up (first use of the kernels)
    torch.cuda.synchronize()
    gram.close()
    gram = mpq.Gram(n)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    done = 0
    while done < rows:
        k = min(chunk, rows - done)
        gram.accumulate(xs[(done // chunk) % 2][:k])
        done += k
    e1.record()
    torch.cuda.synchronize()
    gram.close()
    return e0.elapsed_time(e1) / 1e3


# ------------------------------------------------------------------ dist ---

def dist_init(n_gpus, backend="nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def allreduce_max(x: float, world: int) -> float:
    """Max over ranks (the job's time is that of its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(local_total_ms: float, steps: int, m_out: int, n: int, world: int):
    """Weak scaling: every rank solves its own m_out rows; the job's step time
    is the slowest rank's, and the value counts the weights of all ranks."""
    total_ms = allreduce_max(local_total_ms, world)
    ms_per_step = total_ms / steps
    return world * m_out * n / (ms_per_step / 1e3), ms_per_step


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.lines = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "200"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            threading.Thread(target=self._read, daemon=True).start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------- algorithmic work ---

# fp32-accurate contractions are issued as fp16 tensor-core MMAs on hi/lo
# splits: 3 passes per product (2 when the A operand is exact in fp16)
GEMM_PASSES = {"gemm_project": 3, "gemm_expand": 3, "gemm_energy": 3, "gemm_hessian": 3,
               "gemm_cd_update": 2, "gemm_cd_panel": 2}


def kernel_work(name, m, n, r, d, K, L):
    """(bound, unit, work per launch) -- algorithmic flops or bytes."""
    if name in ("gemm_project", "gemm_energy", "gemm_expand"):
        return "tensor", "TFLOP/s", 2.0 * m * n * r
    if name == "gemm_hessian":
        return "tensor", "TFLOP/s", 2.0 * m * n * n
    if name == "k_denoise_scalar":      # read r1, write xhat1 (+ v per element)
        return "hbm", "GB/s", 8.0 * m * n
    if name == "k_extrinsic_d2l":        # read w, r1, xhat1; write r2, A
        return "hbm", "GB/s", 20.0 * m * n
    if name == "k_extrinsic_l2d":        # read r2, D; write r1
        return "hbm", "GB/s", 12.0 * m * n
    if name == "k_linear_finish":        # per row: the column tiles' two M-step sums
        return "hbm", "GB/s", 8.0 * m * ((r + 127) // 128)
    if name in ("k_denoise_vec", "k_denoise_vec_tc"):  # one exponential per (block, codeword)
        return "sfu", "Gexp/s", float(m) * (n // 8) * K
    if name == "k_vamp_row_scalar":      # read g, r2, w; write r2 and the fp16 hi/lo operand
        return "hbm", "GB/s", 20.0 * m * n
    if name == "k_vamp_row_scalar(map)":  # read g, r2, w; write the level index
        return "hbm", "GB/s", 14.0 * m * n
    if name == "k_cd_tile_decide":       # per 128-column tile: h, idx in; idx, Delta hi/lo out
        return "hbm", "GB/s", 12.0 * m * 128
    if name == "k_ldlq_tile":            # per 128-column tile: W_work in; idx, E hi/lo out
        return "hbm", "GB/s", 10.0 * m * 128
    return None


KERNEL_SOURCE = {"gemm": "gemm_tc.cu", "k_cd_vec_scan": "cd_scan_tc.cu", "k_cd": "kernels_cd.cu",
                 "k_ldlq": "greedy.cu",
                 "k_denoise_vec_tc": "denoise_tc.cu", "k_": "kernels_vamp.cu"}


def source_sha(kernel):
    """Hash of the source file that defines `kernel` plus the device PTX
    helpers it may use (the host-side declarations elsewhere do not change
    what a capture measured)."""
    csrc = os.path.join(ROOT, "post_weight_quantization_row_b200", "csrc")
    fname = next(v for k, v in KERNEL_SOURCE.items() if kernel.startswith(k))
    h = hashlib.sha256()
    for f in (fname, "tc_ptx.cuh"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    sha = source_sha(kernel)
    for line in open(path):
        parts = line.split()
        if len(parts) == 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload:
            return float(parts[2]) if parts[3] == sha else None
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------ workloads ---

def workload(cfg, rank=0):
    import mpq_inputs as mi
    p = mi.make_problem(cfg)
    if rank > 0:
        # weak scaling: rank k solves other rows of an N*m_out-row layer
        cfgno = mi.WORKLOADS[cfg][0]
        g = np.random.default_rng(mi.SEED_BASE + 10 * cfgno + 1000 * rank)
        W = mi.lognormal_rows_w(g, p.m_out, p.n)
        if p.d == 8:
            signs = np.where(mi.rng_for(cfgno, 3).random(p.n) < 0.5, -1.0, 1.0)
            W = mi.random_hadamard_apply(W, signs)
        p.W = np.ascontiguousarray(W, dtype=np.float32)
    return p


def describe(p, cfg, group=0, tau=0.2):
    bits = {8: 3, 16: 4}.get(p.levels, None) if p.d == 1 else 2
    grid = f"group-{group}" if group else "per-row"
    anchor = f"tau={tau:g}" if math.isfinite(tau) else "unanchored (tau=inf)"
    return {"workload": f"{cfg}: W {p.m_out}x{p.n}, X {p.X.shape[0]}x{p.n}, "
                        + (f"{bits}-bit {grid} min-max grid" if p.d == 1 else
                           f"offset-E8 d=8 K={p.levels}, RHT")
                        + f", T_vamp={p.T_vamp}, rho_damp=0.5, {anchor}, CD sweeps<={p.cd_sweeps}",
            "m_out": p.m_out, "n": p.n, "m_calib": int(p.X.shape[0]), "d": p.d,
            "levels_or_K": p.levels, "T_vamp": p.T_vamp, "cd_sweeps": p.cd_sweeps,
            "tau": tau if math.isfinite(tau) else "inf",
            "seeds": p.seeds, "l2": "flushed between timed steps (512 MiB write)"}


def oracle_sample(p, rows, steps=1, group=0, greedy_damp=None, tau=0.2):
    """Time the float64 oracle on `rows` rows of the layer (spectrum excluded)."""
    from oracle import mpq_oracle as orc
    t0 = time.time()
    s, V = orc.spectrum(p.X)
    t_spec = time.time() - t0
    cb = orc.scalar_levels(p.levels) if p.d == 1 else p.codebook.astype(np.float64)
    times = []
    for k in range(steps):
        sel = slice((k * rows) % p.m_out, (k * rows) % p.m_out + rows)
        t0 = time.perf_counter()
        orc.solve(p.W[sel], cb, s, V, p.T_vamp, p.cd_sweeps, group=group, greedy_damp=greedy_damp,
                  tau=tau)
        times.append(time.perf_counter() - t0)
    return times, t_spec


# ------------------------------------------------------------ reference ---

def run_reference(args, world, rank):
    if rank != 0:
        return
    p = workload(args.config)
    if args.greedy:
        p.T_vamp = 0
    rows = max(1, args.cpu_rows // 2)
    times, t_spec = oracle_sample(p, rows, args.warmup + args.steps, args.group_size,
                                  0.01 if args.greedy else None, args.tau)
    timed = times[args.warmup:]
    sec = sum(timed) / len(timed)
    value = rows * p.n / sec
    cores = len(os.sched_getaffinity(0))
    cfgd = describe(p, args.config, args.group_size, args.tau)
    if args.greedy:
        cfgd["workload"] += " (greedy baseline: LDLQ init, damp 0.01, then the same CD)"
        cfgd["init"] = "LDLQ"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfgd,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{rows} rows of the layer per step (rows are independent "
                                       f"problems), full T_vamp and CD; spectrum "
                                       f"({t_spec:.1f} s) excluded"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ mpq ---

def run_mpq(args, world, rank, local):
    import torch

    import post_weight_quantization_row_b200 as mpq

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    p = workload(args.config, rank)
    if args.rows:
        p.W = np.ascontiguousarray(p.W[:args.rows])
    greedy = {}
    if args.greedy:
        p.T_vamp = 0
        greedy = {"greedy_init": 1}
    cfgd = describe(p, args.config, args.group_size, args.tau)
    if args.greedy:
        cfgd["workload"] += " (greedy baseline: LDLQ init, damp 0.01, then the same CD)"
        cfgd["init"] = "LDLQ"
    m, n = p.m_out, p.n
    cb = p.codebook if p.d == 8 else None
    cache = args.spectrum_cache
    if cache and os.path.exists(cache):
        z = np.load(cache)
        plan = mpq.Plan.from_spectrum(torch.from_numpy(z["s"]).to(dev),
                                      torch.from_numpy(z["V"]).to(dev), p.d, p.levels, codebook=cb,
                                      cd_panel=args.cd_panel, group_size=args.group_size,
                                      tau=args.tau, **greedy)
        setup_s = None
    else:
        X = torch.from_numpy(p.X).to(dev)
        torch.cuda.synchronize()
        t0 = time.time()
        plan = mpq.Plan.from_x(X, p.d, p.levels, codebook=cb, cd_panel=args.cd_panel,
                               group_size=args.group_size, tau=args.tau, **greedy)
        torch.cuda.synchronize()
        setup_s = time.time() - t0
        del X
        if cache:
            s_, V_ = plan.spectrum()
            np.savez(cache, s=s_.cpu().numpy(), V=V_.cpu().numpy())
    r = plan.r
    gram_run = None
    if args.gram_rows > 0 and rank == 0:
        gs = gram_timing(n, args.gram_rows, dev)
        gram_run = {"rows": args.gram_rows, "n": n, "s": round(gs, 3),
                    "fp64_tflops": round(2.0 * args.gram_rows * n * n / gs / 1e12, 2),
                    "what": "streamed X^T X in fp64 (mpq_gram_accumulate, 16384-row chunks)"}
    rht_run = None
    if args.rht_rows > 0 and rank == 0 and n & (n - 1) == 0:
        rms = rht_timing(n, args.rht_rows, dev)
        rgbs = 8.0 * args.rht_rows * n / (rms / 1e3) / 1e9  # one fp32 read + one write per element
        rht_run = {"rows": args.rht_rows, "n": n, "ms": round(rms, 4), "gbs": round(rgbs, 1),
                   "hbm_frac": round(rgbs / load_peaks()[0]["hbm_gbs"], 3),
                   "what": "in-place x <- (x .* signs) H_n / sqrt(n) (mpq_rht), 8 B per element"}
    W = torch.from_numpy(p.W).to(dev)
    out = {"idx": torch.empty(m, plan.B, dtype=torch.int16, device=dev),
           "w_hat": torch.empty(m, n, dtype=torch.float32, device=dev),
           "energy": torch.empty(m, dtype=torch.float32, device=dev)}
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        plan.solve(W, p.T_vamp, p.cd_sweeps, out=out, check_status=False)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    plan.status()
    torch.cuda.synchronize()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    # the timed steps run without the per-kernel event profiler (its event
    # pairs would add to every launch); a second pass of the same steps,
    # profiled, gives the per-kernel times behind the roofline
    launches0 = mpq.kernel_launch_count()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    launches = mpq.kernel_launch_count() - launches0
    objective = float(out["energy"].double().mean().item())
    barrier(world)
    mpq.profile_start()
    for i in range(args.steps):
        flush.fill_(float(i))
        step()
    torch.cuda.synchronize()
    prof = mpq.profile_stop()
    plan.status()
    barrier(world)
    value, ms_per_step = job_throughput(sum(a.elapsed_time(b) for a, b in ev), args.steps, m, n,
                                        world)

    # roofline of the dominant kernel (largest share of device time)
    peaks, peak_src = load_peaks()
    dom = max(prof.items(), key=lambda kv: kv[1][1])
    name, (cnt, kms) = dom
    roof = None
    wk = kernel_work(name, m, n, r, p.d, p.levels, p.levels)
    # the whole step against its roofline: every kernel with a fixed
    # algorithmic work at its own bound (the CD's decide kernels at their
    # bytes; the gated CD update GEMMs, whose work depends on the changes,
    # at zero), over the measured step time -- a lower bound on the fraction
    ideal_ms = 0.0
    for kname, (kc, _) in prof.items():
        kw = kernel_work(kname, m, n, r, p.d, p.levels, p.levels)
        if not kw:
            continue
        kb, _, kwork = kw
        if kb == "tensor":
            kpeak = peaks["bf16_tflops"] / GEMM_PASSES.get(kname, 1) * 1e12
        elif kb == "hbm":
            kpeak = peaks["hbm_gbs"] * 1e9
        else:
            kpeak = 148 * 16 * 1.965e9
        ideal_ms += kwork * kc / kpeak * 1e3
    ideal_ms /= args.steps
    solve_roof = {"ideal_ms": ideal_ms, "measured_ms": ms_per_step, "frac": ideal_ms / ms_per_step,
                  "basis": "sum over kernels of launches x algorithmic work / measured peak "
                           "(tensor: bf16 burst / fp16 passes; hbm: copy GB/s; sfu: MUFU ex2 rate); "
                           "CD update GEMMs counted at zero"}
    if wk:
        bound, unit, work = wk
        avg_s = kms / cnt / 1e3
        passes = GEMM_PASSES.get(name, 1)
        if unit == "TFLOP/s":
            achieved = work / avg_s / 1e12
            # fp32-accurate work: the fp16 dense peak divided by the MMA passes
            peak = FP32_ALU_PEAK_TFLOPS if bound == "alu" else peaks["bf16_tflops"] / passes
        elif unit == "GB/s":
            achieved = work / avg_s / 1e9
            peak = peaks["hbm_gbs"]
        else:
            achieved = work / avg_s / 1e9
            peak = 148 * 16 * 1.965  # MUFU ex2 per clock per SM x SMs x GHz -> Gexp/s
        src = {"alu": "derived: 148 SMs x 128 FP32 lanes x 2 x 1965 MHz",
               "tensor": f"{peak_src} bf16/fp16 dense {peaks['bf16_tflops']} TFLOP/s "
                         f"(MEASURED_PEAKS.json) / {passes} fp16 MMA passes per fp32-accurate product",
               }.get(bound, f"{peak_src} MEASURED_PEAKS.json")
        roof = {"bound": bound, "kernel": name, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak,
                "traffic": recorded_traffic(name, args.config if not args.rows
                                            else f"{args.config}:rows{args.rows}"),
                "peak_source": src, "work_per_launch": work, "launches": cnt,
                "avg_launch_ms": kms / cnt}
        if bound == "tensor":
            roof["tensor_pipe_frac"] = achieved * passes / peaks["bf16_tflops"]
    total_prof = sum(v[1] for v in prof.values())
    kernels = {k: {"launches": v[0], "ms": round(v[1], 4), "share": round(v[1] / total_prof, 4)}
               for k, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}

    # end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        Wh = torch.from_numpy(p.W).pin_memory()
        ho = {"idx": torch.empty(m, plan.B, dtype=torch.int16, pin_memory=True),
              "w_hat": torch.empty(m, n, dtype=torch.float32, pin_memory=True),
              "energy": torch.empty(m, dtype=torch.float32, pin_memory=True)}
        plan.solve_host(Wh, p.T_vamp, p.cd_sweeps, out=ho)  # warm the staging buffers
        barrier(world)
        torch.cuda.synchronize()
        e2e_ms = 0.0
        for i in range(args.steps):
            flush.fill_(float(i))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            plan.solve_host(Wh, p.T_vamp, p.cd_sweeps, out=ho)
            b.record(stream)
            torch.cuda.synchronize()
            e2e_ms += a.elapsed_time(b)
        e2e_ms = allreduce_max(e2e_ms, world) / args.steps
        e2e = {"value": world * m * n / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": m * n * 4,
               "d2h_bytes_per_step": m * plan.B * 2 + m * n * 4 + m * 4,
               "ms_per_step": e2e_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        times, t_spec = oracle_sample(p, args.cpu_rows, 1, args.group_size,
                                      0.01 if args.greedy else None, args.tau)
        cpu = {"value": args.cpu_rows * n / times[0], "unit": UNIT,
               "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"rows 0..{args.cpu_rows - 1} of the layer (independent problems), "
                         f"full T_vamp and CD; spectrum ({t_spec:.1f} s) excluded"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic", "config": cfgd,
                "run": {"setup_s": None if setup_s is None else round(setup_s, 3),
                        "gram": gram_run, "rht": rht_run, "rank": r,
                        "cd_panel": args.cd_panel or "auto",
                        "parallelism": f"rows sharded over {world} GPU(s)"},
                "rows_per_s": world * m / (ms_per_step / 1e3),
                "objective": {"mean_energy": objective, "what": "mean over rows of "
                              "1/2 |X (w - w_hat)|^2 after the timed solves"},
                "roofline": roof, "solve_roofline": solve_roof, "cpu_baseline": cpu, "e2e": e2e,
                "clocks": clk.summary(),
                "gpu_launches": launches, "kernels": kernels}
        print(json.dumps(line), flush=True)
    plan.close()


def main():
    args = parse()
    if args.cpu_rows <= 0:
        import mpq_inputs as mi
        args.cpu_rows = 1 if mi.WORKLOADS[args.config][4] == 8 else 8
    world, rank, local = dist_init(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_mpq(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
