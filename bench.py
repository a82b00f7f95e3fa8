"""Benchmark of the W4A4G4 triple-branch linear layer (FourTune, arXiv 2607.05711).

One step = the whole hot path once over one batch: the forward (tensor max, 16x16
block quantization of X, the low-rank down-projection, the 4-bit GEMM with the up-
projections fused in) and the backward (the same for G, the dX GEMM through Q(R)^T,
and the adapter gradients dA, dB).  Workload: the FLUX.1-dev attention QKV projection,
4608 tokens (4096 image + 512 text) x 3072 -> 9216, stabilizer rank 32, LoRA rank 16,
synthetic inputs and random-init weights of that shape (see workloads.py).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs data-parallel under torchrun: each rank processes its own 4608 tokens
(weak scaling) and the adapter gradients are summed with an NCCL all-reduce.  The
reference arm times the CPU oracle (the only reference this method has) on a bounded
sample of the same workload.  One JSON line on rank 0.
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
sys.path.insert(0, ROOT)

METRIC = "W4A4G4 linear fwd+bwd TFLOPS & % FP4 roofline; quantizer GB/s vs HBM"
NOMINAL_FP4_OVER_BF16 = 4.0   # 9 / 2.25 PFLOP/s dense (B200 spec ratio)
NOMINAL_FP4_TFLOPS = 9000.0   # B200 dense FP4 spec

# single-layer workloads (one FourTune linear, forward + backward); the default is the
# attention QKV projection, the others are the MLP and single-stream layers
WORKLOADS = {"qkv": "FLUX_QKV", "mlp_up": "FLUX_MLP_UP", "mlp_down": "FLUX_MLP_DOWN",
             "single_l1": "FLUX_SS_L1", "single_l2": "FLUX_SS_L2"}


def layer_flops(M, K, N, r_s, r):
    R = r_s + r
    fp4 = 4.0 * M * N * K                              # forward GEMM + dX GEMM
    bf16 = 2.0 * R * (2 * M * K + 2 * M * N) + 2.0 * r * (M * N + M * K)
    return fp4, bf16


def pass_flops(M, K, N, r_s, r):
    """(forward, backward) algorithmic FLOPs: FP4 GEMM + low-rank down / up projections,
    plus dB and dA in the backward."""
    R = r_s + r
    fwd = 2.0 * M * N * K + 2.0 * R * (M * K + M * N)
    bwd = 2.0 * M * N * K + 2.0 * R * (M * N + M * K) + 2.0 * r * (M * N + M * K)
    return fwd, bwd


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"ft_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 6 and parts[0].isdigit():
                    rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[2 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(int(r[0]) for r in rows), "sm_max_mhz": int(rows[0][1]),
                "reasons": reasons, "samples": len(rows)}


def run_reference(args, spec):
    """The reference arm: the CPU oracle as it stands, on a bounded token sample."""
    import numpy as np
    import torch

    from diffusion_dit_b200 import prep, workloads as wl
    from oracle import fourtune_oracle as ora
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    rows = args.ref_rows
    inp = wl.make_layer_inputs(spec, seed=0, rows=rows)
    split = prep.svd_split(inp.w, spec.r_s)
    layer = ora.Layer(qr=ora.quantize_residual(split.residual), ls_up=split.ls_up, ls_down=split.ls_down,
                      lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)
    threads = blas_threads()

    def one():
        ora.linear_fwd(inp.x, layer)
        ora.linear_bwd(inp.x, inp.dy, layer)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = (time.perf_counter() - t0) / args.steps
    fp4, bf = layer_flops(rows, spec.K, spec.N, spec.r_s, spec.r)
    value = (fp4 + bf) / dt / 1e12
    sample = f"{rows} of {spec.M} tokens, full weights; oracle quantize+fwd+bwd (fp64 products)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(spec),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def gemm_traffic():
    """DRAM bytes per launch of the 4-bit GEMM from the committed ncu summary, or None
    when the kernel's sources have changed since those counters were taken."""
    import hashlib
    import re
    here = os.path.dirname(os.path.abspath(__file__))
    try:
        text = open(os.path.join(here, "profiles", "gemm_fp4_lowrank_pair_kernel.md")).read()
        m = re.search(r"traffic_bytes_per_launch: (\d+) sources_sha256_16: ([0-9a-f]{16})", text)
        src = b"".join(open(os.path.join(here, "diffusion_dit_b200", "csrc", f), "rb").read()
                       for f in ("ft_gemm2.cu", "ft_ptx.cuh"))
    except OSError:
        return None
    if not m or hashlib.sha256(src).hexdigest()[:16] != m.group(2):
        return None
    return int(m.group(1))


def cublaslt_nvfp4_tflops(M, N, K, iters=20):
    """cuBLASLt's block-scaled NVFP4 GEMM (torch._scaled_mm, bf16 out) at one shape: the
    attainable rate of a library 4-bit GEMM on this GPU, for context.  None if the
    installed torch cannot run it."""
    import torch
    try:
        dev = torch.device("cuda")
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
        b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
        a, b = a.view(torch.float4_e2m1fn_x2), b.view(torch.float4_e2m1fn_x2)
        rup = lambda x, m: (x + m - 1) // m * m  # noqa: E731
        sa = torch.ones(rup(M, 128) * rup(K // 16, 4), device=dev).to(torch.float8_e4m3fn)
        sb = torch.ones(rup(N, 128) * rup(K // 16, 4), device=dev).to(torch.float8_e4m3fn)
        mm = lambda: torch._scaled_mm(a, b.t(), scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16)  # noqa: E731
        mm()
        flush = torch.empty(128 * 1024 * 1024, dtype=torch.float32, device=dev)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ts = []
        for _ in range(iters):
            flush.zero_()
            s.record()
            mm()
            e.record()
            torch.cuda.synchronize()
            ts.append(s.elapsed_time(e))
        return 2.0 * M * N * K / (statistics.median(ts) * 1e-3) / 1e12
    except Exception:
        return None


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def workload_config(spec):
    return {"workload": f"{spec.name} fwd+bwd", "M_tokens_per_gpu": spec.M, "K": spec.K, "N": spec.N,
            "stabilizer_rank": spec.r_s, "lora_rank": spec.r,
            "l2": "flushed between steps (512 MiB write, outside the step events)"}


def cpu_baseline(spec, budget_s=12.0, rows=512):
    """The oracle timed on the host cores on a bounded sample (rank 0, N = 1)."""
    import torch  # noqa: F401

    from diffusion_dit_b200 import prep, workloads as wl
    from oracle import fourtune_oracle as ora
    inp = wl.make_layer_inputs(spec, seed=0, rows=rows)
    split = prep.svd_split(inp.w, spec.r_s)
    layer = ora.Layer(qr=ora.quantize_residual(split.residual), ls_up=split.ls_up, ls_down=split.ls_down,
                      lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)
    n, t0 = 0, time.perf_counter()
    while True:
        ora.linear_fwd(inp.x, layer)
        ora.linear_bwd(inp.x, inp.dy, layer)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = (time.perf_counter() - t0) / n
    fp4, bf = layer_flops(rows, spec.K, spec.N, spec.r_s, spec.r)
    return {"value": (fp4 + bf) / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} of {spec.M} tokens with the full weights, {n} oracle passes "
                      f"(quantize + fwd + bwd, fp64 products) in {time.perf_counter() - t0:.1f} s"}


def run_mlp_pair(args):
    """The MLP pair of a FLUX block (C3): FC1 4608 x 3072 -> 12288, GELU-tanh, FC2 12288 ->
    3072, forward and backward, with GELU and its derivative fused into the 4-bit GEMMs'
    epilogues (FC1's also takes max|H| for FC2's quantizer).  The unfused sequence (separate
    GELU kernels, FC2 taking its own max) is timed in the same run for comparison."""
    import torch

    from diffusion_dit_b200 import fourtune as ft
    from diffusion_dit_b200 import prep, workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    up, down = wl.FLUX_MLP_UP, wl.FLUX_MLP_DOWN
    M = up.M

    def weights(spec):
        inp = wl.make_layer_inputs(spec, seed=0)
        split = prep.svd_split(inp.w, spec.r_s)
        w = ft.prepare_weights(split.residual.to(dev), split.ls_up.to(dev), split.ls_down.to(dev),
                               inp.lora_a.to(dev), inp.lora_b.to(dev), spec.lora_scale)
        return inp, w

    inp_u, wu = weights(up)
    inp_d, wd = weights(down)
    wsu, wsd = ft.Workspace(wu, M, dev), ft.Workspace(wd, M, dev)
    x, dy = inp_u.x.to(dev), inp_d.dy.to(dev)
    bf, f32 = torch.bfloat16, torch.float32
    P = torch.empty(M, up.N, dtype=bf, device=dev)
    H = torch.empty(M, up.N, dtype=bf, device=dev)
    hmax = torch.empty(1, dtype=f32, device=dev)
    tu = torch.empty(M, up.r_s + up.r, dtype=f32, device=dev)
    td = torch.empty(M, down.r_s + down.r, dtype=f32, device=dev)
    Y = torch.empty(M, down.N, dtype=bf, device=dev)
    dP = torch.empty(M, up.N, dtype=bf, device=dev)
    dH = torch.empty(M, up.N, dtype=bf, device=dev)
    dX = torch.empty(M, up.K, dtype=bf, device=dev)
    dAu = torch.empty(up.r, up.K, dtype=f32, device=dev)
    dBu = torch.empty(up.N, up.r, dtype=f32, device=dev)
    dAd = torch.empty(down.r, down.K, dtype=f32, device=dev)
    dBd = torch.empty(down.N, down.r, dtype=f32, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=f32, device=dev)

    def fwd_fused():
        ft.linear_fwd_gelu(wu, x, wsu, p=P, h=H, h_amax=hmax, t_saved=tu)
        ft.linear_fwd(wd, H, wsd, y=Y, t_saved=td, amax=hmax)

    def bwd_fused():
        ft.linear_bwd_gelu(wd, H, td, dy, P, wsd, dp=dP, da=dAd, db=dBd)
        ft.linear_bwd(wu, x, tu, dP, wsu, dx=dX, da=dAu, db=dBu)

    def step_fused():
        fwd_fused()
        bwd_fused()

    def step_unfused():
        ft.linear_fwd(wu, x, wsu, y=P, t_saved=tu)
        ft.gelu_tanh_fwd(P, h=H)
        ft.linear_fwd(wd, H, wsd, y=Y, t_saved=td)
        ft.linear_bwd(wd, H, td, dy, wsd, dx=dH, da=dAd, db=dBd)
        ft.gelu_tanh_bwd(P, dH, dp=dP)
        ft.linear_bwd(wu, x, tu, dP, wsu, dx=dX, da=dAu, db=dBu)

    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    gev = [(E(), E()) for _ in range(4)]
    for b_, a_ in gev:
        b_.record()
        a_.record()
    torch.cuda.synchronize()

    def step_events():  # the four GEMM launches timed by the library, on the launch stream
        ft.time_next_launch(ft.FT_KERNEL_GEMM, *gev[0])
        ft.linear_fwd_gelu(wu, x, wsu, p=P, h=H, h_amax=hmax, t_saved=tu)
        ft.time_next_launch(ft.FT_KERNEL_GEMM, *gev[1])
        ft.linear_fwd(wd, H, wsd, y=Y, t_saved=td, amax=hmax)
        ft.time_next_launch(ft.FT_KERNEL_GEMM, *gev[2])
        ft.linear_bwd_gelu(wd, H, td, dy, P, wsd, dp=dP, da=dAd, db=dBd)
        ft.time_next_launch(ft.FT_KERNEL_GEMM, *gev[3])
        ft.linear_bwd(wu, x, tu, dP, wsu, dx=dX, da=dAu, db=dBu)

    graphs = {}
    for name, fn in (("fused", step_fused), ("unfused", step_unfused), ("fwd", fwd_fused), ("bwd", bwd_fused),
                     ("events", step_events)):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        c0 = ft.launch_count()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        graphs[name] = (g, ft.launch_count() - c0)
        for _ in range(args.warmup):
            flush.zero_()
            g.replay()
    torch.cuda.synchronize()
    if wsu.device_status() or wsd.device_status():
        raise RuntimeError("device status reports a timeout during warm-up")
    Kst = args.steps
    s_, e_ = E(), E()

    def timed(name):
        out = []
        for _ in range(Kst):
            flush.zero_()
            s_.record()
            graphs[name][0].replay()
            e_.record()
            torch.cuda.synchronize()
            out.append(s_.elapsed_time(e_))
        return out

    gemm_ms = []
    with ClockSampler(0) as clocks:
        fused = timed("fused")
        unfused = timed("unfused")
        fwd, bwd = timed("fwd"), timed("bwd")
        for _ in range(Kst):
            flush.zero_()
            graphs["events"][0].replay()
            torch.cuda.synchronize()
            gemm_ms.extend(b_.elapsed_time(a_) for b_, a_ in gev)
    if wsu.device_status() or wsd.device_status():
        raise RuntimeError("device status reports a timeout in the timed region")
    # end to end through the API: pinned host X and dY in, the four adapter gradients out
    x_h, dy_h = inp_u.x.pin_memory(), inp_d.dy.pin_memory()
    outs = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dAu, dBu, dAd, dBd)]
    e2e = []
    for _ in range(Kst):
        flush.zero_()
        s_.record()
        x.copy_(x_h, non_blocking=True)
        dy.copy_(dy_h, non_blocking=True)
        step_fused()
        for o, t in zip(outs, (dAu, dBu, dAd, dBd)):
            o.copy_(t, non_blocking=True)
        e_.record()
        torch.cuda.synchronize()
        e2e.append(s_.elapsed_time(e_))

    fu4, fub = layer_flops(M, up.K, up.N, up.r_s, up.r)
    fd4, fdb = layer_flops(M, down.K, down.N, down.r_s, down.r)
    flops = fu4 + fub + fd4 + fdb
    ms = statistics.mean(fused)
    ms_un = statistics.mean(unfused)
    f_u, b_u = pass_flops(M, up.K, up.N, up.r_s, up.r)
    f_d, b_d = pass_flops(M, down.K, down.N, down.r_s, down.r)
    hbm, bf16_peak, src = peaks()
    fp4_peak = bf16_peak * NOMINAL_FP4_OVER_BF16
    gemm_avg = statistics.mean(gemm_ms)
    achieved = (fu4 + fd4) / 4 / (gemm_avg * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": Kst,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4(e2m1,ue4m3)+bf16", "data": "synthetic",
        "config": {"workload": f"flux_mlp_pair {M}x{up.K}->{up.N}->{down.N} gelu_tanh fwd+bwd",
                   "M_tokens_per_gpu": M, "stabilizer_rank": up.r_s, "lora_rank": up.r,
                   "l2": "flushed between steps (512 MiB write, outside the step events)",
                   "parallelism": "dp1", "flops_per_step": {"fp4": fu4 + fd4, "bf16": fub + fdb}},
        "roofline": {"bound": "tensor", "kernel": "gemm_fp4_lowrank_pair_kernel (4 launches per step)",
                     "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                     "traffic": None, "frac_of_nominal_9pf": achieved / NOMINAL_FP4_TFLOPS,
                     "peak_source": f"{src} bf16 {bf16_peak} TFLOP/s x {NOMINAL_FP4_OVER_BF16}",
                     "avg_launch_ms": gemm_avg},
        "per_pass": {"fwd_ms": statistics.mean(fwd), "fwd_tflops": (f_u + f_d) / (statistics.mean(fwd) * 1e-3) / 1e12,
                     "bwd_ms": statistics.mean(bwd), "bwd_tflops": (b_u + b_d) / (statistics.mean(bwd) * 1e-3) / 1e12},
        "unfused": {"ms_per_step": ms_un, "value": flops / (ms_un * 1e-3) / 1e12,
                    "speedup_of_fusion": ms_un / ms,
                    "what": "separate GELU and GELU-backward kernels, FC2 takes its own max|H|"},
        "e2e": {"value": flops / (statistics.mean(e2e) * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": x.numel() * 2 + dy.numel() * 2,
                "d2h_bytes_per_step": sum(t.numel() * 4 for t in (dAu, dBu, dAd, dBd))},
        "gpu_launches": graphs["fused"][1] * Kst, "launch_mode": "cuda_graph_replay",
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=256)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="replay each step as a captured CUDA graph (default)")
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--workload", default="qkv", choices=sorted(WORKLOADS) + ["mlp"],
                    help="single-layer workload (default: the attention QKV projection), or mlp: "
                         "the MLP pair with GELU, fused")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.workload == "mlp" and args.impl == "ours":
        if int(os.environ.get("WORLD_SIZE", "1")) > 1:
            raise SystemExit("--workload mlp runs on one GPU")
        run_mlp_pair(args)
        return

    from diffusion_dit_b200 import workloads as wl
    spec = getattr(wl, WORKLOADS.get(args.workload, "FLUX_MLP_UP"))
    if args.impl == "reference":
        run_reference(args, spec)
        return

    import torch
    import torch.distributed as dist

    from diffusion_dit_b200 import fourtune as ft
    from diffusion_dit_b200 import dp, prep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # --- setup (untimed): inputs of this rank's shard, offline weight prep ------
    inp = wl.make_layer_inputs(spec, seed=rank)
    split = prep.svd_split(inp.w, spec.r_s)
    w = ft.prepare_weights(split.residual.to(dev), split.ls_up.to(dev), split.ls_down.to(dev),
                           inp.lora_a.to(dev), inp.lora_b.to(dev), spec.lora_scale)
    M, K, N = spec.M, spec.K, spec.N
    R = spec.r_s + spec.r
    ws = ft.Workspace(w, M, dev)
    x = inp.x.to(dev)
    dy = inp.dy.to(dev)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    t = torch.empty(M, R, dtype=torch.float32, device=dev)
    dx = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    da = torch.empty(spec.r, K, dtype=torch.float32, device=dev)
    db = torch.empty(N, spec.r, dtype=torch.float32, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step_kernels():
        ft.linear_fwd(w, x, ws, y=y, t_saved=t)
        ft.linear_bwd(w, x, t, dy, ws, dx=dx, da=da, db=db)

    def step():
        step_kernels()
        if world > 1:
            dp.allreduce_adapter_grads(da, db)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if ws.device_status() != 0:
        raise RuntimeError("device status reports a timeout during warm-up")

    Kst = args.steps
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev_s, ev_e = [E() for _ in range(Kst)], [E() for _ in range(Kst)]
    # per-launch events of the dominant kernel (the 4-bit GEMM: forward and dX), the
    # quantizer and the tensor max; the library records them on the launch stream
    kev = {k: ([E(), E()], [E(), E()]) for k in (ft.FT_KERNEL_GEMM, ft.FT_KERNEL_QUANT, ft.FT_KERNEL_AMAX)}
    for ev in ev_s + ev_e + [e for b_, a_ in kev.values() for e in b_ + a_]:
        ev.record()  # torch creates the CUDA event on first record; the library needs the handle
    torch.cuda.synchronize()

    def one_step_with_events():
        for k, (b_, a_) in kev.items():
            ft.time_next_launch(k, b_[0], a_[0])
        ft.linear_fwd(w, x, ws, y=y, t_saved=t)
        # the backward has no separate tensor-max launch: its adapter-gradient kernel
        # takes max |G| on the way
        for k in (ft.FT_KERNEL_GEMM, ft.FT_KERNEL_QUANT):
            ft.time_next_launch(k, kev[k][0][1], kev[k][1][1])
        ft.linear_bwd(w, x, t, dy, ws, dx=dx, da=da, db=db)

    def fwd_kernels():
        ft.linear_fwd(w, x, ws, y=y, t_saved=t)

    def fwd_1x16_kernels():  # X quantized group-wise 1x16 (the Table 5 comparison, forward only)
        ft.linear_fwd_1x16(w, x, ws, y=y, t_saved=t)

    def bwd_kernels():
        ft.linear_bwd(w, x, t, dy, ws, dx=dx, da=da, db=db)

    # the same layer with Q(R)^T's codes dropped: the dX GEMM transposes Q(R) on the fly
    w_xp = ft.drop_transposed_codes(w)
    xp_ev = (E(), E())
    for ev in xp_ev:
        ev.record()

    def bwd_xpose_kernels():
        ft.linear_bwd(w_xp, x, t, dy, ws, dx=dx, da=da, db=db)

    def bwd_xpose_with_events():  # the dX GEMM is the backward's last GEMM launch
        ft.time_next_launch(ft.FT_KERNEL_GEMM, xp_ev[0], xp_ev[1])
        ft.linear_bwd(w_xp, x, t, dy, ws, dx=dx, da=da, db=db)

    graph = graph_k = graph_f = graph_b = graph_f1 = graph_bx = graph_bxk = None
    launches_per_step = None
    if args.graph:
        # One step (forward + backward: all of the library's kernels) captured once as a
        # CUDA graph and replayed: the same kernels, without the host launch gaps between
        # them.  A second capture adds the per-launch timing events (graph event-record
        # nodes); those serialise the kernels around them and cost ~50 us per step, so the
        # headline steps replay the graph without them and a second pass of as many steps
        # replays the instrumented one to time the kernels.
        c0 = ft.launch_count()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step_kernels()
        launches_per_step = ft.launch_count() - c0
        graph_k = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_k):
            one_step_with_events()
        # forward alone and backward alone, for the per-pass figures
        graph_f, graph_b, graph_f1 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_f):
            fwd_kernels()
        with torch.cuda.graph(graph_b):
            bwd_kernels()
        fwd_1x16_kernels()
        with torch.cuda.graph(graph_f1):
            fwd_1x16_kernels()
        bwd_xpose_kernels()
        graph_bx, graph_bxk = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_bx):
            bwd_xpose_kernels()
        with torch.cuda.graph(graph_bxk):
            bwd_xpose_with_events()
        for _ in range(args.warmup):
            for g_ in (graph, graph_k, graph_f, graph_b, graph_f1, graph_bx, graph_bxk):
                flush.zero_()
                g_.replay()
        torch.cuda.synchronize()

    gemm_ms, quant_ms, amax_ms = [], [], []
    ev_ks, ev_ke = [E() for _ in range(Kst)], [E() for _ in range(Kst)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = ft.launch_count()
    with ClockSampler(local) as clocks:
        for i in range(Kst):
            flush.zero_()
            ev_s[i].record()
            if graph is not None:
                graph.replay()
            else:
                step_kernels()
            if world > 1:
                dp.allreduce_adapter_grads(da, db)
            ev_e[i].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        launches = (launches_per_step * Kst) if graph is not None else ft.launch_count() - launches0
        # kernel-timing pass: the same steps with per-launch events on the launch stream
        for i in range(Kst):
            flush.zero_()
            ev_ks[i].record()
            if graph_k is not None:
                graph_k.replay()
            else:
                one_step_with_events()
            ev_ke[i].record()
            # the per-launch events are reused by every step: read them before the next one
            torch.cuda.synchronize()
            for k, dst in ((ft.FT_KERNEL_GEMM, gemm_ms), (ft.FT_KERNEL_QUANT, quant_ms)):
                b_, a_ = kev[k]
                dst.extend([b_[0].elapsed_time(a_[0]), b_[1].elapsed_time(a_[1])])
            amax_ms.append(kev[ft.FT_KERNEL_AMAX][0][0].elapsed_time(kev[ft.FT_KERNEL_AMAX][1][0]))
        torch.cuda.synchronize()
        ms_per_step_events = sum(ev_ks[i].elapsed_time(ev_ke[i]) for i in range(Kst)) / Kst
        # per-pass pass: the forward alone, then the backward alone, as many steps each
        pass_ms = {"fwd": [], "bwd": [], "fwd_1x16": [], "bwd_xpose": []}
        for name, g_, fn in (("fwd", graph_f, fwd_kernels), ("bwd", graph_b, bwd_kernels),
                             ("fwd_1x16", graph_f1, fwd_1x16_kernels),
                             ("bwd_xpose", graph_bx, bwd_xpose_kernels)):
            for i in range(Kst):
                flush.zero_()
                ev_ks[i].record()
                if g_ is not None:
                    g_.replay()
                else:
                    fn()
                ev_ke[i].record()
            torch.cuda.synchronize()
            pass_ms[name] = [ev_ks[i].elapsed_time(ev_ke[i]) for i in range(Kst)]
        # the transposing dX GEMM alone, by its launch events
        xp_gemm_ms = []
        for i in range(Kst):
            flush.zero_()
            if graph_bxk is not None:
                graph_bxk.replay()
            else:
                bwd_xpose_with_events()
            torch.cuda.synchronize()
            xp_gemm_ms.append(xp_ev[0].elapsed_time(xp_ev[1]))
    if ws.device_status() != 0:
        raise RuntimeError("device status reports a timeout in the timed region")

    total_ms = sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(Kst))
    tm = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
    total_ms = float(tm.item())
    ms_per_step = total_ms / Kst
    fp4, bf = layer_flops(M, K, N, spec.r_s, spec.r)
    value = world * (fp4 + bf) * Kst / (total_ms * 1e-3) / 1e12

    # --- end to end through the API with host buffers (pinned), copies timed ---
    x_h = inp.x.pin_memory()
    dy_h = inp.dy.pin_memory()
    da_h = torch.empty(da.shape, dtype=da.dtype).pin_memory()
    db_h = torch.empty(db.shape, dtype=db.dtype).pin_memory()
    e_s, e_e = [E() for _ in range(Kst)], [E() for _ in range(Kst)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(Kst):
        flush.zero_()
        e_s[i].record()
        x.copy_(x_h, non_blocking=True)
        dy.copy_(dy_h, non_blocking=True)
        ft.linear_fwd(w, x, ws, y=y, t_saved=t)
        ft.linear_bwd(w, x, t, dy, ws, dx=dx, da=da, db=db)
        if world > 1:
            dp.allreduce_adapter_grads(da, db)
        da_h.copy_(da, non_blocking=True)
        db_h.copy_(db, non_blocking=True)
        e_e[i].record()
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([sum(e_s[i].elapsed_time(e_e[i]) for i in range(Kst))], dtype=torch.float64,
                          device=dev)
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    e2e_value = world * (fp4 + bf) * Kst / (float(e2e_ms.item()) * 1e-3) / 1e12
    h2d = x.numel() * 2 + dy.numel() * 2
    d2h = da.numel() * 4 + db.numel() * 4

    if rank == 0:
        hbm, bf16_peak, src = peaks()
        fp4_peak = bf16_peak * NOMINAL_FP4_OVER_BF16
        gemm_avg = statistics.mean(gemm_ms)
        achieved = 2.0 * M * N * K / (gemm_avg * 1e-3) / 1e12
        # ncu dram read + write per launch (mean of fwd and dX), captured on this workload
        traffic = gemm_traffic() if args.workload == "qkv" else None
        # quantizer: X [M, K] and G [M, N] alternate; algorithmic bytes per element:
        # 2 (read bf16) + 0.5 (codes) + 1/256 (block scales).  The tensor max of X is one
        # more read of X, by the forward's prologue kernel (which also builds the low-rank
        # factors: its whole duration counts); max |G| is taken by the dB kernel.
        elems = [M * K, M * N] * Kst
        qbytes = sum(e * (2.0 + 0.5 + 1.0 / 256) for e in elems)
        q_gbs = qbytes / (sum(quant_ms) * 1e-3) / 1e9
        qa_gbs = (qbytes + 2.0 * M * K * Kst) / ((sum(quant_ms) + sum(amax_ms)) * 1e-3) / 1e9
        fl_f, fl_b = pass_flops(M, K, N, spec.r_s, spec.r)
        fwd_ms, bwd_ms = statistics.median(pass_ms["fwd"]), statistics.median(pass_ms["bwd"])
        lt_fwd = cublaslt_nvfp4_tflops(M, N, K)
        lt_dx = cublaslt_nvfp4_tflops(M, K, N)
        lt_mean = (lt_fwd + lt_dx) / 2 if lt_fwd and lt_dx else None
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": Kst,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4(e2m1,ue4m3)+bf16", "data": "synthetic",
            "config": dict(workload_config(spec), parallelism=f"dp{world}",
                           flops_per_step={"fp4": fp4, "bf16": bf}),
            "roofline": {"bound": "tensor", "kernel": "gemm_fp4_lowrank_pair_kernel (fwd and dX)",
                         "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": achieved / fp4_peak, "traffic": traffic,
                         "peak_source": f"{src} bf16 {bf16_peak} TFLOP/s x {NOMINAL_FP4_OVER_BF16} "
                                        f"(nominal fp4/bf16 ratio)",
                         "avg_launch_ms": gemm_avg,
                         "frac_of_nominal_9pf": achieved / NOMINAL_FP4_TFLOPS,
                         "cublaslt_nvfp4_tflops": {"fwd_shape": lt_fwd, "dx_shape": lt_dx},
                         "frac_of_cublaslt": achieved / lt_mean if lt_mean else None,
                         "timing": "CUDA events around each launch, recorded in a second pass of "
                                   f"{Kst} steps (that pass: {ms_per_step_events:.4f} ms per step)"},
            "quantizer": {"kernel": "quant_down_kernel (quantizer fused with the down-projection)", "achieved_gbs": q_gbs,
                          "with_amax_pass_gbs": qa_gbs, "peak_gbs": hbm, "frac": q_gbs / hbm,
                          "frac_with_amax": qa_gbs / hbm, "avg_launch_ms": statistics.mean(quant_ms)},
            "per_pass": {"fwd_ms": fwd_ms, "fwd_tflops": fl_f / (fwd_ms * 1e-3) / 1e12,
                         "bwd_ms": bwd_ms, "bwd_tflops": fl_b / (bwd_ms * 1e-3) / 1e12,
                         "fwd_1x16_ms": statistics.median(pass_ms["fwd_1x16"]),
                         "timing": f"median of {Kst} replays of a forward-only / backward-only graph"},
            "xpose_on_the_fly": {
                "what": "backward with Q(R)^T's codes dropped: the dX GEMM transposes Q(R)'s tiles in "
                        "shared memory (section 3.2)",
                "bwd_ms": statistics.median(pass_ms["bwd_xpose"]), "bwd_ms_stored_copy": bwd_ms,
                "dx_gemm_ms": statistics.mean(xp_gemm_ms),
                "dx_gemm_ms_stored_copy": statistics.mean(gemm_ms[1::2]),
                "bytes_saved": N * K // 2 + N * K // 256},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "launch_mode": "cuda_graph_replay" if graph is not None else "stream",
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(spec)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
