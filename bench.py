"""Benchmark of the W4A4G4 triple-branch linear layer (FourTune, arXiv 2607.05711).

One step = the whole hot path once over one batch, for every layer of the workload: the
forward (tensor max, 16x16 block quantization of X fused with the low-rank down-
projection, the 4-bit GEMM with the up-projections in its accumulator) and the backward
(the same for G, the dX GEMM through Q(R)^T, the adapter gradients dA, dB).  Default
workload: the linears of a FLUX.1-dev single-stream block at batch 2 x 4608 tokens --
linear1 9216 x 3072 -> 21504 (fused QKV + MLP-up) and linear2 9216 x 15360 -> 3072,
stabilizer rank 32, LoRA rank 64 -- forward through both, then backward through both,
synthetic inputs (independent per layer) and random-init weights of that shape
(workloads.py).  The same line carries the quantizer-only sweep (16x16-block quantizer
with its fused rank-32 down-projection, bf16 4608x3072 ... 36864x21504) in GB/s against
HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload single|qkv|mlp|mlp_up|mlp_down|single_l1|single_l2]
                    [--scaling weak|strong] [--tokens M] [--profile]
                    [--no-cpu-baseline] [--no-quant-sweep]

N > 1 runs data-parallel under torchrun: each rank processes its own batch (weak
scaling), or a token shard of one batch with --scaling strong, and the adapter
gradients are summed with an NCCL all-reduce.  The reference arm
times the CPU oracle (the only reference this method has) on a bounded sample of the same
workload.  --tokens M replaces the token count (a smaller case for profilers);
--profile runs the plain step only (no graphs, no side measurements), for ncu.  One JSON
line on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
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

# workload -> (description, layer specs in forward order); "mlp" is the fused MLP pair
WORKLOADS = {
    "single": ("flux_single_stream_block linear1 9216x3072->21504 + linear2 9216x15360->3072",
               ["FLUX_SS_L1", "FLUX_SS_L2"]),
    "qkv": ("flux_qkv 4608x3072->9216", ["FLUX_QKV"]),
    "mlp_up": ("flux_mlp_up 4608x3072->12288", ["FLUX_MLP_UP"]),
    "mlp_down": ("flux_mlp_down 4608x12288->3072", ["FLUX_MLP_DOWN"]),
    "single_l1": ("flux_single_l1 9216x3072->21504", ["FLUX_SS_L1"]),
    "single_l2": ("flux_single_l2 9216x15360->3072", ["FLUX_SS_L2"]),
}
DEFAULT_WORKLOAD = "single"

# ncu DRAM read + write per launch of the 4-bit GEMM (mean over the step's GEMM launches)
# on a workload, with the hash of the GEMM's sources the counters were taken from: the
# figure is reported only while the sources still hash to that value.
GEMM_DRAM_BYTES = {"single": (271287232, "6b406da2ee05d402")}
GEMM_SOURCES = ("ft_gemm2.cu", "ft_ptx.cuh")


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
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained under the power cap, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def gemm_roofline_peak(clock_summary):
    """The FP4 peak a GEMM timed in this run is held against: the measured bf16 peak x the
    nominal FP4/bf16 ratio, sustained if the clock samples of the timed region saw the
    power cap (the kernel then ran inside a long, power-capped loop), else burst."""
    _, burst, sustained, src = peaks()
    capped = "sw_power_cap" in (clock_summary.get("reasons") or [])
    bf16 = sustained if capped else burst
    return (bf16 * NOMINAL_FP4_OVER_BF16, burst * NOMINAL_FP4_OVER_BF16, sustained * NOMINAL_FP4_OVER_BF16,
            f"{src} bf16 {'sustained' if capped else 'burst'} {bf16} TFLOP/s x {NOMINAL_FP4_OVER_BF16} (nominal "
            f"fp4/bf16 ratio; sustained when the timed region ran under sw_power_cap)")


def gemm_sources_hash():
    src = b"".join(open(os.path.join(ROOT, "diffusion_dit_b200", "csrc", f), "rb").read() for f in GEMM_SOURCES)
    return hashlib.sha256(src).hexdigest()[:16]


def gemm_traffic(workload):
    rec = GEMM_DRAM_BYTES.get(workload)
    if not rec or rec[1] != gemm_sources_hash():
        return None
    return rec[0]


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


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count() or 1


def specs_of(args):
    from diffusion_dit_b200 import workloads as wl
    desc, names = WORKLOADS[args.workload]
    specs = [getattr(wl, n) for n in names]
    if args.tokens:
        import dataclasses
        specs = [dataclasses.replace(s, name=f"{s.name}@M{args.tokens}", M=args.tokens) for s in specs]
        desc = f"{desc} with M={args.tokens} tokens"
    return desc, specs


def workload_config(args, desc, specs):
    return {"workload": f"{desc}, fwd+bwd", "layers": [
        {"name": s.name, "M": s.M, "K": s.K, "N": s.N, "stabilizer_rank": s.r_s, "lora_rank": s.r}
        for s in specs], "M_tokens_per_gpu": specs[0].M,
        "l2": "flushed between steps (512 MiB write, outside the step events); the single-stream "
              "layers' operands are larger than L2"}


def oracle_layers(specs, splits, rows):
    """The oracle's view of each layer on a bounded token sample (the full weights)."""
    from diffusion_dit_b200 import workloads as wl
    from oracle import fourtune_oracle as ora
    out = []
    for spec, split in zip(specs, splits):
        inp = wl.make_layer_inputs(spec, seed=0, rows=rows)
        layer = ora.Layer(qr=ora.quantize_residual(split.residual), ls_up=split.ls_up, ls_down=split.ls_down,
                          lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)
        out.append((inp, layer))
    return out


def oracle_pass(layers):
    from oracle import fourtune_oracle as ora
    for inp, layer in layers:
        ora.linear_fwd(inp.x, layer)
    for inp, layer in reversed(layers):
        ora.linear_bwd(inp.x, inp.dy, layer)


def sample_flops(specs, rows):
    return sum(sum(layer_flops(rows, s.K, s.N, s.r_s, s.r)) for s in specs)


def run_reference(args, desc, specs):
    """The reference arm: the CPU oracle as it stands, on a bounded token sample."""
    from diffusion_dit_b200 import prep
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    rows = args.ref_rows
    from diffusion_dit_b200 import workloads as wl
    splits = [prep.svd_split(wl.make_layer_inputs(s, seed=0, rows=rows).w, s.r_s) for s in specs]
    layers = oracle_layers(specs, splits, rows)
    threads = blas_threads()
    for _ in range(args.warmup):
        oracle_pass(layers)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_pass(layers)
    dt = (time.perf_counter() - t0) / args.steps
    value = sample_flops(specs, rows) / dt / 1e12
    sample = (f"{rows} tokens of each layer's {specs[0].M}, full weights; oracle quantize + fwd + bwd "
              f"(fp64 products) through every layer")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args, desc, specs),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline(specs, splits, budget_s=12.0, rows=128):
    """The oracle timed on the host cores on a bounded sample (rank 0, N = 1)."""
    layers = oracle_layers(specs, splits, rows)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_pass(layers)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = (time.perf_counter() - t0) / n
    return {"value": sample_flops(specs, rows) / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{rows} of {specs[0].M} tokens of every layer with the full weights, {n} oracle passes "
                      f"(quantize + fwd + bwd, fp64 products) in {time.perf_counter() - t0:.1f} s"}


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


def cublaslt_nvfp4_sustained_tflops(M, N, K, seconds=0.4):
    """The same cuBLASLt GEMM back to back for ~`seconds` (no flush), timed over the last
    launches: its rate under the power cap, as a GEMM inside a long step runs."""
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
        torch.cuda.synchronize()
        t_end = time.time() + seconds
        while time.time() < t_end:
            for _ in range(8):
                mm()
            torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(20):
            mm()
        e.record()
        torch.cuda.synchronize()
        return 2.0 * M * N * K / (s.elapsed_time(e) / 20 * 1e-3) / 1e12
    except Exception:
        return None


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
    clock_summary = clocks.summary()
    fp4_peak, fp4_burst, fp4_sustained, peak_src = gemm_roofline_peak(clock_summary)
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
                     "traffic": None, "frac_of_burst_peak": achieved / fp4_burst,
                     "frac_of_sustained_peak": achieved / fp4_sustained,
                     "frac_of_nominal_9pf": achieved / NOMINAL_FP4_TFLOPS,
                     "peak_source": peak_src, "avg_launch_ms": gemm_avg},
        "per_pass": {"fwd_ms": statistics.mean(fwd), "fwd_tflops": (f_u + f_d) / (statistics.mean(fwd) * 1e-3) / 1e12,
                     "bwd_ms": statistics.mean(bwd), "bwd_tflops": (b_u + b_d) / (statistics.mean(bwd) * 1e-3) / 1e12},
        "unfused": {"ms_per_step": ms_un, "value": flops / (ms_un * 1e-3) / 1e12,
                    "speedup_of_fusion": ms_un / ms,
                    "what": "separate GELU and GELU-backward kernels, FC2 takes its own max|H|"},
        "e2e": {"value": flops / (statistics.mean(e2e) * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": x.numel() * 2 + dy.numel() * 2,
                "d2h_bytes_per_step": sum(t.numel() * 4 for t in (dAu, dBu, dAd, dBd))},
        "gpu_launches": graphs["fused"][1] * Kst, "launch_mode": "cuda_graph_replay",
        "clocks": clock_summary,
    }
    print(json.dumps(line), flush=True)


class LayerRun:
    """One layer of the step: its weights (prepared once, offline), workspace, synthetic
    inputs resident on the device, and outputs."""

    def __init__(self, spec, dev, seed, weight_spec=None, weight_seed=None):
        """spec: this rank's shape (its token count M); the frozen weights and the adapter
        are drawn from weight_spec / weight_seed (the same on every rank: they are
        replicated), the inputs X and dY from spec / seed."""
        import torch

        from diffusion_dit_b200 import fourtune as ft
        from diffusion_dit_b200 import prep, workloads as wl
        self.spec = spec
        inp = wl.make_layer_inputs(spec, seed=seed)
        wdraw = inp if weight_spec is None else wl.make_layer_inputs(weight_spec, seed=weight_seed)
        self.inp = inp
        self.split = prep.svd_split(wdraw.w, spec.r_s)
        self.w = ft.prepare_weights(self.split.residual.to(dev), self.split.ls_up.to(dev),
                                    self.split.ls_down.to(dev), wdraw.lora_a.to(dev), wdraw.lora_b.to(dev),
                                    spec.lora_scale)
        self.w_xp = ft.drop_transposed_codes(self.w)
        M, K, N, R = spec.M, spec.K, spec.N, spec.r_s + spec.r
        self.ws = ft.Workspace(self.w, M, dev)
        self.x = inp.x.to(dev)
        self.dy = inp.dy.to(dev)
        bf, f32 = torch.bfloat16, torch.float32
        self.y = torch.empty(M, N, dtype=bf, device=dev)
        self.t = torch.empty(M, R, dtype=f32, device=dev)
        self.dx = torch.empty(M, K, dtype=bf, device=dev)
        self.da = torch.empty(spec.r, K, dtype=f32, device=dev)
        self.db = torch.empty(N, spec.r, dtype=f32, device=dev)

    def fwd(self, x1x16=False):
        from diffusion_dit_b200 import fourtune as ft
        (ft.linear_fwd_1x16 if x1x16 else ft.linear_fwd)(self.w, self.x, self.ws, y=self.y, t_saved=self.t)

    def bwd(self, xpose=False):
        from diffusion_dit_b200 import fourtune as ft
        ft.linear_bwd(self.w_xp if xpose else self.w, self.x, self.t, self.dy, self.ws, dx=self.dx, da=self.da,
                      db=self.db)

    def flops(self):
        s = self.spec
        return layer_flops(s.M, s.K, s.N, s.r_s, s.r)


def quant_sweep(dev, warmup, reps, flush):
    """The quantizer-only workload: Q(x) in 16x16 blocks with the fused rank-32
    down-projection x A^T, on bf16 inputs of the sweep's shapes, through
    fourtune_quantize_block16.  Timed as a CUDA graph of the whole call: with the call's
    own tensor max (one extra read of x), and with a caller-supplied max; and the fused
    quantizer kernel alone, by its launch events.  GB/s = algorithmic bytes (read x 2 B,
    write codes 0.5 B and block scales 1/256 B per element, x A^T 4 B per row and rank)
    / time; with the max pass, 2 B more per element."""
    import torch

    from diffusion_dit_b200 import fourtune as ft
    from diffusion_dit_b200 import workloads as wl
    hbm = peaks()[0]
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    out = []
    for qs in wl.QUANT_SWEEP:
        x, down = wl.make_quant_input(qs, seed=0)
        x, down = x.to(dev), down.to(dev)
        rows, cols, r = qs.rows, qs.cols, qs.r_down
        q = ft.QuantizedMatrix.empty(rows, cols, dev, with_sf=False)
        t = torch.empty(rows, r, dtype=torch.float32, device=dev)
        amax = x.abs().amax().float().reshape(1)
        nws = ft.lib().fourtune_quantize_workspace_bytes(rows, cols, r)
        ws = torch.zeros(nws, dtype=torch.uint8, device=dev)

        def call(given):
            ft.quantize_block16_into(x, q, ws, amax=amax if given else None, down=down, down_out=t)

        kev = (E(), E())
        for e in kev:
            e.record()
        torch.cuda.synchronize()

        def call_events():
            ft.time_next_launch(ft.FT_KERNEL_QUANT, *kev)
            call(False)

        graphs = {}
        for name, fn in (("own_max", lambda: call(False)), ("given_max", lambda: call(True)),
                         ("events", call_events)):
            fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            for _ in range(warmup):
                flush.zero_()
                g.replay()
            graphs[name] = g
        torch.cuda.synchronize()
        s_, e_ = E(), E()
        res = {}
        for name in ("own_max", "given_max", "events"):
            ts = []
            for _ in range(reps):
                flush.zero_()
                s_.record()
                graphs[name].replay()
                e_.record()
                torch.cuda.synchronize()
                ts.append(kev[0].elapsed_time(kev[1]) if name == "events" else s_.elapsed_time(e_))
            res[name] = statistics.median(ts)
        n = rows * cols
        base = n * (2.0 + 0.5 + 1.0 / 256) + rows * r * 4.0
        entry = {"shape": [rows, cols], "r_down": r,
                 "call_ms": res["own_max"], "call_gbs": (base + 2.0 * n) / (res["own_max"] * 1e-3) / 1e9,
                 "call_given_max_ms": res["given_max"],
                 "call_given_max_gbs": base / (res["given_max"] * 1e-3) / 1e9,
                 "kernel_ms": res["events"], "kernel_gbs": base / (res["events"] * 1e-3) / 1e9}
        entry["frac_call"] = entry["call_gbs"] / hbm
        entry["frac_call_given_max"] = entry["call_given_max_gbs"] / hbm
        entry["frac_kernel"] = entry["kernel_gbs"] / hbm
        out.append(entry)
        del graphs, x, down, q, t, ws
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return {"what": "fourtune_quantize_block16 with the fused rank-32 down-projection, bf16 inputs "
                    "~N(0,1) with 1% Laplace(10) entries; median of replays with L2 flushed; "
                    "call = the whole entry point (tensor max pass, factor prologue, fused quantizer, "
                    "split sum), given_max = the same with the caller's max, kernel = the fused "
                    "quantizer launch alone (launch events)",
            "peak_gbs": hbm, "shapes": out}


def run_layers(args, desc, specs):
    import torch
    import torch.distributed as dist

    from diffusion_dit_b200 import dp
    from diffusion_dit_b200 import fourtune as ft

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # --- setup (untimed): this rank's synthetic inputs, offline weight prep -------------
    # Weak scaling: every rank a full batch of the workload.  Strong scaling: the ranks
    # split the workload's batch into token shards (dp.token_shard, multiples of the pair
    # GEMM's 256 rows).  The frozen weights and the adapter are the same on every rank.
    import dataclasses
    rank_specs = specs
    if args.scaling == "strong" and world > 1:
        lo, hi = dp.token_shard(specs[0].M, world, rank, multiple=256)
        rank_specs = [dataclasses.replace(s, M=hi - lo) for s in specs]
    layers = [LayerRun(rs, dev, seed=1000 + 31 * rank + i, weight_spec=s, weight_seed=17 * i)
              for i, (rs, s) in enumerate(zip(rank_specs, specs))]
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step_kernels(x1x16=False, xpose=False, fwd=True, bwd=True):
        if fwd:
            for L in layers:
                L.fwd(x1x16)
        if bwd:
            for L in reversed(layers):
                L.bwd(xpose)

    def allreduce():
        for L in reversed(layers):
            dp.allreduce_adapter_grads(L.da, L.db)

    def step():
        step_kernels()
        if world > 1:
            allreduce()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if any(L.ws.device_status() for L in layers):
        raise RuntimeError("device status reports a timeout during warm-up")

    Kst = args.steps
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    fp4 = sum(L.flops()[0] for L in layers)
    bf = sum(L.flops()[1] for L in layers)
    # whole-job FLOPs per step: every rank's own batch (weak) or the one global batch (strong)
    if args.scaling == "strong":
        job_flops = sum(sum(layer_flops(s.M, s.K, s.N, s.r_s, s.r)) for s in specs)
    else:
        job_flops = world * (fp4 + bf)

    if args.profile:
        # the plain step, eagerly, for profilers: no graphs, no side measurements
        s_, e_ = E(), E()
        torch.cuda.synchronize()
        s_.record()
        for _ in range(Kst):
            step()
        e_.record()
        torch.cuda.synchronize()
        ms = s_.elapsed_time(e_) / Kst
        if rank == 0:
            print(json.dumps({"profile": True, "workload": desc, "ms_per_step_eager": ms,
                              "value_eager": job_flops / (ms * 1e-3) / 1e12}), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    # per-launch events: every GEMM and quantizer launch of one step (and the forward
    # prologue that takes max|X|), recorded by the library on the launch stream
    GEMM, QUANT, AMAX = ft.FT_KERNEL_GEMM, ft.FT_KERNEL_QUANT, ft.FT_KERNEL_AMAX
    LOWRANK, DB, DA = ft.FT_KERNEL_LOWRANK, ft.FT_KERNEL_LORA_DB, ft.FT_KERNEL_LORA_DA
    nL = len(layers)
    kev = {(k, i): (E(), E()) for k in (GEMM, QUANT, LOWRANK) for i in range(2 * nL)}
    kev.update({(k, i): (E(), E()) for k in (AMAX, DB, DA) for i in range(nL)})
    xp_ev = [(E(), E()) for _ in range(nL)]
    for ev in [e for p_ in list(kev.values()) + xp_ev for e in p_]:
        ev.record()  # torch creates the CUDA event on first record; the library needs the handle
    torch.cuda.synchronize()

    def step_with_events():
        for i, L in enumerate(layers):
            for k in (GEMM, QUANT, LOWRANK):
                ft.time_next_launch(k, *kev[(k, i)])
            ft.time_next_launch(AMAX, *kev[(AMAX, i)])
            L.fwd()
        for j, L in enumerate(reversed(layers)):
            for k in (GEMM, QUANT, LOWRANK):
                ft.time_next_launch(k, *kev[(k, nL + j)])
            for k in (DB, DA):
                ft.time_next_launch(k, *kev[(k, j)])
            L.bwd()

    def bwd_xpose_with_events():  # each layer's dX GEMM is its backward's last GEMM launch
        for j, L in enumerate(reversed(layers)):
            ft.time_next_launch(GEMM, *xp_ev[j])
            L.bwd(xpose=True)

    # Each pass is captured once as a CUDA graph and replayed: the same kernels without
    # the host launch gaps.  Event-record nodes between kernels serialise them (~50 us per
    # step), so the headline steps replay graphs without them and a second pass of as many
    # steps replays the instrumented one to time the kernels.
    variants = {"step": step_kernels, "events": step_with_events,
                "fwd": lambda: step_kernels(bwd=False), "bwd": lambda: step_kernels(fwd=False),
                "fwd_1x16": lambda: step_kernels(x1x16=True, bwd=False),
                "bwd_xpose": lambda: step_kernels(xpose=True, fwd=False), "bwd_xpose_events": bwd_xpose_with_events}
    graphs, launches_per_step = {}, None
    if args.graph:
        for name, fn in variants.items():
            fn()
            torch.cuda.synchronize()
            c0 = ft.launch_count()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            if name == "step":
                launches_per_step = ft.launch_count() - c0
            graphs[name] = g
        for _ in range(args.warmup):
            for g in graphs.values():
                flush.zero_()
                g.replay()
        torch.cuda.synchronize()

    def run(name):
        if name in graphs:
            graphs[name].replay()
        else:
            variants[name]()

    ev_s, ev_e = [E() for _ in range(Kst)], [E() for _ in range(Kst)]
    gemm_ms, quant_ms, amax_ms, xp_gemm_ms, other_ms = [], [], [], [], []
    pass_ms = {}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = ft.launch_count()
    with ClockSampler(local) as clocks:
        for i in range(Kst):
            flush.zero_()
            ev_s[i].record()
            run("step")
            if world > 1:
                allreduce()
            ev_e[i].record()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        launches = (launches_per_step * Kst) if launches_per_step is not None else ft.launch_count() - launches0
        total_ms = sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(Kst))
        # kernel-timing pass: the same steps with per-launch events on the launch stream
        ev_k = []
        for i in range(Kst):
            flush.zero_()
            ev_s[i].record()
            run("events")
            ev_e[i].record()
            torch.cuda.synchronize()  # the per-launch events are reused: read them now
            ev_k.append(ev_s[i].elapsed_time(ev_e[i]))
            gemm_ms.append([kev[(GEMM, j)][0].elapsed_time(kev[(GEMM, j)][1]) for j in range(2 * nL)])
            quant_ms.append([kev[(QUANT, j)][0].elapsed_time(kev[(QUANT, j)][1]) for j in range(2 * nL)])
            amax_ms.append([kev[(AMAX, j)][0].elapsed_time(kev[(AMAX, j)][1]) for j in range(nL)])
            other_ms.append({name: [kev[(k, j)][0].elapsed_time(kev[(k, j)][1]) for j in range(n)]
                             for name, k, n in (("lowrank_finalize", LOWRANK, 2 * nL), ("lora_grad_db", DB, nL),
                                                ("lora_grad_da", DA, nL))})
        # per-pass figures: forward alone, backward alone, 1x16 forward, transposing backward
        for name in ("fwd", "bwd", "fwd_1x16", "bwd_xpose"):
            ts = []
            for i in range(Kst):
                flush.zero_()
                ev_s[i].record()
                run(name)
                ev_e[i].record()
            torch.cuda.synchronize()
            pass_ms[name] = statistics.median(ev_s[i].elapsed_time(ev_e[i]) for i in range(Kst))
        for i in range(Kst):
            flush.zero_()
            run("bwd_xpose_events")
            torch.cuda.synchronize()
            xp_gemm_ms.append([b_.elapsed_time(a_) for b_, a_ in xp_ev])
    if any(L.ws.device_status() for L in layers):
        raise RuntimeError("device status reports a timeout in the timed region")

    tm = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tm, op=dist.ReduceOp.MAX)
    total_ms = float(tm.item())
    ms_per_step = total_ms / Kst
    value = job_flops * Kst / (total_ms * 1e-3) / 1e12

    # --- end to end through the API: every layer's X and dY copied in from pinned host
    # memory, dA and dB copied out, inside the timed region ----------------------------
    hx = [L.inp.x.pin_memory() for L in layers]
    hdy = [L.inp.dy.pin_memory() for L in layers]
    hda = [torch.empty(L.da.shape, dtype=L.da.dtype).pin_memory() for L in layers]
    hdb = [torch.empty(L.db.shape, dtype=L.db.dtype).pin_memory() for L in layers]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # The copies in go on a second stream in the order the step needs them (each layer's X
    # for the forward, then each dY in the backward's layer order) and the step waits for
    # each just before its first use, so later copies overlap earlier layers' kernels.  A
    # step's copies start only after the previous step is done with the buffers.
    copy_stream = torch.cuda.Stream(device=dev)
    main = torch.cuda.current_stream()
    need = [(L, "x") for L in layers] + [(L, "dy") for L in reversed(layers)]
    host = {id(L.x): a for L, a in zip(layers, hx)}
    host.update({id(L.dy): b for L, b in zip(layers, hdy)})
    for i in range(Kst):
        flush.zero_()
        ev_s[i].record()
        copy_stream.wait_stream(main)
        ready = {}
        with torch.cuda.stream(copy_stream):
            for L, name in need:
                t = getattr(L, name)
                t.copy_(host[id(t)], non_blocking=True)
                ready[(id(L), name)] = torch.cuda.Event()
                ready[(id(L), name)].record(copy_stream)
        for L in layers:
            main.wait_event(ready[(id(L), "x")])
            L.fwd()
        for L in reversed(layers):
            main.wait_event(ready[(id(L), "dy")])
            L.bwd()
        if world > 1:
            allreduce()
        for L, a, b in zip(layers, hda, hdb):
            a.copy_(L.da, non_blocking=True)
            b.copy_(L.db, non_blocking=True)
        ev_e[i].record()
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(Kst))], dtype=torch.float64,
                          device=dev)
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
    e2e_value = job_flops * Kst / (float(e2e_ms.item()) * 1e-3) / 1e12
    h2d = sum(L.x.numel() * 2 + L.dy.numel() * 2 for L in layers)
    d2h = sum(L.da.numel() * 4 + L.db.numel() * 4 for L in layers)

    if rank == 0:
        hbm = peaks()[0]
        clock_summary = clocks.summary()
        fp4_peak, fp4_burst, fp4_sustained, peak_src = gemm_roofline_peak(clock_summary)
        # the GEMM launches of a step, in order: each layer's forward, then the backward's
        # dX GEMMs in reverse layer order; FLOPs 2 M N K each
        gemm_flops = [2.0 * L.spec.M * L.spec.N * L.spec.K for L in layers + list(reversed(layers))]
        gemm_avg = statistics.mean(sum(r) for r in gemm_ms) / len(gemm_flops)
        achieved = statistics.mean(gemm_flops) / (gemm_avg * 1e-3) / 1e12
        per_launch = []
        names = [f"{L.spec.name} fwd" for L in layers] + [f"{L.spec.name} dX" for L in reversed(layers)]
        specs_order = [L.spec for L in layers] + [L.spec for L in reversed(layers)]
        shapes = [(s.M, s.N, s.K) if j < nL else (s.M, s.K, s.N) for j, s in enumerate(specs_order)]
        # every shape's burst figure before any sustained loop (which leaves the GPU power-capped)
        lt = {shape: cublaslt_nvfp4_tflops(*shape) for shape in dict.fromkeys(shapes)}
        lts = {shape: cublaslt_nvfp4_sustained_tflops(*shape) for shape in dict.fromkeys(shapes)}
        for j, (nm, shape) in enumerate(zip(names, shapes)):
            ms_j = statistics.mean(r[j] for r in gemm_ms)
            per_launch.append({"launch": nm, "M_N_K": list(shape), "ms": ms_j,
                               "tflops": gemm_flops[j] / (ms_j * 1e-3) / 1e12, "cublaslt_tflops": lt[shape],
                               "cublaslt_sustained_tflops": lts[shape]})

        def lt_frac(key):  # cuBLASLt's time for the step's GEMM FLOPs over ours
            if not all(p[key] for p in per_launch):
                return None
            t = sum(gemm_flops[j] / (p[key] * 1e12) for j, p in enumerate(per_launch))
            return t * 1e3 / sum(p["ms"] for p in per_launch)
        # quantizer launches: X of each layer (forward), G of each layer (backward)
        q_elems = [L.spec.M * L.spec.K for L in layers] + [L.spec.M * L.spec.N for L in reversed(layers)]
        q_rank = [L.spec.r_s + L.spec.r for L in layers] + [L.spec.r_s + L.spec.r for L in reversed(layers)]
        q_rows = [L.spec.M for L in layers] + [L.spec.M for L in reversed(layers)]
        q_bytes = [e * (2.0 + 0.5 + 1.0 / 256) + m * r * 4.0 for e, m, r in zip(q_elems, q_rows, q_rank)]
        q_ms = [statistics.mean(r[j] for r in quant_ms) for j in range(2 * nL)]
        q_gbs = sum(q_bytes) / (sum(q_ms) * 1e-3) / 1e9
        a_ms = [statistics.mean(r[j] for r in amax_ms) for j in range(nL)]
        qa_gbs = (sum(q_bytes) + sum(2.0 * L.spec.M * L.spec.K for L in layers)) / \
            ((sum(q_ms) + sum(a_ms)) * 1e-3) / 1e9
        fl_f = sum(pass_flops(L.spec.M, L.spec.K, L.spec.N, L.spec.r_s, L.spec.r)[0] for L in layers)
        fl_b = sum(pass_flops(L.spec.M, L.spec.K, L.spec.N, L.spec.r_s, L.spec.r)[1] for L in layers)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": Kst,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if args.scaling == "strong" and world > 1 else "weak",
            "vs_baseline": None, "dtype": "nvfp4(e2m1,ue4m3)+bf16", "data": "synthetic",
            "config": dict(workload_config(args, desc, specs), parallelism=f"dp{world}",
                           M_tokens_per_gpu=layers[0].spec.M,
                           flops_per_step_per_gpu={"fp4": fp4, "bf16": bf}),
            "roofline": {"bound": "tensor", "kernel": "gemm_fp4_lowrank_pair_kernel (every forward and dX GEMM)",
                         "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": achieved / fp4_peak, "traffic": gemm_traffic(args.workload),
                         "peak_source": peak_src,
                         "avg_launch_ms": gemm_avg,
                         "frac_of_burst_peak": achieved / fp4_burst,
                         "frac_of_sustained_peak": achieved / fp4_sustained,
                         "frac_of_nominal_9pf": achieved / NOMINAL_FP4_TFLOPS,
                         "frac_of_cublaslt": lt_frac("cublaslt_tflops"),
                         "frac_of_cublaslt_sustained": lt_frac("cublaslt_sustained_tflops"),
                         "cublaslt": "torch._scaled_mm NVFP4 (bf16 out) at each launch's M, N, K: cublaslt_tflops "
                                     "with L2 flushed between launches (burst); cublaslt_sustained_tflops back "
                                     "to back for 0.4 s, under the power cap",
                         "launches": per_launch,
                         "timing": "CUDA events around each launch, recorded in a second pass of "
                                   f"{Kst} steps (that pass: {statistics.mean(ev_k):.4f} ms per step)"},
            "quantizer": {"kernel": "quant_down_kernel (quantizer fused with the down-projection)",
                          "achieved_gbs": q_gbs, "with_amax_pass_gbs": qa_gbs, "peak_gbs": hbm,
                          "frac": q_gbs / hbm, "frac_with_amax": qa_gbs / hbm,
                          "launch_ms": q_ms, "amax_pass_ms": a_ms,
                          "bytes_per_element": "2 (read) + 0.5 (codes) + 1/256 (block scales), + 4 R per row"},
            "other_kernels_ms": {name: [statistics.mean(r[name][j] for r in other_ms)
                                        for j in range(len(other_ms[0][name]))] for name in other_ms[0]},
            "per_pass": {"fwd_ms": pass_ms["fwd"], "fwd_tflops": fl_f / (pass_ms["fwd"] * 1e-3) / 1e12,
                         "bwd_ms": pass_ms["bwd"], "bwd_tflops": fl_b / (pass_ms["bwd"] * 1e-3) / 1e12,
                         "fwd_1x16_ms": pass_ms["fwd_1x16"],
                         "timing": f"median of {Kst} replays of a forward-only / backward-only graph"},
            "xpose_on_the_fly": {
                "what": "backward with Q(R)^T's codes dropped: the dX GEMM transposes Q(R)'s tiles in "
                        "shared memory (section 3.2)",
                "bwd_ms": pass_ms["bwd_xpose"], "bwd_ms_stored_copy": pass_ms["bwd"],
                "dx_gemm_ms": [statistics.mean(r[j] for r in xp_gemm_ms) for j in range(nL)],
                "dx_gemm_ms_stored_copy": [statistics.mean(r[nL + j] for r in gemm_ms) for j in range(nL)],
                "bytes_saved": sum(L.spec.N * L.spec.K // 2 + L.spec.N * L.spec.K // 256 for L in layers)},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "what": "each step copies every layer's X and dY in from pinned host memory (on a second "
                            "stream, each waited for just before its first use, so later copies overlap earlier "
                            "layers' kernels) and its dA and dB out; Y and dX stay on the device (in a training "
                            "step they are the next layer's input and the previous layer's gradient)"},
            "gpu_launches": launches,
            "launch_mode": "cuda_graph_replay" if graphs else "stream",
            "clocks": clock_summary,
        }
        if world == 1 and not args.no_quant_sweep:
            line["quantizer_sweep"] = quant_sweep(dev, args.warmup, min(Kst, 20), flush)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(specs, [L.split for L in layers])
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-quant-sweep", action="store_true")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="replay each step as a captured CUDA graph (default)")
    ap.add_argument("--no-graph", dest="graph", action="store_false")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS) + ["mlp"],
                    help="default: the FLUX single-stream block's two linears; mlp: the MLP pair with "
                         "GELU, fused")
    ap.add_argument("--tokens", type=int, default=0, help="replace the token count M (multiple of 256)")
    ap.add_argument("--profile", action="store_true", help="plain eager steps only (for profilers)")
    ap.add_argument("--scaling", default="weak", choices=["weak", "strong"],
                    help="N > 1: every rank its own batch (weak, default) or token shards of one batch (strong)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.tokens and args.tokens % 256:
        raise SystemExit("--tokens must be a multiple of 256")
    if args.workload == "mlp" and args.impl == "ours":
        if int(os.environ.get("WORLD_SIZE", "1")) > 1:
            raise SystemExit("--workload mlp runs on one GPU")
        run_mlp_pair(args)
        return
    if args.workload == "mlp":
        args.workload = "mlp_up"  # the reference arm of the pair: its first layer
    desc, specs = specs_of(args)
    if args.impl == "reference":
        run_reference(args, desc, specs)
        return
    run_layers(args, desc, specs)


if __name__ == "__main__":
    main()
