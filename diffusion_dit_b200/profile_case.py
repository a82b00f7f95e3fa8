"""Runs the layer's forward + backward a few times on a chosen shape, for profilers.

    python -m diffusion_dit_b200.profile_case [--M 2048] [--K 3072] [--N 9216]
        [--r_s 32] [--r 16] [--steps 3]

Used for ncu captures that need a smaller case than the benchmark workload (the
default keeps the FLUX QKV projection's K and N with fewer tokens: a few hundred MB
on the device, still larger than L2 so DRAM counters mean something).
"""
from __future__ import annotations

import argparse

import torch

from diffusion_dit_b200 import fourtune as ft
from diffusion_dit_b200 import prep
from diffusion_dit_b200 import workloads as wl


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--K", type=int, default=3072)
    ap.add_argument("--N", type=int, default=9216)
    ap.add_argument("--r_s", type=int, default=32)
    ap.add_argument("--r", type=int, default=16)
    ap.add_argument("--steps", type=int, default=3)
    a = ap.parse_args()
    spec = wl.flux_layer("profile_case", a.M, a.K, a.N, a.r_s, a.r)
    inp = wl.make_layer_inputs(spec, seed=0)
    split = prep.svd_split(inp.w, spec.r_s)
    dev = torch.device("cuda", 0)
    w = ft.prepare_weights(split.residual.to(dev), split.ls_up.to(dev), split.ls_down.to(dev),
                           inp.lora_a.to(dev), inp.lora_b.to(dev), spec.lora_scale)
    ws = ft.Workspace(w, spec.M, dev)
    x, dy = inp.x.to(dev), inp.dy.to(dev)
    for _ in range(a.steps):
        _, t = ft.linear_fwd(w, x, ws)
        ft.linear_bwd(w, x, t, dy, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    print("profile_case done")


if __name__ == "__main__":
    main()
