"""GELU fused into the 4-bit GEMM's epilogues (FourTune section 3.3, "MLP Fusion").
Forward: fourtune_linear_fwd_gelu must give exactly what the unfused path gives -- the
layer output P of fourtune_linear_fwd, H = the stand-alone GELU kernel applied to P, and
max |H| as the max kernel would take it -- and a next layer fed that max must produce the
same bits as one that takes its own.  Backward: fourtune_linear_bwd_gelu must write the
same bits as fourtune_linear_bwd followed by the stand-alone GELU-backward kernel.  Both
GEMM kernels are covered (CTA pairs when M % 256 == 0, single CTAs otherwise)."""
import functools

import numpy as np
import pytest
import torch

from diffusion_dit_b200 import prep
from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora

pytestmark = pytest.mark.gpu

MID = wl.LayerSpec(name="mid_384x1024x768", M=384, K=1024, N=768, r_s=16, r=16, alpha=32.0,
                   n_outlier_cols=5, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                   b_std=0.01, dy_std=1e-2)


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


@functools.lru_cache(maxsize=3)
def _setup(spec: wl.LayerSpec):
    ft = _ft()
    inp = wl.make_layer_inputs(spec, seed=0)
    split = prep.svd_split(inp.w, spec.r_s)
    w = ft.prepare_weights(split.residual.cuda(), split.ls_up.cuda(), split.ls_down.cuda(),
                           inp.lora_a.cuda(), inp.lora_b.cuda(), spec.lora_scale)
    return inp, w


def _check_fused_equals_unfused(spec):
    ft = _ft()
    inp, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    x = inp.x.cuda()
    y, t = ft.linear_fwd(w, x, ws)
    y, t = y.clone(), t.clone()
    p, h, h_amax, t2 = ft.linear_fwd_gelu(w, x, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    assert torch.equal(p, y), "P differs from the unfused forward's output"
    assert torch.equal(t2, t)
    h_ref = ft.gelu_tanh_fwd(p)
    torch.cuda.synchronize()
    assert torch.equal(h, h_ref), "H differs from the stand-alone GELU kernel"
    assert h_amax.item() == h.float().abs().max().item()
    return p, h, h_amax


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_fused_gelu_forward_equals_unfused(spec):
    p, h, _ = _check_fused_equals_unfused(spec)
    # and H against the oracle's GELU of the same P: within one bf16 step per element
    P = p.float().cpu().numpy().astype(np.float64)
    H = h.float().cpu().numpy().astype(np.float64)
    Href = ora.gelu_tanh(P)
    step = np.abs(torch.from_numpy(Href).to(torch.bfloat16).float().numpy().astype(np.float64))
    step = np.maximum(step * 2.0 ** -7, 2.0 ** -133)
    assert np.all(np.abs(H - Href) <= step)


def test_fused_gelu_full_size_mlp_up_then_down():
    ft = _ft()
    up, down = wl.FLUX_MLP_UP, wl.FLUX_MLP_DOWN
    p, h, h_amax = _check_fused_equals_unfused(up)
    _, wd = _setup(down)
    ws = ft.Workspace(wd, down.M, "cuda")
    y_own, t_own = ft.linear_fwd(wd, h, ws)
    y_own, t_own = y_own.clone(), t_own.clone()
    y_fed, t_fed = ft.linear_fwd(wd, h, ws, amax=h_amax)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    assert torch.equal(y_fed, y_own)
    assert torch.equal(t_fed, t_own)


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_fused_gelu_backward_equals_unfused(spec):
    ft = _ft()
    inp, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    x, dy = inp.x.cuda(), inp.dy.cuda()
    # a pre-activation P of the layer's input shape [M, K]: bf16 values around the GELU's
    # curved region, with zeros, negatives and a few large magnitudes
    g = torch.Generator().manual_seed(7)
    p = (torch.randn(spec.M, spec.K, generator=g) * 2.0).to(torch.bfloat16)
    p[0, :8] = 0.0
    p[1, :8] = torch.tensor([-12.0, -6.0, -0.75, 0.5, 3.0, 9.0, -1e-3, 1e-3]).to(torch.bfloat16)
    p = p.cuda()
    _, t = ft.linear_fwd(w, x, ws)
    t = t.clone()
    dx, da, db = ft.linear_bwd(w, x, t, dy, ws)
    dx, da, db = dx.clone(), da.clone(), db.clone()
    dp_ref = ft.gelu_tanh_bwd(p, dx)
    dp, da2, db2 = ft.linear_bwd_gelu(w, x, t, dy, p, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    assert torch.equal(dp, dp_ref), "dP differs from dX followed by the GELU-backward kernel"
    assert torch.equal(da2, da) and torch.equal(db2, db)
