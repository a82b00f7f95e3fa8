"""GPU W4A4G4 linear vs the oracle: forward Eq. (2), backward Eq. (3), adapter gradients
(FourTune section 3.2).  Tolerance: relative Frobenius error <= 2e-3 against the
oracle's fp64 products over the same dequantized operands (Y and dX are bf16, whose
own rounding contributes ~1.7e-3 for Gaussian-like data)."""
import functools

import numpy as np
import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


@functools.lru_cache(maxsize=4)
def _setup(spec: wl.LayerSpec, seed: int = 0):
    """Inputs, the oracle's SVD split and layer, and the GPU weights built from the same
    split (the two paths consume the same R and stabilizer factors)."""
    ft = _ft()
    inp = wl.make_layer_inputs(spec, seed=seed)
    split = ora.svd_split(inp.w, spec.r_s)
    layer = ora.Layer(qr=ora.quantize_residual(split.r), ls_up=split.ls_up, ls_down=split.ls_down,
                      lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)
    w = ft.prepare_weights(split.r.cuda(), split.ls_up.cuda(), split.ls_down.cuda(), inp.lora_a.cuda(),
                           inp.lora_b.cuda(), spec.lora_scale)
    return inp, layer, w


MID = wl.LayerSpec(name="mid_384x1024x768", M=384, K=1024, N=768, r_s=16, r=16, alpha=32.0,
                   n_outlier_cols=5, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                   b_std=0.01, dy_std=1e-2)


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_prepared_residual_codes_match_oracle(spec):
    inp, layer, w = _setup(spec)
    assert w.qr.g.item() == np.float32(layer.qr.g)
    assert np.array_equal(w.qr.codes.cpu().numpy(), layer.qr.codes)
    assert np.array_equal(w.qr.scales.cpu().numpy(), layer.qr.scales)
    qt = layer.qr.transpose()
    assert np.array_equal(w.qr_t.codes.cpu().numpy(), qt.codes)
    assert np.array_equal(w.qr_t.scales.cpu().numpy(), qt.scales)


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_forward_matches_oracle(spec):
    ft = _ft()
    inp, layer, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    y, t = ft.linear_fwd(w, inp.x.cuda(), ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    ref = ora.linear_fwd(inp.x, layer)
    err_y = ora.rel_frobenius(y.double().cpu().numpy(), ref.y)
    err_t = ora.rel_frobenius(t.double().cpu().numpy(), ref.t)
    assert err_t < 1e-5, err_t
    assert err_y < TOL, err_y


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_backward_matches_oracle(spec):
    ft = _ft()
    inp, layer, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    x = inp.x.cuda()
    _, t = ft.linear_fwd(w, x, ws)
    dx, da, db = ft.linear_bwd(w, x, t, inp.dy.cuda(), ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    ref = ora.linear_bwd(inp.x, inp.dy, layer)
    e_dx = ora.rel_frobenius(dx.double().cpu().numpy(), ref.dx)
    e_da = ora.rel_frobenius(da.double().cpu().numpy(), ref.da)
    e_db = ora.rel_frobenius(db.double().cpu().numpy(), ref.db)
    assert e_dx < TOL, e_dx
    assert e_da < TOL, e_da
    assert e_db < TOL, e_db


def test_backbone_only_gemm_is_a_block_scaled_fp4_product():
    # r_s = 0 and B = 0: Y is the plain 4-bit product of the dequantized operands.
    ft = _ft()
    spec = MID
    inp, layer, _ = _setup(spec)
    z_b = torch.zeros_like(inp.lora_b)
    w0 = ft.prepare_weights(layer_r := ora.svd_split(inp.w, 0).r.cuda(),
                            torch.zeros(spec.N, 0, dtype=torch.bfloat16, device="cuda"),
                            torch.zeros(0, spec.K, dtype=torch.bfloat16, device="cuda"),
                            inp.lora_a.cuda(), z_b.cuda(), 1.0)
    ws = ft.Workspace(w0, spec.M, "cuda")
    y, _ = ft.linear_fwd(w0, inp.x.cuda(), ws)
    xh = ora.quantize_block16(inp.x).dequantize()
    rh = ora.quantize_block16(layer_r.cpu()).dequantize()
    assert ora.rel_frobenius(y.double().cpu().numpy(), xh @ rh.T) < TOL


def test_repeated_calls_are_deterministic():
    ft = _ft()
    inp, layer, w = _setup(MID)
    ws = ft.Workspace(w, MID.M, "cuda")
    x, dy = inp.x.cuda(), inp.dy.cuda()
    y1, t1 = ft.linear_fwd(w, x, ws)
    dx1, da1, db1 = ft.linear_bwd(w, x, t1, dy, ws)
    y1, dx1, da1, db1 = y1.clone(), dx1.clone(), da1.clone(), db1.clone()
    y2, t2 = ft.linear_fwd(w, x, ws)
    dx2, da2, db2 = ft.linear_bwd(w, x, t2, dy, ws)
    assert torch.equal(y1, y2) and torch.equal(dx1, dx2)
    assert torch.equal(da1, da2) and torch.equal(db1, db2)


# r = 32 with K = 2048: dA's and dB's split sums are too much work for the dX GEMM's
# epilogue warps before its first tile (N = 512: two k steps), so they run in a launch of
# their own; the gradients must meet the same bar.
WIDE_R = wl.LayerSpec(name="wide_r_256x2048x512", M=256, K=2048, N=512, r_s=16, r=32, alpha=32.0,
                      n_outlier_cols=10, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                      b_std=0.01, dy_std=1e-2)


def test_backward_with_separate_split_sums_matches_oracle():
    test_backward_matches_oracle(WIDE_R)


def test_given_max_equal_to_the_true_max_gives_the_same_forward():
    # the prologue's per-CTA maxima (reduced by the quantizer) and a caller's max of the
    # same value are two routes to one g: Y and T must agree bit for bit
    ft = _ft()
    inp, _, w = _setup(MID)
    ws = ft.Workspace(w, MID.M, "cuda")
    x = inp.x.cuda()
    y0, t0 = ft.linear_fwd(w, x, ws)
    y0, t0 = y0.clone(), t0.clone()
    amax = x.float().abs().max().reshape(1)
    y1, t1 = ft.linear_fwd(w, x, ws, amax=amax)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    assert torch.equal(y0, y1) and torch.equal(t0, t1)


# M = 384 (one-CTA GEMM kernel) with split sums small enough for its epilogue warps
# ((N + K) r = 12288 outputs; N = 1024: four k steps in the dX GEMM's first tile)
SIDE_ONE_CTA = wl.LayerSpec(name="side_one_cta_384x512x1024", M=384, K=512, N=1024, r_s=16, r=8, alpha=8.0,
                            n_outlier_cols=3, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                            b_std=0.01, dy_std=1e-2)


def test_backward_one_cta_gemm_with_side_split_sums_matches_oracle():
    test_backward_matches_oracle(SIDE_ONE_CTA)
