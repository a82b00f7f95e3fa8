"""GPU W4A4G4 linear vs the oracle: forward Eq. (2), backward Eq. (3), adapter gradients
(FourTune section 3.2).

Two levels, both against the oracle's fp64 products over the same dequantized operands:
  * the bar: relative Frobenius error <= 2e-3 for Y, dX, dA and dB (Y and dX are bf16,
    whose own rounding contributes ~1.7e-3 of that for Gaussian-like data);
  * element by element for the bf16 outputs Y and dX: within one bf16 ulp of the oracle's
    value rounded to bf16, plus the fp32 accumulation allowance of each element
    (tests/parity.py), and within FROB_ROUNDED of bf16(oracle) in relative Frobenius norm.
Edge cases through the layer calls: X = 0, G = 0, no adapter (r = 0), no stabilizer
(r_s = 0), a caller's tensor max above the true one, and seeds 1 and 2 of the small layer.
"""
import functools

import numpy as np
import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora
from tests import parity

pytestmark = pytest.mark.gpu

TOL = 2e-3
# relative Frobenius distance of a bf16 output from the correctly rounded oracle value
FROB_ROUNDED = 2e-4


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


def _oracle_layer(spec: wl.LayerSpec, inp, split):
    return ora.Layer(qr=ora.quantize_residual(split.r), ls_up=split.ls_up, ls_down=split.ls_down,
                     lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)


@functools.lru_cache(maxsize=6)
def _setup(spec: wl.LayerSpec, seed: int = 0):
    """Inputs, the oracle's SVD split and layer, and the GPU weights built from the same
    split (the two paths consume the same R and stabilizer factors)."""
    ft = _ft()
    inp = wl.make_layer_inputs(spec, seed=seed)
    split = ora.svd_split(inp.w, spec.r_s)
    layer = _oracle_layer(spec, inp, split)
    w = ft.prepare_weights(split.r.cuda(), split.ls_up.cuda(), split.ls_down.cuda(), inp.lora_a.cuda(),
                           inp.lora_b.cuda(), spec.lora_scale)
    return inp, layer, w


def _np(t):
    return t.double().cpu().numpy()


def check_forward(x, layer, y, t, amax=None):
    fr = ora.linear_fwd(x, layer, amax_x=amax)
    st = parity.compare_bf16("y", _np(y), fr.y, parity.fwd_allowance(x, layer, fr))
    parity.assert_bf16_parity(st, FROB_ROUNDED, TOL)
    if t is not None and fr.t.size:
        err_t = ora.rel_frobenius(_np(t)[:, : fr.t.shape[1]], fr.t)
        assert err_t < 1e-5, err_t
    return fr, st


def check_backward(x, dy, layer, dx, da, db, amax=None):
    br = ora.linear_bwd(x, dy, layer, amax_g=amax)
    st = parity.compare_bf16("dx", _np(dx), br.dx, parity.bwd_allowance(dy, layer, br))
    parity.assert_bf16_parity(st, FROB_ROUNDED, TOL)
    if layer.r:
        e_da = ora.rel_frobenius(_np(da), br.da)
        e_db = ora.rel_frobenius(_np(db), br.db)
        assert e_da < TOL, e_da
        assert e_db < TOL, e_db
    return br, st


MID = wl.LayerSpec(name="mid_384x1024x768", M=384, K=1024, N=768, r_s=16, r=16, alpha=32.0,
                   n_outlier_cols=5, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                   b_std=0.01, dy_std=1e-2)

# M = 1408 (11 x 128, not a multiple of 256): the one-CTA GEMM kernel with more tiles than
# SMs (11 x 16 = 176 forward tiles, 11 x 4 dX tiles of 128 x 256), so CTAs loop over
# several tiles and the accumulator hand-off runs between them
ONE_CTA_MANY = wl.LayerSpec(name="one_cta_many_1408x1024x4096", M=1408, K=1024, N=4096, r_s=16, r=16,
                            alpha=32.0, n_outlier_cols=5, outlier_gain=20.0, w_std=0.02, plant_rank=4,
                            plant_sigma=6.0, b_std=0.01, dy_std=1e-2)

CASES = [(wl.PARITY_SMALL, 0), (wl.PARITY_SMALL, 1), (wl.PARITY_SMALL, 2), (MID, 0), (ONE_CTA_MANY, 0)]
IDS = [f"{s.name}-seed{k}" for s, k in CASES]


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_prepared_residual_codes_match_oracle(spec):
    inp, layer, w = _setup(spec)
    assert w.qr.g.item() == np.float32(layer.qr.g)
    assert np.array_equal(w.qr.codes.cpu().numpy(), layer.qr.codes)
    assert np.array_equal(w.qr.scales.cpu().numpy(), layer.qr.scales)
    qt = layer.qr.transpose()
    assert np.array_equal(w.qr_t.codes.cpu().numpy(), qt.codes)
    assert np.array_equal(w.qr_t.scales.cpu().numpy(), qt.scales)


@pytest.mark.parametrize("spec,seed", CASES, ids=IDS)
def test_forward_matches_oracle(spec, seed):
    ft = _ft()
    inp, layer, w = _setup(spec, seed)
    ws = ft.Workspace(w, spec.M, "cuda")
    y, t = ft.linear_fwd(w, inp.x.cuda(), ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    check_forward(inp.x, layer, y, t)


@pytest.mark.parametrize("spec,seed", CASES, ids=IDS)
def test_backward_matches_oracle(spec, seed):
    ft = _ft()
    inp, layer, w = _setup(spec, seed)
    ws = ft.Workspace(w, spec.M, "cuda")
    x = inp.x.cuda()
    _, t = ft.linear_fwd(w, x, ws)
    dx, da, db = ft.linear_bwd(w, x, t, inp.dy.cuda(), ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    check_backward(inp.x, inp.dy, layer, dx, da, db)


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


def _bwd_launches(spec, seed=0):
    """Kernels one backward call launches (7 with dA's and dB's split sums in a launch of
    their own, 6 when the dX GEMM's epilogue warps run them)."""
    ft = _ft()
    inp, _, w = _setup(spec, seed)
    ws = ft.Workspace(w, spec.M, "cuda")
    x = inp.x.cuda()
    _, t = ft.linear_fwd(w, x, ws)
    c0 = ft.launch_count()
    ft.linear_bwd(w, x, t, inp.dy.cuda(), ws)
    torch.cuda.synchronize()
    return ft.launch_count() - c0


# r = 32 with K = 2048: dA's and dB's split sums are too much work for the dX GEMM's
# epilogue warps before its first tile (N = 512: two k steps), so they run in a launch of
# their own; the gradients must meet the same bar.
WIDE_R = wl.LayerSpec(name="wide_r_256x2048x512", M=256, K=2048, N=512, r_s=16, r=32, alpha=32.0,
                      n_outlier_cols=10, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                      b_std=0.01, dy_std=1e-2)


def test_backward_with_separate_split_sums_matches_oracle():
    assert _bwd_launches(WIDE_R) == 7
    test_backward_matches_oracle(WIDE_R, 0)


# N = 4096 (17 k steps in the dX GEMM's first tile) with r = 8 and enough GEMM CTAs (M = 1024,
# K = 2048: 32 pair tiles, 8192 epilogue threads): the split sums fit on the pair GEMM's
# epilogue warps before their first accumulator
SIDE_PAIR = wl.LayerSpec(name="side_pair_1024x2048x4096", M=1024, K=2048, N=4096, r_s=16, r=8, alpha=8.0,
                         n_outlier_cols=3, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                         b_std=0.01, dy_std=1e-2)


def test_backward_pair_gemm_with_side_split_sums_matches_oracle():
    assert _bwd_launches(SIDE_PAIR) == 6
    test_backward_matches_oracle(SIDE_PAIR, 0)


# r = 64 (V' 128 columns wide, as in the FLUX single-stream layers) at sizes the oracle
# checks in full: the adapter-gradient schedule with token ranges only (8 and 6 tiles,
# split over up to 8 token ranges), and with whole tiles then split ones (N = 19200:
# 150 tiles on 148 SMs).
WIDE_LORA_SPLIT = wl.LayerSpec(name="wide_lora_split_512x1024x768", M=512, K=1024, N=768, r_s=16, r=64,
                               alpha=64.0, n_outlier_cols=5, outlier_gain=20.0, w_std=0.02, plant_rank=4,
                               plant_sigma=6.0, b_std=0.01, dy_std=1e-2)
WIDE_LORA_FULL = wl.LayerSpec(name="wide_lora_full_256x512x19200", M=256, K=512, N=19200, r_s=16, r=64,
                              alpha=64.0, n_outlier_cols=3, outlier_gain=20.0, w_std=0.02, plant_rank=4,
                              plant_sigma=6.0, b_std=0.01, dy_std=1e-2)


@pytest.mark.parametrize("spec", [WIDE_LORA_SPLIT, WIDE_LORA_FULL], ids=lambda s: s.name)
def test_backward_rank_64_adapter_gradients(spec):
    test_backward_matches_oracle(spec, 0)


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
# ((N + K) r = 69632 outputs; N = 8192: 32 k steps in the dX GEMM's first tile)
SIDE_ONE_CTA = wl.LayerSpec(name="side_one_cta_384x512x8192", M=384, K=512, N=8192, r_s=16, r=8, alpha=8.0,
                            n_outlier_cols=3, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                            b_std=0.01, dy_std=1e-2)


def test_backward_one_cta_gemm_with_side_split_sums_matches_oracle():
    assert _bwd_launches(SIDE_ONE_CTA) == 6
    test_backward_matches_oracle(SIDE_ONE_CTA, 0)


# ---------------------------------------------------------------- edge cases of the layer

def test_zero_input_gives_zero_output_and_zero_adapter_gradients():
    # X = 0: max|X| = 0, so g = 1 and every code and scale is 0 (the quantizer's degenerate
    # case); T = 0, so Y = 0 exactly; dA = s (G B)^T X = 0 and dB = s G^T (X A^T) = 0
    # exactly, while dX still carries the backward of G.
    ft = _ft()
    spec = MID
    inp, layer, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    x0 = torch.zeros_like(inp.x)
    y, t = ft.linear_fwd(w, x0.cuda(), ws)
    dx, da, db = ft.linear_bwd(w, x0.cuda(), t, inp.dy.cuda(), ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    assert not torch.any(y) and not torch.any(t)
    assert not torch.any(da) and not torch.any(db)
    check_backward(x0, inp.dy, layer, dx, da, db)


def test_zero_gradient_gives_zero_gradients():
    ft = _ft()
    spec = MID
    inp, layer, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    x = inp.x.cuda()
    _, t = ft.linear_fwd(w, x, ws)
    dx, da, db = ft.linear_bwd(w, x, t, torch.zeros_like(inp.dy).cuda(), ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    assert not torch.any(dx) and not torch.any(da) and not torch.any(db)


def _variant(spec, inp, split, *, no_lora=False, no_stab=False):
    """The layer with the adapter (r = 0) or the stabilizer (r_s = 0) removed."""
    ft = _ft()
    a, b = inp.lora_a, inp.lora_b
    if no_lora:
        a, b = a[:0].contiguous(), b[:, :0].contiguous()
    ls_up, ls_down, r = split.ls_up, split.ls_down, split.r
    if no_stab:
        s0 = ora.svd_split(inp.w, 0)
        ls_up, ls_down, r = s0.ls_up, s0.ls_down, s0.r
    layer = ora.Layer(qr=ora.quantize_residual(r), ls_up=ls_up, ls_down=ls_down, lora_a=a, lora_b=b,
                      lora_scale=spec.lora_scale)
    w = ft.prepare_weights(r.cuda(), ls_up.cuda(), ls_down.cuda(), a.cuda(), b.cuda(), spec.lora_scale)
    return layer, w


@pytest.mark.parametrize("which", ["no_lora", "no_stabilizer"])
def test_layer_without_one_low_rank_branch(which):
    ft = _ft()
    spec = MID
    inp = wl.make_layer_inputs(spec, seed=0)
    split = ora.svd_split(inp.w, spec.r_s)
    layer, w = _variant(spec, inp, split, no_lora=which == "no_lora", no_stab=which == "no_stabilizer")
    ws = ft.Workspace(w, spec.M, "cuda")
    x, dy = inp.x.cuda(), inp.dy.cuda()
    y, t = ft.linear_fwd(w, x, ws)
    dx, da, db = ft.linear_bwd(w, x, t, dy, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    check_forward(inp.x, layer, y, t)
    check_backward(inp.x, inp.dy, layer, dx, da, db)


def test_caller_max_above_the_true_max():
    # a caller-supplied max|X| (and max|G|) larger than the true one is valid: g shrinks,
    # the codes change, and the layer must match the oracle run with the same max
    ft = _ft()
    spec = MID
    inp, layer, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    x, dy = inp.x.cuda(), inp.dy.cuda()
    ax = float(np.float32(3.0 * ora.amax(inp.x)))
    ag = float(np.float32(2.5 * ora.amax(inp.dy)))
    y, t = ft.linear_fwd(w, x, ws, amax=torch.tensor([ax], device="cuda"))
    dx, da, db = ft.linear_bwd(w, x, t, dy, ws, amax=torch.tensor([ag], device="cuda"))
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    check_forward(inp.x, layer, y, t, amax=ax)
    check_backward(inp.x, inp.dy, layer, dx, da, db, amax=ag)


# ---------------------------------------------------------------- autograd wrapper

def test_autograd_wrapper_matches_oracle_and_uses_its_adapter_arguments():
    ft = _ft()
    spec = wl.PARITY_SMALL
    inp, layer, w = _setup(spec)
    ws = ft.Workspace(w, spec.M, "cuda")
    x = inp.x.cuda().requires_grad_(True)
    a = inp.lora_a.float().cuda().requires_grad_(True)   # fp32 master copies of the adapter
    b = inp.lora_b.float().cuda().requires_grad_(True)
    y = ft.FourTuneLinearFunction.apply(x, a, b, w, ws)
    y.backward(inp.dy.cuda())
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    check_forward(inp.x, layer, y.detach(), None)
    br = ora.linear_bwd(inp.x, inp.dy, layer)
    assert ora.rel_frobenius(_np(x.grad), br.dx) < TOL
    assert a.grad.dtype == torch.float32 and b.grad.dtype == torch.float32
    assert ora.rel_frobenius(_np(a.grad), br.da) < TOL
    assert ora.rel_frobenius(_np(b.grad), br.db) < TOL
    # new adapter values passed in are the ones used (not the ones held by `w`)
    b2 = (inp.lora_b.float() * -3.0).to(torch.bfloat16)
    layer2 = ora.Layer(qr=layer.qr, ls_up=layer.ls_up, ls_down=layer.ls_down, lora_a=inp.lora_a, lora_b=b2,
                       lora_scale=spec.lora_scale)
    y2 = ft.FourTuneLinearFunction.apply(inp.x.cuda(), a.detach(), b2.float().cuda(), w, ws)
    torch.cuda.synchronize()
    check_forward(inp.x, layer2, y2, None)
