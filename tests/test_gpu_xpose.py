"""Q(R)^T transposed on the fly in the backward's dX GEMM (FourTune section 3.2, "4-Bit
Backward Pass via Block-Quantization"; the on-the-fly transposition of section 1): with
Q(R)^T's codes dropped, the GEMM loads Q(R)'s untransposed tiles and its scale warps
rewrite them in shared memory into the K-major layout the MMA reads.  The
MMA then sees the same operand bits as with the stored copy, so the backward must write
exactly the same dX, dA and dB, and meet the oracle's bar.  Covers both GEMM kernels (CTA
pairs when M % 256 == 0, single CTAs otherwise), the GELU-backward epilogue, several
output tiles and k steps, and the full-size FLUX QKV layer."""
import functools

import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora

pytestmark = pytest.mark.gpu

TOL = 2e-3

MID = wl.LayerSpec(name="mid_384x1024x768", M=384, K=1024, N=768, r_s=16, r=16, alpha=32.0,
                   n_outlier_cols=5, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                   b_std=0.01, dy_std=1e-2)
WIDE = wl.LayerSpec(name="wide_256x2048x512", M=256, K=2048, N=512, r_s=16, r=32, alpha=32.0,
                    n_outlier_cols=10, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                    b_std=0.01, dy_std=1e-2)
SPECS = [wl.PARITY_SMALL, MID, WIDE]


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


@functools.lru_cache(maxsize=3)
def _setup(spec: wl.LayerSpec):
    ft = _ft()
    inp = wl.make_layer_inputs(spec, seed=0)
    split = ora.svd_split(inp.w, spec.r_s)
    layer = ora.Layer(qr=ora.quantize_residual(split.r), ls_up=split.ls_up, ls_down=split.ls_down,
                      lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)
    w = ft.prepare_weights(split.r.cuda(), split.ls_up.cuda(), split.ls_down.cuda(), inp.lora_a.cuda(),
                           inp.lora_b.cuda(), spec.lora_scale)
    return inp, layer, w


def _bwd(w, spec, x, dy, p=None):
    ft = _ft()
    ws = ft.Workspace(w, spec.M, "cuda")
    _, t = ft.linear_fwd(w, x, ws)
    if p is None:
        out = ft.linear_bwd(w, x, t, dy, ws)
    else:
        out = ft.linear_bwd_gelu(w, x, t, dy, p, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    return [o.clone() for o in out]


def test_dropping_the_transposed_codes_keeps_the_scale_layout():
    ft = _ft()
    _, _, w = _setup(wl.PARITY_SMALL)
    wf = ft.drop_transposed_codes(w)
    assert wf.qr_t.codes is None and wf.qr_t.scales is None
    assert wf.qr_t.sf_mma is w.qr_t.sf_mma and wf.qr is w.qr
    s = wf.c_struct()
    assert not s.qr_t.codes and s.qr_t.sf_mma


@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
def test_backward_transposing_on_the_fly_equals_stored_copy(spec):
    ft = _ft()
    inp, layer, w = _setup(spec)
    x, dy = inp.x.cuda(), inp.dy.cuda()
    dx, da, db = _bwd(w, spec, x, dy)
    dx_f, da_f, db_f = _bwd(ft.drop_transposed_codes(w), spec, x, dy)
    assert torch.equal(dx_f, dx), "dX differs from the stored-transpose path"
    assert torch.equal(da_f, da) and torch.equal(db_f, db)
    ref = ora.linear_bwd(inp.x, inp.dy, layer)
    assert ora.rel_frobenius(dx_f.double().cpu().numpy(), ref.dx) < TOL


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_gelu_backward_transposing_on_the_fly_equals_stored_copy(spec):
    ft = _ft()
    inp, _, w = _setup(spec)
    x, dy = inp.x.cuda(), inp.dy.cuda()
    g = torch.Generator().manual_seed(11)
    p = ((torch.randn(spec.M, spec.K, generator=g) * 2.0).to(torch.bfloat16)).cuda()
    dp, da, db = _bwd(w, spec, x, dy, p)
    dp_f, da_f, db_f = _bwd(ft.drop_transposed_codes(w), spec, x, dy, p)
    assert torch.equal(dp_f, dp) and torch.equal(da_f, da) and torch.equal(db_f, db)


@pytest.mark.slow
def test_full_size_qkv_backward_transposing_on_the_fly_equals_stored_copy():
    # a random residual stands in for the SVD split: the check is the equality of the two
    # operand paths, which holds for any Q(R)
    ft = _ft()
    spec = wl.FLUX_QKV
    inp = wl.make_layer_inputs(spec, seed=0)
    g = torch.Generator().manual_seed(5)
    r = (torch.randn(spec.N, spec.K, generator=g) * 0.02).cuda()
    ls_up = (torch.randn(spec.N, spec.r_s, generator=g) * 0.1).to(torch.bfloat16).cuda()
    ls_down = (torch.randn(spec.r_s, spec.K, generator=g) * 0.1).to(torch.bfloat16).cuda()
    w = ft.prepare_weights(r, ls_up, ls_down, inp.lora_a.cuda(), inp.lora_b.cuda(), spec.lora_scale)
    x, dy = inp.x.cuda(), inp.dy.cuda()
    dx, da, db = _bwd(w, spec, x, dy)
    dx_f, da_f, db_f = _bwd(ft.drop_transposed_codes(w), spec, x, dy)
    assert torch.equal(dx_f, dx) and torch.equal(da_f, da) and torch.equal(db_f, db)
