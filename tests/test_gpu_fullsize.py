"""Parity at the workloads' full sizes (FLUX-shaped layers), through the same C-ABI
calls bench.py times.  The oracle checks what it can compute row by row: sampled token
rows of Y and dX (fp64 over the same dequantized operands), the adapter gradients in
full, and the quantizer's codes and scales bit for bit on sampled 16-row bands (with the
tensor max fixed, every 16x16 block is independent of the others).

Tolerance as everywhere: relative Frobenius error <= 2e-3; codes and scales exact.
"""
import functools

import numpy as np
import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

TOL = 2e-3
# The down-projections (T, U, the quantizer's fused x down^T) are fp32 tensor-core
# accumulations of up to ~21500 terms: their error grows like sqrt(K) * 2^-24 (about
# 1e-5 at K = 21504 on heavy-tailed inputs); 1e-4 bounds that with margin.
DOWN_TOL = 1e-4


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


def _rows(M, n=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(M, size=n - 2, replace=False))
    return np.unique(np.concatenate([[0], rows, [M - 1]]))


@functools.lru_cache(maxsize=2)
def _layer(spec: wl.LayerSpec, seed: int = 0):
    ft = _ft()
    inp = wl.make_layer_inputs(spec, seed=seed)
    split = ora.svd_split(inp.w, spec.r_s)
    layer = ora.Layer(qr=ora.quantize_residual(split.r), ls_up=split.ls_up, ls_down=split.ls_down,
                      lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)
    w = ft.prepare_weights(split.r.cuda(), split.ls_up.cuda(), split.ls_down.cuda(), inp.lora_a.cuda(),
                           inp.lora_b.cuda(), spec.lora_scale)
    return inp, layer, w


def _check_layer(spec, x=None, dy=None):
    ft = _ft()
    inp, layer, w = _layer(spec)
    x = inp.x if x is None else x
    dy = inp.dy if dy is None else dy
    ws = ft.Workspace(w, spec.M, "cuda")
    xg, dyg = x.cuda(), dy.cuda()
    y, t = ft.linear_fwd(w, xg, ws)
    dx, da, db = ft.linear_bwd(w, xg, t, dyg, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    rows = _rows(spec.M)
    fr = ora.linear_fwd(x, layer, rows=rows)
    br = ora.linear_bwd(x, dy, layer, rows=rows)
    errs = {
        "y": ora.rel_frobenius(y[rows].double().cpu().numpy(), fr.y),
        "t": ora.rel_frobenius(t.double().cpu().numpy(), fr.t),
        "dx": ora.rel_frobenius(dx[rows].double().cpu().numpy(), br.dx),
        "da": ora.rel_frobenius(da.double().cpu().numpy(), br.da),
        "db": ora.rel_frobenius(db.double().cpu().numpy(), br.db),
    }
    assert errs["t"] < DOWN_TOL, errs
    for k in ("y", "dx", "da", "db"):
        assert errs[k] < TOL, errs
    return y, dx, errs


def test_flux_qkv_full_size():
    _check_layer(wl.FLUX_QKV)


def test_flux_single_stream_linear1_full_size():
    _check_layer(wl.FLUX_SS_L1)


def test_flux_single_stream_linear2_full_size():
    _check_layer(wl.FLUX_SS_L2)


def test_flux_mlp_pair_with_gelu_full_size():
    """Up layer -> GELU-tanh (bf16) -> down layer, forward and backward.  Each layer is
    checked against the oracle on the GPU's own input to that layer (for the down layer:
    the GPU's H), and the GELU step against the textbook formula."""
    ft = _ft()
    up, down = wl.FLUX_MLP_UP, wl.FLUX_MLP_DOWN
    inp_u, layer_u, w_u = _layer(up)
    inp_d, layer_d, w_d = _layer(down)
    ws_u = ft.Workspace(w_u, up.M, "cuda")
    ws_d = ft.Workspace(w_d, down.M, "cuda")
    x = inp_u.x.cuda()
    p, t_u = ft.linear_fwd(w_u, x, ws_u)
    h = ft.gelu_tanh_fwd(p)
    yd, t_d = ft.linear_fwd(w_d, h, ws_d)
    g = inp_d.dy.cuda()                      # upstream gradient of the down output
    dh, da_d, db_d = ft.linear_bwd(w_d, h, t_d, g, ws_d)
    dp = ft.gelu_tanh_bwd(p, dh)
    dx, da_u, db_u = ft.linear_bwd(w_u, x, t_u, dp, ws_u)
    torch.cuda.synchronize()
    assert ws_u.device_status() == 0 and ws_d.device_status() == 0
    # GELU: H = bf16(gelu(P)) and dP = bf16(dH gelu'(P)), evaluated in fp32 on the GPU:
    # each element within one bf16 step (2^-7 relative) of the fp64 formula
    P = p.double().cpu().numpy()
    H = h.double().cpu().numpy()
    Href = ora.gelu_tanh(P)
    assert np.all(np.abs(H - Href) <= np.abs(Href) * 2.0 ** -7 + 1e-30)
    dH = dh.double().cpu().numpy()
    dPref = dH * ora.gelu_tanh_grad(P)
    # gelu' crosses zero near p = -0.75, where its two fp32 terms (each of size ~1 + |p|)
    # cancel: allow their fp32 rounding on top of one bf16 step
    tol = np.abs(dPref) * 2.0 ** -7 + np.abs(dH) * (1.0 + np.abs(P)) * 2.0 ** -20
    assert np.all(np.abs(dp.double().cpu().numpy() - dPref) <= tol)
    rows = _rows(up.M)
    # up layer on X, backward with the GPU's dP
    fr = ora.linear_fwd(inp_u.x, layer_u, rows=rows)
    assert ora.rel_frobenius(p[rows].double().cpu().numpy(), fr.y) < TOL
    br = ora.linear_bwd(inp_u.x, dp.cpu(), layer_u, rows=rows)
    assert ora.rel_frobenius(dx[rows].double().cpu().numpy(), br.dx) < TOL
    assert ora.rel_frobenius(da_u.double().cpu().numpy(), br.da) < TOL
    assert ora.rel_frobenius(db_u.double().cpu().numpy(), br.db) < TOL
    # down layer on the GPU's H (its codes are the oracle's codes of that H)
    h_cpu = h.cpu()
    fr_d = ora.linear_fwd(h_cpu, layer_d, rows=rows)
    assert ora.rel_frobenius(yd[rows].double().cpu().numpy(), fr_d.y) < TOL
    br_d = ora.linear_bwd(h_cpu, inp_d.dy, layer_d, rows=rows)
    assert ora.rel_frobenius(dh[rows].double().cpu().numpy(), br_d.dx) < TOL
    assert ora.rel_frobenius(da_d.double().cpu().numpy(), br_d.da) < TOL
    assert ora.rel_frobenius(db_d.double().cpu().numpy(), br_d.db) < TOL


@pytest.mark.parametrize("qspec", wl.QUANT_SWEEP, ids=lambda s: s.name)
def test_quantizer_sweep_full_size(qspec):
    """The quantizer-only workload at full size, with its fused rank-32 down-projection:
    codes, block scales and g bit for bit on sampled 16-row bands (the tensor max is
    the oracle's, over the whole matrix), the down-projection on sampled rows."""
    ft = _ft()
    x, down = wl.make_quant_input(qspec, seed=0)
    xg = x.cuda()
    q, _, t = ft.quantize_block16(xg, with_sf=True, down=down.cuda())
    torch.cuda.synchronize()
    amax = ora.amax(x)
    assert q.g.item() == np.float32(ora.global_scale(amax))
    rng = np.random.default_rng(1)
    bands = np.unique(np.concatenate([[0, qspec.rows // 16 - 1],
                                      rng.choice(qspec.rows // 16, size=14, replace=False)]))
    codes = q.codes.cpu().numpy()
    scales = q.scales.cpu().numpy()
    for b in bands:
        xb = x[16 * b:16 * (b + 1)].contiguous()
        qo = ora.quantize_block16(xb, amax)
        assert np.array_equal(scales[b], qo.scales[0]), b
        assert np.array_equal(codes[16 * b:16 * (b + 1)], qo.codes), b
    rows = _rows(qspec.rows, n=64)
    ref = x[rows].double().numpy() @ down.double().numpy().T
    assert ora.rel_frobenius(t[rows].double().cpu().numpy(), ref) < DOWN_TOL
