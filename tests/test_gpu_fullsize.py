"""Parity at the workloads' full sizes (FLUX-shaped layers), through the same C-ABI
calls bench.py times.  The oracle checks what it can compute row by row: sampled token
rows of Y and dX (fp64 over the same dequantized operands; one row from every 32-row
group, so every 128-row band and every TMEM lane quarter of every output tile is seen,
with all N or K columns of each), the adapter gradients in full, and the quantizer's codes
and scales bit for bit on sampled 16-row bands (with the tensor max fixed, every 16x16
block is independent of the others).

Y, dX and the MLP's dP are bf16: each sampled element within one bf16 ulp of the rounded
oracle value plus its fp32 accumulation allowance (tests/parity.py), the relative
Frobenius error against fp64 <= 2e-3, and against the rounded oracle <= FROB_ROUNDED.
dA and dB: relative Frobenius <= 2e-3.  Codes and scales exact.
"""
import functools

import numpy as np
import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora
from tests import parity

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

TOL = 2e-3
FROB_ROUNDED = 2e-4
# The down-projections (T, U, the quantizer's fused x down^T) are fp32 tensor-core
# accumulations of up to ~21500 terms: their error grows like sqrt(K) * 2^-24 (about
# 1e-5 at K = 21504 on heavy-tailed inputs); 1e-4 bounds that with margin.
DOWN_TOL = 1e-4


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


def _np(t):
    return t.double().cpu().numpy()


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


def _fwd_parity(x, layer, y, rows, amax=None):
    fr = ora.linear_fwd(x, layer, amax_x=amax, rows=rows)
    st = parity.compare_bf16("y", _np(y[torch.from_numpy(rows).to(y.device)]), fr.y,
                             parity.fwd_allowance(x, layer, fr, rows))
    parity.assert_bf16_parity(st, FROB_ROUNDED, TOL)
    return fr, st


def _bwd_parity(x, dy, layer, dx, da, db, rows, amax=None, name="dx"):
    br = ora.linear_bwd(x, dy, layer, amax_g=amax, rows=rows)
    st = parity.compare_bf16(name, _np(dx[torch.from_numpy(rows).to(dx.device)]), br.dx,
                             parity.bwd_allowance(dy, layer, br, rows))
    parity.assert_bf16_parity(st, FROB_ROUNDED, TOL)
    errs = {"da": ora.rel_frobenius(_np(da), br.da), "db": ora.rel_frobenius(_np(db), br.db)}
    assert errs["da"] < TOL and errs["db"] < TOL, errs
    return br, st


def _check_layer(spec, seed=0):
    ft = _ft()
    inp, layer, w = _layer(spec, seed)
    ws = ft.Workspace(w, spec.M, "cuda")
    xg, dyg = inp.x.cuda(), inp.dy.cuda()
    y, t = ft.linear_fwd(w, xg, ws)
    dx, da, db = ft.linear_bwd(w, xg, t, dyg, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    rows = parity.sample_rows(spec.M, seed=seed)
    fr, sy = _fwd_parity(inp.x, layer, y, rows)
    assert ora.rel_frobenius(_np(t), fr.t) < DOWN_TOL
    _, sdx = _bwd_parity(inp.x, inp.dy, layer, dx, da, db, rows)
    print(spec.name, seed, sy, sdx)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_flux_qkv_full_size(seed):
    _check_layer(wl.FLUX_QKV, seed)


def test_flux_single_stream_linear1_full_size():
    _check_layer(wl.FLUX_SS_L1)


def test_flux_single_stream_linear2_full_size():
    _check_layer(wl.FLUX_SS_L2)


def _gelu_step_ok(got, ref):
    """Each element within one bf16 step (2^-7 relative) of the fp64 value."""
    return np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-30)


def test_flux_mlp_pair_with_gelu_full_size():
    """Up layer -> GELU-tanh (bf16) -> down layer, forward and backward, unfused calls.
    Each layer is checked against the oracle on the GPU's own input to that layer (for
    the down layer: the GPU's H), and the GELU step against the textbook formula."""
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
    P = _np(p)
    assert _gelu_step_ok(_np(h), ora.gelu_tanh(P))
    dH = _np(dh)
    dPref = dH * ora.gelu_tanh_grad(P)
    # gelu' crosses zero near p = -0.75, where its two fp32 terms (each of size ~1 + |p|)
    # cancel: allow their fp32 rounding on top of one bf16 step
    tol = np.abs(dPref) * 2.0 ** -7 + np.abs(dH) * (1.0 + np.abs(P)) * 2.0 ** -20
    assert np.all(np.abs(_np(dp) - dPref) <= tol)
    rows = parity.sample_rows(up.M)
    _fwd_parity(inp_u.x, layer_u, p, rows)
    _bwd_parity(inp_u.x, dp.cpu(), layer_u, dx, da_u, db_u, rows)
    h_cpu = h.cpu()
    _fwd_parity(h_cpu, layer_d, yd, rows)
    _bwd_parity(h_cpu, inp_d.dy, layer_d, dh, da_d, db_d, rows, name="dh")


def test_flux_mlp_pair_fused_against_the_oracle_full_size():
    """The fused MLP path (section 3.3 "MLP Fusion") directly against the oracle, at full
    size: fourtune_linear_fwd_gelu's P (the up layer's Eq. (2) output), H = bf16(gelu(P))
    and max|H|; the down layer's Y through fourtune_linear_fwd fed that max;
    fourtune_linear_bwd_gelu's dP, dA and dB; and the up layer's backward from that dP.
    dP is defined as bf16(dH * gelu'(P)) with dH the down layer's bf16 dX (its output dtype),
    so the oracle's dP is bf16(dH_oracle) * gelu'(P): against it, in fp64, relative Frobenius
    <= 2e-3 (one rounding: dP's own); element by element, dP within one bf16 ulp of it plus
    gelu'(P) times the distance of the GPU's dH (the unfused call's dX, which the fused call
    never stores; itself checked element by element against the oracle) from bf16(dH_oracle),
    plus the fp32 rounding of gelu' where its two terms cancel."""
    ft = _ft()
    up, down = wl.FLUX_MLP_UP, wl.FLUX_MLP_DOWN
    inp_u, layer_u, w_u = _layer(up)
    inp_d, layer_d, w_d = _layer(down)
    ws_u = ft.Workspace(w_u, up.M, "cuda")
    ws_d = ft.Workspace(w_d, down.M, "cuda")
    x, g = inp_u.x.cuda(), inp_d.dy.cuda()
    p, h, hmax, t_u = ft.linear_fwd_gelu(w_u, x, ws_u)
    yd, t_d = ft.linear_fwd(w_d, h, ws_d, amax=hmax)
    dp, da_d, db_d = ft.linear_bwd_gelu(w_d, h, t_d, g, p, ws_d)
    dp, da_d, db_d = dp.clone(), da_d.clone(), db_d.clone()
    dx, da_u, db_u = ft.linear_bwd(w_u, x, t_u, dp, ws_u)
    dh_unfused, _, _ = ft.linear_bwd(w_d, h, t_d, g, ws_d)   # the dH the fused call never writes
    torch.cuda.synchronize()
    assert ws_u.device_status() == 0 and ws_d.device_status() == 0
    rows = parity.sample_rows(up.M)
    # forward: P against Eq. (2), H against the textbook GELU of P, max|H| exact
    _fwd_parity(inp_u.x, layer_u, p, rows)
    P, H = _np(p), _np(h)
    assert _gelu_step_ok(H, ora.gelu_tanh(P))
    assert hmax.item() == float(np.max(np.abs(H)))
    h_cpu = h.cpu()
    _fwd_parity(h_cpu, layer_d, yd, rows, amax=hmax.item())
    # backward of the down layer: dH element by element (unfused call), then dP
    br_d, _ = _bwd_parity(h_cpu, inp_d.dy, layer_d, dh_unfused, da_d, db_d, rows, name="dh")
    gp = ora.gelu_tanh_grad(P[rows])
    dp_rows = _np(dp)[rows]
    dh_ref = parity.bf16_round(br_d.dx)          # dH as the layer's bf16 output
    dp_ref = dh_ref * gp
    assert ora.rel_frobenius(dp_rows, dp_ref) < TOL
    dH = _np(dh_unfused)[rows]
    ulp = parity.bf16_ulp(np.maximum(np.abs(dp_ref), np.abs(dp_rows)))
    tol = ulp + np.abs(gp) * np.abs(dH - dh_ref) + np.abs(dH) * (1.0 + np.abs(P[rows])) * 2.0 ** -20
    assert np.all(np.abs(dp_rows - parity.bf16_round(dp_ref)) <= tol)
    assert ora.rel_frobenius(dp_rows, parity.bf16_round(dp_ref)) < FROB_ROUNDED
    # the up layer's backward from the fused dP
    _bwd_parity(inp_u.x, dp.cpu(), layer_u, dx, da_u, db_u, rows)


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
    rows = parity.sample_rows(qspec.rows, group=128)
    ref = x[rows].double().numpy() @ down.double().numpy().T
    assert ora.rel_frobenius(t[rows].double().cpu().numpy(), ref) < DOWN_TOL
