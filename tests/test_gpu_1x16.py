"""GPU group-wise 1x16 quantization (FourTune section 4.3, "Impact of Quantization
Granularity", Table 5) against the oracle: codes, per-group scales and g bit for bit, the
tensor-core scale layout, and the layer forward with X quantized 1x16 (forward use)."""
import numpy as np
import pytest
import torch

from diffusion_dit_b200 import prep
from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


def _sf_mma_expected(scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """The documented tensor-core scale layout, built from a [rows, cols/16] group grid."""
    out = np.zeros(rows * cols // 16, dtype=np.uint8)
    per_band = cols // 64
    for row in range(rows):
        band, m = divmod(row, 128)
        within_row = 16 * (m % 32) + 4 * (m // 32)
        for cb in range(cols // 16):
            out[(band * per_band + cb // 4) * 512 + within_row + cb % 4] = scales[row, cb]
    return out


def _with_outliers(rows, cols, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g) * std
    mask = torch.rand(rows, cols, generator=g) < 0.01
    x[mask] = torch.distributions.Laplace(0.0, 10.0 * std).sample((int(mask.sum()),))
    x[3, :] = 0.0  # an all-zero row: zero scales and codes
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("shape", [(128, 64), (256, 512), (384, 1024), (4608, 3072)], ids=str)
def test_quantize_1x16_bit_exact(shape):
    ft = _ft()
    rows, cols = shape
    x = _with_outliers(rows, cols, seed=rows + cols)
    q = ft.quantize_1x16(x.cuda())
    torch.cuda.synchronize()
    qo = ora.quantize_1x16(x)
    assert q.g.item() == np.float32(qo.g)
    assert np.array_equal(q.scales.cpu().numpy(), qo.scales)
    assert np.array_equal(q.codes.cpu().numpy(), qo.codes)
    if rows * cols <= 512 * 1024:
        assert np.array_equal(q.sf_mma.cpu().numpy(), _sf_mma_expected(qo.scales, rows, cols))


def test_quantize_1x16_with_given_amax_and_gradient_like_values():
    ft = _ft()
    x = _with_outliers(512, 768, seed=11, std=1e-3)  # dY-like magnitudes
    amax = 4.0 * float(x.float().abs().max())
    q = ft.quantize_1x16(x.cuda(), amax=torch.tensor([amax], dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    qo = ora.quantize_1x16(x, amax)
    assert q.g.item() == np.float32(qo.g)
    assert np.array_equal(q.scales.cpu().numpy(), qo.scales)
    assert np.array_equal(q.codes.cpu().numpy(), qo.codes)


MID = wl.LayerSpec(name="mid_384x1024x768", M=384, K=1024, N=768, r_s=16, r=16, alpha=32.0,
                   n_outlier_cols=5, outlier_gain=20.0, w_std=0.02, plant_rank=4, plant_sigma=6.0,
                   b_std=0.01, dy_std=1e-2)


@pytest.mark.parametrize("spec", [wl.PARITY_SMALL, MID], ids=lambda s: s.name)
def test_linear_forward_1x16_matches_oracle(spec):
    ft = _ft()
    inp = wl.make_layer_inputs(spec, seed=0)
    split = ora.svd_split(inp.w, spec.r_s)
    layer = ora.Layer(qr=ora.quantize_residual(split.r), ls_up=split.ls_up, ls_down=split.ls_down,
                      lora_a=inp.lora_a, lora_b=inp.lora_b, lora_scale=spec.lora_scale)
    w = ft.prepare_weights(split.r.cuda(), split.ls_up.cuda(), split.ls_down.cuda(), inp.lora_a.cuda(),
                           inp.lora_b.cuda(), spec.lora_scale)
    ws = ft.Workspace(w, spec.M, "cuda")
    x = inp.x.cuda()
    y16, t16 = ft.linear_fwd(w, x, ws)
    y16, t16 = y16.clone(), t16.clone()
    y, t = ft.linear_fwd_1x16(w, x, ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    ref = ora.linear_fwd(inp.x, layer, x_block_rows=1)
    err = ora.rel_frobenius(y.float().cpu().numpy().astype(np.float64), ref.y)
    assert err <= TOL, err
    # the down-projection does not depend on the granularity of Q(X)
    assert torch.equal(t, t16)
    # and the 1x16 output is a different quantization of X than the 16x16 one
    assert not torch.equal(y, y16)
