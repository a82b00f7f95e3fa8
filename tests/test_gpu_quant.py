"""GPU quantizer vs the oracle: codes, block scales and g bit for bit (FourTune sections
3.1-3.2, 16x16 NVFP4 blocks), the tensor-core scale layout, and the transposed copy."""
import numpy as np
import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora

pytestmark = pytest.mark.gpu


def _ft():
    from diffusion_dit_b200 import fourtune as ft
    return ft


def _sf_mma_expected(scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """The documented tensor-core scale layout, built from a [rows/16, cols/16] grid."""
    out = np.zeros(rows * cols // 16, dtype=np.uint8)
    per_band = cols // 64
    for row in range(rows):
        band, m = divmod(row, 128)
        within_row = 16 * (m % 32) + 4 * (m // 32)
        for cb in range(cols // 16):
            atom = band * per_band + cb // 4
            out[atom * 512 + within_row + cb % 4] = scales[row // 16, cb]
    return out


def _check_equal(q_gpu, q_ora):
    assert q_gpu.g.item() == np.float32(q_ora.g)
    assert np.array_equal(q_gpu.scales.cpu().numpy(), q_ora.scales)
    got = q_gpu.codes.cpu().numpy()
    bad = np.argwhere(got != q_ora.codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"


CASES = {
    "gauss_outliers_256x512": lambda: wl.make_layer_inputs(wl.PARITY_SMALL).x,
    "heavy_tail_384x640": lambda: wl.make_quant_input(
        wl.QuantSpec("t", 384, 640, 0, 0.01, 10.0), seed=3)[0],
    "tiny_values_128x256": lambda: (wl.make_gaussian_bf16((128, 256), 1e-3, 5)),
    "wide_range_128x128": lambda: (torch.randn(128, 128, generator=torch.Generator().manual_seed(9))
                                   * torch.logspace(-6, 3, 128).unsqueeze(0)).to(torch.bfloat16),
    "ragged_16x48": lambda: wl.make_gaussian_bf16((16, 48), 1.0, 11),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_quantize_bf16_matches_oracle(name):
    ft = _ft()
    x = CASES[name]()
    rows, cols = x.shape
    want_sf = rows % 128 == 0 and cols % 64 == 0
    q, _, _ = ft.quantize_block16(x.cuda(), with_sf=want_sf)
    qo = ora.quantize_block16(x)
    _check_equal(q, qo)
    if want_sf:
        assert np.array_equal(q.sf_mma.cpu().numpy(), _sf_mma_expected(qo.scales, rows, cols))


def test_quantize_fp32_residual_and_transpose():
    ft = _ft()
    g = torch.Generator().manual_seed(1)
    r = torch.randn(256, 384, generator=g) * 0.02
    r[:, 7] *= 30
    q, qt, _ = ft.quantize_block16(r.cuda(), transposed=True)
    qo = ora.quantize_block16(r)
    _check_equal(q, qo)
    qto = qo.transpose()
    _check_equal(qt, qto)
    assert np.array_equal(qt.sf_mma.cpu().numpy(), _sf_mma_expected(qto.scales, 384, 256))


def test_caller_supplied_amax():
    ft = _ft()
    x = wl.make_gaussian_bf16((128, 256), 1.0, 2)
    amax = 2.0 * ora.amax(x)   # a larger bound is valid; g changes accordingly
    q, _, _ = ft.quantize_block16(x.cuda(), amax=torch.tensor([amax], device="cuda"))
    _check_equal(q, ora.quantize_block16(x, amax))


def test_zero_input_gives_zero_output():
    ft = _ft()
    x = torch.zeros(128, 128, dtype=torch.bfloat16)
    q, _, _ = ft.quantize_block16(x.cuda())
    assert q.g.item() == 1.0
    assert int(q.codes.sum()) == 0 and int(q.scales.sum()) == 0


def test_fused_down_projection_of_the_quantizer():
    ft = _ft()
    spec = wl.QuantSpec("t", 256, 512, 32, 0.01, 10.0)
    x, down = wl.make_quant_input(spec, seed=4)
    q, _, t = ft.quantize_block16(x.cuda(), down=down.cuda())
    _check_equal(q, ora.quantize_block16(x))
    ref = x.double().numpy() @ down.double().numpy().T
    assert ora.rel_frobenius(t.cpu().double().numpy(), ref) < 1e-5


def test_strided_input_matches_oracle():
    # a column window of a wider matrix (row pitch ld = 576 > cols = 512, base 128 bytes
    # into each row): the tensor max over the window only, the fused quantizer's TMA box
    # walk over the pitch, and its down-projection
    ft = _ft()
    g = torch.Generator().manual_seed(21)
    big = (torch.randn(256, 576, generator=g) * 0.5).to(torch.bfloat16)
    big[:, :64] = 100.0  # outside the window: must not reach the tensor max
    x = big[:, 64:]
    down = (torch.randn(32, 512, generator=g) * 0.05).to(torch.bfloat16)
    q, _, t = ft.quantize_block16(big.cuda()[:, 64:], with_sf=True, down=down.cuda())
    qo = ora.quantize_block16(x.contiguous())
    _check_equal(q, qo)
    assert np.array_equal(q.sf_mma.cpu().numpy(), _sf_mma_expected(qo.scales, 256, 512))
    ref = x.double().numpy() @ down.double().numpy().T
    assert ora.rel_frobenius(t.cpu().double().numpy(), ref) < 1e-5


@pytest.mark.parametrize("amax_t", [1e-30, 3e-4, 1.0, 250.0, 3e5, 1e30])
def test_every_bf16_block_max(amax_t):
    # Each 16x16 block is the constant v for one of the 32639 positive finite bf16 values
    # (plus one zero block), so the block-scale arithmetic fl32(fl32(v / 6) * g) and the
    # UE4M3 rounding are exercised on every possible block max, for several g
    # (amax_t is supplied; blocks above it saturate, as in the oracle).
    ft = _ft()
    vals = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    vals = np.concatenate([vals, np.zeros(1, np.float32)])
    nb = vals.size + (-vals.size) % 8          # pad to a multiple of 8 blocks (128 columns)
    vals = np.concatenate([vals, np.full(nb - vals.size, 1.0, np.float32)])
    row = np.repeat(vals, 16)
    x = torch.from_numpy(np.tile(row, (128, 1))).to(torch.bfloat16)   # 128 rows x 16*nb columns
    q, _, _ = ft.quantize_block16(x.cuda(), amax=torch.tensor([amax_t], dtype=torch.float32, device="cuda"),
                                  with_sf=True)
    qo = ora.quantize_block16(x[:16].contiguous(), float(np.float32(amax_t)))
    got_scales = q.scales.cpu().numpy()
    for band in range(8):
        assert np.array_equal(got_scales[band], qo.scales[0])
    assert np.array_equal(q.codes[:16].cpu().numpy(), qo.codes)
