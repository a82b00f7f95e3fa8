"""Pins for the oracle's group-wise 1x16 quantizer (FourTune section 4.3, "Impact of
Quantization Granularity", Table 5: one UE4M3 scale per row and 16 consecutive columns,
with the same tensor factor g as the 16x16 blocks of section 3.1).  Each pin ties it to
something other than its own formula: the already-pinned 16x16 quantizer it must reduce
to, the locality of a row's result, the ordering of its scales against the 16x16 ones,
and the E2M1 rounding bound on every element."""
import numpy as np
import pytest
import torch

from oracle import fourtune_oracle as ora


def _x(rows, cols, seed=0, outliers=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    if outliers:
        mask = torch.rand(rows, cols, generator=g) < 0.02
        x[mask] *= 30.0
    return x.to(torch.bfloat16)


def test_reduces_to_16x16_when_rows_repeat_within_each_band():
    # every 16-row band is one row repeated: each 1x16 group's max is its 16x16 block's
    base = _x(4, 96, seed=1)
    x = base.repeat_interleave(16, dim=0)  # [64, 96]
    q1 = ora.quantize_1x16(x)
    q16 = ora.quantize_block16(x)
    assert q1.g == q16.g
    assert np.array_equal(q1.codes, q16.codes)
    assert np.array_equal(q1.scales, np.repeat(q16.scales, 16, axis=0))


def test_a_rows_result_depends_on_that_row_only():
    x = _x(32, 64, seed=2)
    amax = float(x.float().abs().max())
    q = ora.quantize_1x16(x, amax)
    y = x.clone()
    y[5] = (y[5].float() * 0.25).to(torch.bfloat16)  # change one row, keep the tensor max
    assert float(y.float().abs().max()) <= amax
    qy = ora.quantize_1x16(y, amax)
    others = [i for i in range(32) if i != 5]
    assert np.array_equal(q.codes[others], qy.codes[others])
    assert np.array_equal(q.scales[others], qy.scales[others])
    assert not np.array_equal(q.scales[5], qy.scales[5])


def test_group_scales_never_exceed_the_block_scale():
    x = _x(48, 128, seed=3)
    q1 = ora.quantize_1x16(x)
    q16 = ora.quantize_block16(x)
    assert q1.g == q16.g
    # UE4M3 codes of non-negative values are ordered like the values
    assert np.all(q1.scales <= np.repeat(q16.scales, 16, axis=0))
    # and on outlier-heavy data the finer groups are strictly finer somewhere
    assert np.any(q1.scales < np.repeat(q16.scales, 16, axis=0))


def test_every_element_within_the_e2m1_rounding_bound():
    x = _x(32, 160, seed=4)
    q = ora.quantize_1x16(x)
    xd = x.double().numpy()
    xh = q.dequantize()
    unit = np.array([ora.ue4m3_value(int(s)) for s in q.scales.ravel()]).reshape(q.scales.shape) / q.g
    unit = np.repeat(unit, 16, axis=1)                  # per element: val(sb) / g
    v = np.abs(xd) / np.where(unit > 0, unit, 1.0)      # magnitude in units of the scale
    # E2M1 spacing is 0.5 below 2, 1 in [2, 4), 2 in [4, 6]: half of it bounds the
    # rounding error; beyond 6 the code saturates
    half = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
    bound = (half + np.maximum(v - 6.0, 0.0)) * unit
    # the scaled value is formed in fp32 (inv = g / val(sb), then x * inv: two roundings),
    # so a value a hair above a grid midpoint in fp64 can be the midpoint in fp32 and
    # round to even: allow those two roundings
    bound += np.abs(xd) * 2.0 ** -22
    assert np.all(np.abs(xd - xh) <= bound + 1e-300)
    # the group max lands near the top of the grid: the scale is not oversized
    gmax = np.abs(xd).reshape(32, -1, 16).max(axis=2)
    scale = unit[:, ::16]
    ratio = gmax / np.where(scale > 0, scale, np.inf)
    assert np.all(ratio[gmax > 0] > 3.0)


def test_zero_rows_and_degenerate_tensor():
    x = _x(16, 32, seed=5)
    x[3] = 0
    q = ora.quantize_1x16(x)
    assert np.all(q.scales[3] == 0) and np.all(q.codes[3] == 0)
    z = torch.zeros(8, 48, dtype=torch.bfloat16)
    qz = ora.quantize_1x16(z)
    assert qz.g == 1.0 and not qz.codes.any() and not qz.scales.any()


def test_transpose_is_refused_for_1x16():
    q = ora.quantize_1x16(_x(16, 32, seed=6))
    with pytest.raises(ValueError):
        q.transpose()
