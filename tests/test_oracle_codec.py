"""Pins of the oracle's codec against facts that do not come from the oracle.

* The E2M1 and UE4M3 value sets and rounding rules of the NVFP4 format (FourTune
  section 3.1), as golden tables under tests/golden/.
* torch's own fp32 -> float8_e4m3fn conversion (a library routine) for every
  UE4M3 decision below the saturation point.
* A threshold formulation of E2M1 round-to-nearest-even, written independently
  of the oracle's nearest-value search.
* Closed-form cases of the 16x16 block quantizer (FourTune section 3.2, Table 5):
  constant blocks, zero tensors, block positions, idempotence, and the
  transpose property that lets Q(R)^T reuse the same blocks.
"""
import os

import numpy as np
import pytest
import torch

from oracle import fourtune_oracle as ora

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    sections, cur = {}, None
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.startswith("["):
                cur = line.strip("[]")
                sections[cur] = []
                continue
            a, b = line.split()
            sections[cur].append((a, b))
    return sections


def test_e2m1_value_set_matches_format():
    g = _read_golden("e2m1_format.txt")
    for code, val in g["values"]:
        v = ora.e2m1_value(int(code))
        assert v == float(val) and np.signbit(v) == val.startswith("-"), (code, v, val)


def test_e2m1_rounding_golden():
    g = _read_golden("e2m1_format.txt")
    xs = np.array([float(a) for a, _ in g["round"]], dtype=np.float32)
    want = np.array([int(b) for _, b in g["round"]], dtype=np.uint8)
    got = ora.e2m1_encode(xs)
    assert np.array_equal(got, want), list(zip(xs, got, want))


def _e2m1_by_thresholds(v: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even onto {0,.5,1,1.5,2,3,4,6} written as threshold
    counting: a midpoint whose upper neighbour has an even code is included with
    >=, otherwise with >."""
    a = np.abs(v.astype(np.float64))
    code = ((a > 0.25).astype(int) + (a >= 0.75) + (a > 1.25) + (a >= 1.75)
            + (a > 2.5) + (a >= 3.5) + (a > 5.0))
    return (code | (np.signbit(v).astype(int) << 3)).astype(np.uint8)


def test_e2m1_matches_threshold_form_on_dense_sweep():
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.uniform(-8, 8, 200_000).astype(np.float32),
        np.linspace(-7, 7, 100_001, dtype=np.float32),
    ])
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    near = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 10)])
    xs = np.concatenate([xs, near, -near])
    assert np.array_equal(ora.e2m1_encode(xs), _e2m1_by_thresholds(xs))


def test_ue4m3_golden():
    g = _read_golden("ue4m3_format.txt")
    xs = np.array([float(a) for a, _ in g["round"]], dtype=np.float32)
    want = np.array([int(b) for _, b in g["round"]], dtype=np.uint8)
    assert np.array_equal(ora.ue4m3_encode(xs), want)


def test_ue4m3_matches_torch_float8_below_saturation():
    # every UE4M3 value, every midpoint between neighbours, their fp32 neighbours,
    # and a dense random sweep of [0, 448]
    vals = np.array([ora.ue4m3_value(c) for c in range(127)])
    mids = (vals[1:] + vals[:-1]) / 2
    base = np.concatenate([vals, mids]).astype(np.float32)
    rng = np.random.default_rng(3)
    xs = np.concatenate([base, np.nextafter(base, 0), np.nextafter(base, 1e9),
                         rng.uniform(0, 448, 200_000).astype(np.float32),
                         np.exp2(rng.uniform(-12, 8.8, 200_000)).astype(np.float32)])
    xs = xs[(xs >= 0) & (xs <= 448)]
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ora.ue4m3_encode(xs), ref)


def test_ue4m3_saturates_above_448():
    xs = np.array([448.00003, 460, 479.9, 480, 1e6, 3e38], dtype=np.float32)
    assert np.all(ora.ue4m3_encode(xs) == 0x7E)


@pytest.mark.parametrize("v", [1.0, -1.0, 2.0, -0.5, 3.0, -6.0, 0.375, 96.0, -1536.0])
def test_constant_block_maps_exactly(v):
    x = torch.full((16, 16), v).to(torch.bfloat16)
    q = ora.quantize_block16(x)
    assert q.scales.tolist() == [[0x7E]]
    code = 0xF if v < 0 else 0x7
    assert np.all(q.codes == (code | (code << 4)))
    # g = 2688/|v|, val(sb) = 448, so xhat = 6 * 448 / g = |v| exactly when 2688/|v|
    # is an fp32 value (true for +-2^k and +-3 * 2^k)
    assert np.all(q.dequantize() == v)


def test_zero_tensor_is_all_zero():
    q = ora.quantize_block16(torch.zeros(32, 48, dtype=torch.bfloat16))
    assert q.g == 1.0
    assert not q.codes.any() and not q.scales.any()


def test_block_scale_positions_and_values():
    # block (i, j) is the constant c_ij, one of them sets amax_t; the scale of each
    # block must be UE4M3(fl32(fl32(c/6) * g)), computed here with torch fp32 ops
    # and torch's float8 conversion, at the block's own grid position.
    rng = np.random.default_rng(11)
    nb_r, nb_c = 4, 3
    c = rng.uniform(0.01, 9.0, (nb_r, nb_c)).astype(np.float32)
    c = torch.from_numpy(c).to(torch.bfloat16).float()
    c[1, 2] = 10.0  # the tensor max
    x = c.repeat_interleave(16, 0).repeat_interleave(16, 1).to(torch.bfloat16)
    q = ora.quantize_block16(x)
    g = torch.tensor(2688.0, dtype=torch.float32) / torch.tensor(10.0, dtype=torch.float32)
    assert q.g == g.item()
    s = (c / torch.tensor(6.0)) * g
    want = s.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q.scales, want)
    # every element of a constant block is within 1/16 of the block max after
    # scaling, so all codes are +6
    assert np.all(q.codes == 0x77)


def test_sign_of_zero_code():
    x = torch.zeros(16, 16, dtype=torch.bfloat16)
    x[0, 0] = 1.0
    x[0, 1] = -0.01   # rounds to -0 -> code 8 (sign bit kept)
    x[0, 2] = -0.0
    q = ora.quantize_block16(x)
    assert q.codes[0, 0] == (0x7 | (0x8 << 4))
    assert q.codes[0, 1] & 0xF == 0x8


def _layerish(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    x[:, :3] *= 20
    return x.to(torch.bfloat16)


def test_idempotence_with_fixed_g():
    x = _layerish(256, 512, 0)
    amax = ora.amax(x)
    q = ora.quantize_block16(x, amax)
    xhat = torch.from_numpy(q.dequantize().astype(np.float32))
    q2 = ora.quantize_block16(xhat, amax)
    assert q2.g == q.g
    assert np.array_equal(q2.scales, q.scales)
    assert np.array_equal(q2.codes, q.codes)
    n_sub = int(((q.scales > 0) & (q.scales < 8)).sum())
    assert n_sub == 0


def test_scaled_error_bound():
    # |x * inv - val(code)| <= 1 (largest half-gap of E2M1 is between 4 and 6; the
    # saturated excess is at most 6 * 2^-4), checked through the dequantized values
    x = _layerish(64, 128, 1)
    q = ora.quantize_block16(x)
    xd = x.double().numpy()
    xh = q.dequantize()
    sb = np.array([[ora.ue4m3_value(s) for s in row] for row in q.scales])
    step = np.repeat(np.repeat(sb, 16, 0), 16, 1) / q.g
    assert np.all(np.abs(xd - xh) <= 1.0 * step * (1 + 1e-6))


def test_transpose_equals_quantizing_the_transpose():
    # 16x16 blocks are symmetric under transposition (FourTune section 3.2): the
    # quantized transpose is the transpose of the quantized matrix, codes and
    # scales alike, so Q(R)^T needs no requantization.
    x = _layerish(96, 160, 2)
    q = ora.quantize_block16(x)
    qt = q.transpose()
    q_of_t = ora.quantize_block16(x.t().contiguous())
    assert np.array_equal(qt.codes, q_of_t.codes)
    assert np.array_equal(qt.scales, q_of_t.scales)
    assert np.array_equal(qt.dequantize(), q.dequantize().T)


def test_fp32_input_matches_bf16_input_on_bf16_values():
    x = _layerish(48, 64, 3)
    a = ora.quantize_block16(x)
    b = ora.quantize_block16(x.float())
    assert a.g == b.g and np.array_equal(a.codes, b.codes) and np.array_equal(a.scales, b.scales)


def test_bad_shape_rejected():
    with pytest.raises(ValueError):
        ora.quantize_block16(torch.zeros(20, 32, dtype=torch.bfloat16))
