"""The product's offline stabilizer split (FourTune Eq. (1), section 3.1), on the CPU.

prep.svd_split is what the benchmark uses to build the frozen layer; every parity test
feeds both paths from the oracle's split instead, so this file pins the product's split on
its own: R + Ls_up Ls_down reconstructs W to within the rounding of R to fp32, the
stabilizer's singular values are W's top ones (LAPACK's full SVD as the reference), and
each singular value is split as sqrt(sigma) on both sides.
"""
import numpy as np
import pytest
import torch

from diffusion_dit_b200 import prep
from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora


@pytest.fixture(scope="module")
def small():
    spec = wl.PARITY_SMALL
    inp = wl.make_layer_inputs(spec, seed=0)
    return spec, inp.w, prep.svd_split(inp.w, spec.r_s)


def _half_ulp_f32(r: np.ndarray) -> np.ndarray:
    r32 = r.astype(np.float32)
    return np.abs(np.spacing(r32).astype(np.float64)) / 2.0


def test_split_shapes_and_dtypes(small):
    spec, w, s = small
    assert s.ls_up.shape == (spec.N, spec.r_s) and s.ls_up.dtype == torch.bfloat16
    assert s.ls_down.shape == (spec.r_s, spec.K) and s.ls_down.dtype == torch.bfloat16
    assert s.residual.shape == (spec.N, spec.K) and s.residual.dtype == torch.float32


def test_residual_reconstructs_w_within_fp32_rounding(small):
    # R = fl32(W - Ls_up Ls_down) with the product exact in fp64: W - L - R is only the
    # rounding of R, at most half an fp32 ulp of R per element
    _, w, s = small
    W = w.double().numpy()
    L = s.ls_up.double().numpy() @ s.ls_down.double().numpy()
    R = s.residual.double().numpy()
    assert np.all(np.abs(W - L - R) <= _half_ulp_f32(R))


def test_stabilizer_holds_the_top_singular_values(small):
    spec, w, s = small
    W = w.double().numpy()
    sig = np.linalg.svd(W, compute_uv=False)
    L = s.ls_up.double().numpy() @ s.ls_down.double().numpy()
    got = np.linalg.svd(L, compute_uv=False)[: spec.r_s]
    # the planted rank-4 component (singular values near 5, far above the bulk near 0.9)
    # is found to within the bf16 rounding of the factors
    k = spec.plant_rank
    assert np.allclose(got[:k], sig[:k], rtol=2e-3)
    # the rest of the rank r_s comes from the bulk, whose singular values are close
    # together: a Rayleigh-Ritz value never exceeds the true one (up to the factors' bf16
    # rounding), and the captured energy is most of the true top-r_s energy
    assert np.all(got <= sig[: spec.r_s] * (1 + 2e-3))
    assert np.sum(got ** 2) >= 0.95 * np.sum(sig[: spec.r_s] ** 2)
    # and the planted values agree with the oracle's own split (subspace iteration, fp64)
    o = ora.svd_split(w, spec.r_s)
    assert np.allclose(got[:k], o.sigma[:k], rtol=2e-3)


def test_sqrt_sigma_on_both_sides(small):
    # Ls_up[:, i] = u_i sqrt(s_i), Ls_down[i, :] = sqrt(s_i) v_i: equal column / row norms
    _, _, s = small
    up = np.linalg.norm(s.ls_up.double().numpy(), axis=0)
    dn = np.linalg.norm(s.ls_down.double().numpy(), axis=1)
    assert np.allclose(up, dn, rtol=5e-3)


def test_rank_zero_is_the_weight_itself(small):
    spec, w, _ = small
    s0 = prep.svd_split(w, 0)
    assert s0.ls_up.shape == (spec.N, 0) and s0.ls_down.shape == (0, spec.K)
    assert torch.equal(s0.residual, w.float())
