"""Pins of the oracle's layer algebra (FourTune Eq. 1-3 and the adapter gradients
of section 3.2) against brute force, library routines and exact identities."""
import itertools

import numpy as np
import pytest
import torch

from diffusion_dit_b200 import workloads as wl
from oracle import fourtune_oracle as ora


def _tiny_layer(M=16, K=32, N=48, r_s=2, r=2, seed=0, alpha=None):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) * 0.3).to(torch.bfloat16)
    a = (torch.randn(r, K, generator=g) * 0.2).to(torch.bfloat16)
    b = (torch.randn(N, r, generator=g) * 0.2).to(torch.bfloat16)
    dy = (torch.randn(M, N, generator=g) * 0.1).to(torch.bfloat16)
    split = ora.svd_split(w, r_s)
    layer = ora.Layer(qr=ora.quantize_residual(split.r), ls_up=split.ls_up, ls_down=split.ls_down,
                      lora_a=a, lora_b=b, lora_scale=(alpha if alpha is not None else r) / r)
    return x, dy, layer


def test_svd_split_reconstructs_w():
    inp = wl.make_layer_inputs(wl.PARITY_SMALL, seed=0)
    split = ora.svd_split(inp.w, wl.PARITY_SMALL.r_s)
    W = inp.w.double().numpy()
    L = split.ls_up.double().numpy() @ split.ls_down.double().numpy()
    R = split.r.double().numpy()
    # R = fl32(W - L): the only error is R's own fp32 rounding (half an ulp)
    half_ulp = np.spacing(np.abs(split.r.numpy())).astype(np.float64) / 2
    assert np.all(np.abs(R + L - W) <= half_ulp + 1e-30)


@pytest.mark.parametrize("shape", [(24, 512), (40, 3072), (8, 9)])
def test_jacobi_svd_against_lapack(shape):
    # the oracle's Rayleigh-Ritz step: singular values equal LAPACK's, the factors
    # reconstruct the matrix and are orthonormal, on a matrix with a wide range of
    # singular values and two nearly equal ones
    rng = np.random.default_rng(3)
    p, n = shape
    U0, _ = np.linalg.qr(rng.standard_normal((p, p)))
    V0, _ = np.linalg.qr(rng.standard_normal((n, p)))
    sig = np.logspace(2, -3, p)
    if p > 2:
        sig[1] = sig[2] * (1 + 1e-9)
    B = U0 @ np.diag(sig) @ V0.T
    U, S, Vt = ora.jacobi_svd(B)
    assert np.allclose(S, np.linalg.svd(B, compute_uv=False), rtol=1e-10, atol=1e-13 * sig[0])
    assert np.allclose(U @ np.diag(S) @ Vt, B, atol=1e-11 * sig[0])
    assert np.allclose(U.T @ U, np.eye(p), atol=1e-12)
    assert np.allclose(Vt @ Vt.T, np.eye(p), atol=1e-10)
    assert np.all(np.diff(S) <= 0)


def test_svd_split_singular_values_match_lapack():
    inp = wl.make_layer_inputs(wl.PARITY_SMALL, seed=0)
    W = inp.w.double().numpy()
    s_ref = np.linalg.svd(W, compute_uv=False)
    split = ora.svd_split(inp.w, wl.PARITY_SMALL.r_s)
    # the planted rank-4 component is well separated: exact to solver precision
    assert np.allclose(split.sigma[:4], s_ref[:4], rtol=1e-10)
    # the planted singular value 5 is recovered to within the bulk's spectral norm
    bulk = 0.02 * (np.sqrt(512) + np.sqrt(512))
    assert np.all(np.abs(split.sigma[:4] - 5.0) <= bulk)
    # the rest of the top 16 sit in a near-degenerate bulk; subspace iteration
    # still gets them to within a few percent
    assert np.allclose(split.sigma[:16], s_ref[:16], rtol=5e-2)
    # and the stabilizer removes the planted part: R's spectral norm is bulk-sized
    assert np.linalg.norm(split.r.double().numpy(), 2) < 1.5 * bulk


def _brute_fwd(x, layer):
    Xh = ora.quantize_block16(x).dequantize()
    Rh = layer.qr.dequantize()
    Xd = x.double().numpy()
    Ld = layer.ls_down.double().numpy()
    Lu = layer.ls_up.double().numpy()
    A = layer.lora_a.double().numpy()
    B = layer.lora_b.double().numpy()
    M, K = Xd.shape
    N = Rh.shape[0]
    Y = np.zeros((M, N))
    for m, n in itertools.product(range(M), range(N)):
        acc = 0.0
        for k in range(K):
            acc += Xh[m, k] * Rh[n, k]
        for j in range(Ld.shape[0]):
            acc += sum(Xd[m, k] * Ld[j, k] for k in range(K)) * Lu[n, j]
        for j in range(A.shape[0]):
            acc += layer.lora_scale * sum(Xd[m, k] * A[j, k] for k in range(K)) * B[n, j]
        Y[m, n] = acc
    return Y


def test_forward_matches_brute_force():
    x, dy, layer = _tiny_layer(M=16, K=32, N=16, r_s=2, r=2, alpha=4.0)
    got = ora.linear_fwd(x, layer).y
    assert np.allclose(got, _brute_fwd(x, layer), rtol=1e-12, atol=1e-12)


def test_backward_matches_brute_force():
    x, dy, layer = _tiny_layer(M=16, K=32, N=16, r_s=2, r=3, alpha=6.0)
    res = ora.linear_bwd(x, dy, layer)
    Gh = ora.quantize_block16(dy).dequantize()
    Rh = layer.qr.dequantize()
    G = dy.double().numpy()
    X = x.double().numpy()
    Ld = layer.ls_down.double().numpy()
    Lu = layer.ls_up.double().numpy()
    A = layer.lora_a.double().numpy()
    B = layer.lora_b.double().numpy()
    s = layer.lora_scale
    M, K = X.shape
    N = G.shape[1]
    dx = np.zeros((M, K))
    for m, k in itertools.product(range(M), range(K)):
        acc = sum(Gh[m, n] * Rh[n, k] for n in range(N))
        acc += sum(G[m, n] * Lu[n, j] * Ld[j, k] for n in range(N) for j in range(Ld.shape[0]))
        acc += sum(s * G[m, n] * B[n, j] * A[j, k] for n in range(N) for j in range(A.shape[0]))
        dx[m, k] = acc
    db = np.zeros_like(B)
    for n, j in itertools.product(range(N), range(B.shape[1])):
        db[n, j] = s * sum(G[m, n] * sum(X[m, k] * A[j, k] for k in range(K)) for m in range(M))
    da = np.zeros_like(A)
    for j, k in itertools.product(range(A.shape[0]), range(K)):
        da[j, k] = s * sum(sum(G[m, n] * B[n, j] for n in range(N)) * X[m, k] for m in range(M))
    assert np.allclose(res.dx, dx, rtol=1e-11, atol=1e-13)
    assert np.allclose(res.db, db, rtol=1e-11, atol=1e-13)
    assert np.allclose(res.da, da, rtol=1e-11, atol=1e-13)


def _backbone_only(layer):
    r = layer.r
    return ora.Layer(qr=layer.qr, ls_up=layer.ls_up[:, :0], ls_down=layer.ls_down[:0],
                     lora_a=torch.zeros(r, layer.lora_a.shape[1], dtype=torch.bfloat16),
                     lora_b=torch.zeros(layer.lora_b.shape[0], r, dtype=torch.bfloat16),
                     lora_scale=1.0)


def test_identity_and_permutation_weights():
    K = 64
    x, _, _ = _tiny_layer(M=32, K=K, N=K)
    perm = torch.randperm(K, generator=torch.Generator().manual_seed(5))
    for w in (torch.eye(K), torch.eye(K)[perm]):
        # a 0/1 matrix quantizes exactly: every nonzero block has amax 1 -> scale 448,
        # code 6, value 6 * 448 / 2688 = 1
        q = ora.quantize_block16(w.to(torch.bfloat16))
        assert np.array_equal(q.dequantize(), w.double().numpy())
        layer = ora.Layer(qr=q, ls_up=torch.zeros(K, 0, dtype=torch.bfloat16),
                          ls_down=torch.zeros(0, K, dtype=torch.bfloat16),
                          lora_a=torch.zeros(1, K, dtype=torch.bfloat16),
                          lora_b=torch.zeros(K, 1, dtype=torch.bfloat16), lora_scale=1.0)
        y = ora.linear_fwd(x, layer).y
        xh = ora.quantize_block16(x).dequantize()
        assert np.array_equal(y, xh @ w.double().numpy().T)


def test_adjoint_forward_and_backward_backbones():
    # <Ghat, Xhat Rhat^T> = <Ghat Rhat, Xhat>: catches any transposition mismatch
    # between the forward GEMM and the backward GEMM through Q(R)^T.
    x, dy, layer = _tiny_layer(M=64, K=96, N=80, r_s=4, r=4)
    bb = _backbone_only(layer)
    y = ora.linear_fwd(x, bb).y
    dx = ora.linear_bwd(x, dy, bb).dx
    gh = ora.quantize_block16(dy).dequantize()
    xh = ora.quantize_block16(x).dequantize()
    lhs = float(np.sum(gh * y))
    rhs = float(np.sum(dx * xh))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_backward_through_transposed_qtensor():
    # the backbone pathway of Eq. (3) equals Ghat times the dequantized transpose
    x, dy, layer = _tiny_layer(M=32, K=48, N=64)
    bb = _backbone_only(layer)
    dx = ora.linear_bwd(x, dy, bb).dx
    gh = ora.quantize_block16(dy).dequantize()
    rt = layer.qr.transpose().dequantize()  # [K, N]
    assert np.allclose(dx, gh @ rt.T, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("which", ["b", "a"])
def test_adapter_gradients_are_exact_directional_derivatives(which):
    # L = <G, Y> is linear in A and in B (the adapter branch never quantizes), so
    # changing one entry by d changes L by exactly d * grad (up to fp64 rounding).
    x, dy, layer = _tiny_layer(M=32, K=48, N=64, r_s=2, r=4, alpha=8.0)
    G = dy.double().numpy()
    base = float(np.sum(G * ora.linear_fwd(x, layer).y))
    grads = ora.linear_bwd(x, dy, layer)
    rng = np.random.default_rng(0)
    for _ in range(6):
        if which == "b":
            t = layer.lora_b.clone()
            i, j = rng.integers(t.shape[0]), rng.integers(t.shape[1])
            grad = grads.db[i, j]
        else:
            t = layer.lora_a.clone()
            i, j = rng.integers(t.shape[0]), rng.integers(t.shape[1])
            grad = grads.da[i, j]
        old = float(t[i, j])
        t[i, j] = torch.tensor(old + 0.375, dtype=torch.bfloat16)
        d = float(t[i, j]) - old
        kw = dict(lora_b=t) if which == "b" else dict(lora_a=t)
        lay2 = ora.Layer(qr=layer.qr, ls_up=layer.ls_up, ls_down=layer.ls_down,
                         lora_a=kw.get("lora_a", layer.lora_a), lora_b=kw.get("lora_b", layer.lora_b),
                         lora_scale=layer.lora_scale)
        new = float(np.sum(G * ora.linear_fwd(x, lay2).y))
        assert abs((new - base) - d * grad) <= 1e-9 * max(1.0, abs(base))


def test_sampled_rows_match_full():
    x, dy, layer = _tiny_layer(M=64, K=64, N=48)
    rows = np.array([0, 5, 17, 63])
    full = ora.linear_fwd(x, layer)
    part = ora.linear_fwd(x, layer, rows=rows)
    assert np.allclose(part.y, full.y[rows], rtol=1e-13, atol=1e-13)
    fb = ora.linear_bwd(x, dy, layer)
    pb = ora.linear_bwd(x, dy, layer, rows=rows)
    assert np.allclose(pb.dx, fb.dx[rows], rtol=1e-13, atol=1e-13)


def test_gelu_tanh_against_torch_and_identities():
    p = np.linspace(-9, 9, 20001)
    ref = torch.nn.functional.gelu(torch.from_numpy(p), approximate="tanh").numpy()
    assert np.allclose(ora.gelu_tanh(p), ref, rtol=1e-14, atol=1e-15)
    assert ora.gelu_tanh(np.array([0.0]))[0] == 0.0
    # gelu(x) - gelu(-x) = x for the tanh form
    assert np.allclose(ora.gelu_tanh(p) - ora.gelu_tanh(-p), p, atol=1e-13)


def test_gelu_tanh_grad_against_central_difference_and_autograd():
    p = np.linspace(-7, 7, 2001)
    h = 1e-6
    fd = (ora.gelu_tanh(p + h) - ora.gelu_tanh(p - h)) / (2 * h)
    assert np.allclose(ora.gelu_tanh_grad(p), fd, atol=1e-8)
    t = torch.from_numpy(p).requires_grad_(True)
    torch.nn.functional.gelu(t, approximate="tanh").sum().backward()
    assert np.allclose(ora.gelu_tanh_grad(p), t.grad.numpy(), rtol=1e-12, atol=1e-14)
