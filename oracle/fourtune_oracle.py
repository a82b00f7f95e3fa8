"""FourTune oracle: a plain, slow, CPU statement of the W4A4G4 triple-branch linear.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, ``__graft_entry__.smoke()``
and bench.py's cpu_baseline / reference arms may import this module.  It shares
no code with the CUDA library in ``diffusion_dit_b200`` and imports nothing from
it.

Source: "FourTune: Towards Fully 4-Bit Efficient Post-Training for Diffusion
Models" (arXiv 2607.05711).  Layout: PyTorch's, X [M, K], W and R [N, K],
Y [M, N]; the paper writes Y = X W with W in R^{m x n}, the same algebra
transposed.

  * Eq. (1), section 3.1: W ~= R + L_stab, L_stab = L1 L2, the top singular
    triplets of W.  Here Ls_up [N, r_s] and Ls_down [r_s, K] with
    L_stab = Ls_up Ls_down (sqrt of the singular values on each side, bf16) and
    R = fl32(W - Ls_up Ls_down).
  * Eq. (2), section 3.1: Y = GEMM4(Q(X), Q(R)) + X L_stab + X (A B); Q is applied
    offline to R and dynamically to X.  LoRA here: A [r, K], B [N, r], scale
    s = alpha / r, so the adapter branch is s (X A^T) B^T.
  * Eq. (3), section 3.2: dX = GEMM4(Q(G), Q(R)^T) + G L_stab^T + G (A B)^T, with
    Q(R)^T the same 16x16 blocks transposed (no requantization).
  * Section 3.2, adapter gradients: dB = (X A)^T G, dA = X^T (G B^T) in the
    paper's layout; here dB = s G^T (X A^T) [N, r], dA = s (G B)^T X [r, K].
    R and L_stab receive no gradient.

The 4-bit GEMMs are exact definitions: the dequantized operands multiplied in
fp64.  The stabilizer and adapter branches use the unquantized bf16 X and G.
The codec (block amax -> scale -> E2M1) is the C file next to this one.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fourtune_codec.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libfourtune_oracle.so")

E2M1_TOP = 6.0
UE4M3_TOP = 448.0


def build_oracle(force: bool = False) -> str:
    """Compile the C codec with gcc (no FMA contraction, IEEE fp32)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build_oracle())
        i64, f32, vp = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        L.ora_e2m1_encode.argtypes = [f32]
        L.ora_e2m1_encode.restype = ctypes.c_int
        L.ora_ue4m3_encode.argtypes = [f32]
        L.ora_ue4m3_encode.restype = ctypes.c_int
        L.ora_e2m1_value.argtypes = [ctypes.c_int]
        L.ora_e2m1_value.restype = ctypes.c_double
        L.ora_ue4m3_value.argtypes = [ctypes.c_int]
        L.ora_ue4m3_value.restype = ctypes.c_double
        L.ora_amax_bf16.argtypes = [vp, i64, i64, i64]
        L.ora_amax_bf16.restype = f32
        L.ora_global_scale.argtypes = [f32]
        L.ora_global_scale.restype = f32
        L.ora_quantize_block16.argtypes = [vp, i64, i64, i64, f32, vp, vp, vp]
        L.ora_quantize_block16.restype = ctypes.c_int
        L.ora_quantize_block16_f32.argtypes = [vp, i64, i64, i64, f32, vp, vp, vp]
        L.ora_quantize_block16_f32.restype = ctypes.c_int
        L.ora_amax_f32.argtypes = [vp, i64, i64, i64]
        L.ora_amax_f32.restype = f32
        L.ora_dequantize_block16.argtypes = [vp, vp, f32, i64, i64, vp]
        L.ora_quantize_1x16.argtypes = [vp, i64, i64, i64, f32, vp, vp, vp]
        L.ora_quantize_1x16.restype = ctypes.c_int
        L.ora_dequantize_blocks.argtypes = [vp, vp, f32, i64, i64, ctypes.c_int, vp]
        L.ora_transpose_block16.argtypes = [vp, vp, i64, i64, vp, vp]
        L.ora_e2m1_encode_array.argtypes = [vp, i64, vp]
        L.ora_ue4m3_encode_array.argtypes = [vp, i64, vp]
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (C-contiguous copy)."""
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.contiguous().view(torch.int16).numpy().view(np.uint16))


def bf16_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


# ----------------------------------------------------------------------------
# codec (section 2.3 Round(W/s); section 3.1 NVFP4; 16x16 blocks, Table 5)
# ----------------------------------------------------------------------------

def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().ora_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def ue4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().ora_ue4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_value(code: int) -> float:
    return lib().ora_e2m1_value(int(code))


def ue4m3_value(code: int) -> float:
    return lib().ora_ue4m3_value(int(code))


def amax(x: torch.Tensor) -> float:
    if x.dtype == torch.float32:
        xb = np.ascontiguousarray(x.contiguous().numpy())
        return float(lib().ora_amax_f32(_ptr(xb), xb.shape[0], xb.shape[1], xb.shape[1]))
    xb = bf16_bits(x)
    return float(lib().ora_amax_bf16(_ptr(xb), xb.shape[0], xb.shape[1], xb.shape[1]))


def global_scale(amax_t: float) -> float:
    return float(lib().ora_global_scale(float(amax_t)))


@dataclasses.dataclass
class QTensor:
    """A block-quantized matrix: codes [rows, cols/2] (element 2j in the low nibble),
    scales [rows/block_rows, cols/16] UE4M3 bytes, tensor factor g (fp32).  block_rows is
    16 for the 16x16 blocks of section 3.1, 1 for the group-wise 1x16 of Table 5."""

    codes: np.ndarray
    scales: np.ndarray
    g: float
    rows: int
    cols: int
    block_rows: int = 16

    def dequantize(self) -> np.ndarray:
        out = np.empty((self.rows, self.cols), dtype=np.float64)
        lib().ora_dequantize_blocks(_ptr(self.codes), _ptr(self.scales), np.float32(self.g),
                                    self.rows, self.cols, self.block_rows, _ptr(out))
        return out

    def transpose(self) -> "QTensor":
        if self.block_rows != 16:
            raise ValueError("only 16x16 blocks transpose without requantization")
        ct = np.empty((self.cols, self.rows // 2), dtype=np.uint8)
        st = np.empty((self.cols // 16, self.rows // 16), dtype=np.uint8)
        lib().ora_transpose_block16(_ptr(self.codes), _ptr(self.scales), self.rows, self.cols,
                                    _ptr(ct), _ptr(st))
        return QTensor(ct, st, self.g, self.cols, self.rows)


def quantize_block16(x: torch.Tensor, amax_t: Optional[float] = None) -> QTensor:
    """Q(.) of section 3.1 with 16x16 blocks.  ``x`` is a bf16 or fp32 [rows, cols]
    tensor; ``amax_t`` (optional) replaces the tensor max used for g."""
    if x.dtype == torch.float32:
        xb = np.ascontiguousarray(x.contiguous().numpy())
        fn = lib().ora_quantize_block16_f32
    else:
        xb = bf16_bits(x)
        fn = lib().ora_quantize_block16
    rows, cols = xb.shape
    codes = np.empty((rows, cols // 2), dtype=np.uint8)
    scales = np.empty((rows // 16, cols // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    rc = fn(_ptr(xb), rows, cols, cols, -1.0 if amax_t is None else float(amax_t),
            _ptr(codes), _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError("rows and cols must be multiples of 16")
    return QTensor(codes, scales, float(g[0]), rows, cols)


def quantize_1x16(x: torch.Tensor, amax_t: Optional[float] = None) -> QTensor:
    """The group-wise 1x16 granularity FourTune compares its 16x16 blocks with (section
    4.3, "Impact of Quantization Granularity", Table 5): each row's 16 consecutive
    elements share one UE4M3 scale, with the same tensor factor g.  ``x`` is bf16."""
    xb = bf16_bits(x)
    rows, cols = xb.shape
    codes = np.empty((rows, cols // 2), dtype=np.uint8)
    scales = np.empty((rows, cols // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    rc = lib().ora_quantize_1x16(_ptr(xb), rows, cols, cols, -1.0 if amax_t is None else float(amax_t),
                                 _ptr(codes), _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError("cols must be a multiple of 16")
    return QTensor(codes, scales, float(g[0]), rows, cols, block_rows=1)


# ----------------------------------------------------------------------------
# Eq. (1): the SVD stabilizer split, applied offline
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Split:
    ls_up: torch.Tensor    # bf16 [N, r_s]
    ls_down: torch.Tensor  # bf16 [r_s, K]
    r: torch.Tensor        # fp32 [N, K] residual
    sigma: np.ndarray      # fp64 top singular values found


def jacobi_svd(B: np.ndarray, tol: float = 1e-15, max_sweeps: int = 60):
    """Thin SVD of a small fp64 matrix B [p, n] (p <= n) by one-sided (Hestenes) Jacobi
    rotations, written out: the p rows of B are rotated in pairs until every pair is
    orthogonal (to `tol` relative), accumulating the rotations in V [p, p].  Then the row
    norms are the singular values and B = V diag(S) Q with Q the normalised rows.  Returns
    (U [p, p], S [p] descending, Vt [p, n]) with B = U diag(S) Vt."""
    W = np.array(B, dtype=np.float64, copy=True)      # rows are rotated in place
    p = W.shape[0]
    V = np.eye(p)
    for _ in range(max_sweeps):
        rotated = False
        for i in range(p - 1):
            for j in range(i + 1, p):
                a = W[i] @ W[i]
                b = W[j] @ W[j]
                c = W[i] @ W[j]
                if abs(c) <= tol * np.sqrt(a * b) or c == 0.0:
                    continue
                rotated = True
                # the rotation that zeroes the (i, j) entry of the 2x2 Gram matrix
                zeta = (b - a) / (2.0 * c)
                t = np.copysign(1.0, zeta) / (abs(zeta) + np.sqrt(1.0 + zeta * zeta))
                cs = 1.0 / np.sqrt(1.0 + t * t)
                sn = cs * t
                wi, wj = W[i].copy(), W[j].copy()
                W[i], W[j] = cs * wi - sn * wj, sn * wi + cs * wj
                vi, vj = V[:, i].copy(), V[:, j].copy()
                V[:, i], V[:, j] = cs * vi - sn * vj, sn * vi + cs * vj
        if not rotated:
            break
    S = np.sqrt(np.einsum("ij,ij->i", W, W))
    order = np.argsort(-S, kind="stable")
    S, W, V = S[order], W[order], V[:, order]
    Vt = W / np.where(S > 0, S, 1.0)[:, None]
    return V, S, Vt


def svd_split(w: torch.Tensor, r_s: int, sweeps: int = 8, oversample: int = 8,
              seed: int = 1234) -> Split:
    """Top-r_s singular triplets of W (bf16 [N, K]) by subspace iteration in fp64:
    a Gaussian start block of width r_s + oversample, ``sweeps`` power sweeps with
    a QR re-orthonormalisation after each product, then Rayleigh-Ritz (the SVD of
    the small projected matrix, by the one-sided Jacobi rotations of jacobi_svd).  L_stab = Ls_up Ls_down with sqrt(S) on each
    side, both stored bf16; R = W - Ls_up Ls_down in fp64, rounded once to fp32."""
    W = bf16_f64(w)
    N, K = W.shape
    if r_s == 0:
        return Split(torch.zeros(N, 0, dtype=torch.bfloat16), torch.zeros(0, K, dtype=torch.bfloat16),
                     torch.from_numpy(W.astype(np.float32)), np.zeros(0))
    p = min(r_s + oversample, min(N, K))
    rng = np.random.default_rng(seed)
    Q, _ = np.linalg.qr(W @ rng.standard_normal((K, p)))
    for _ in range(sweeps):
        Z, _ = np.linalg.qr(W.T @ Q)
        Q, _ = np.linalg.qr(W @ Z)
    Bsmall = Q.T @ W                      # [p, K]
    Ub, S, Vt = jacobi_svd(Bsmall)        # Rayleigh-Ritz: the small projected problem
    U = Q @ Ub[:, :r_s]                   # [N, r_s]
    S = S[:r_s]
    V = Vt[:r_s].T                        # [K, r_s]
    root = np.sqrt(S)
    ls_up = torch.from_numpy(U * root[None, :]).to(torch.bfloat16)
    ls_down = torch.from_numpy((V * root[None, :]).T.copy()).to(torch.bfloat16)
    L = bf16_f64(ls_up) @ bf16_f64(ls_down)
    R = torch.from_numpy((W - L).astype(np.float32))
    return Split(ls_up, ls_down, R, S)


def quantize_residual(R: torch.Tensor) -> QTensor:
    """Q(R), applied offline to the fp32 residual (section 3.1)."""
    return quantize_block16(R.float())


# ----------------------------------------------------------------------------
# Eq. (2) forward and Eq. (3) backward
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Layer:
    qr: QTensor            # Q(R) [N, K]
    ls_up: torch.Tensor    # bf16 [N, r_s]
    ls_down: torch.Tensor  # bf16 [r_s, K]
    lora_a: torch.Tensor   # bf16 [r, K]
    lora_b: torch.Tensor   # bf16 [N, r]
    lora_scale: float

    @property
    def r_s(self) -> int:
        return self.ls_down.shape[0]

    @property
    def r(self) -> int:
        return self.lora_a.shape[0]

    def down(self) -> np.ndarray:
        """[Ls_down; A] in fp64, [r_s + r, K]."""
        return np.concatenate([bf16_f64(self.ls_down), bf16_f64(self.lora_a)], axis=0)

    def up(self) -> np.ndarray:
        """[Ls_up, s B] in fp64, [N, r_s + r]."""
        return np.concatenate([bf16_f64(self.ls_up), self.lora_scale * bf16_f64(self.lora_b)], axis=1)


@dataclasses.dataclass
class FwdResult:
    y: np.ndarray          # fp64 [M, N] (or the sampled rows)
    t: np.ndarray          # fp64 [M, r_s + r] = X [Ls_down; A]^T  (saved for backward)
    qx: QTensor


def linear_fwd(x: torch.Tensor, layer: Layer, amax_x: Optional[float] = None,
               rows: Optional[np.ndarray] = None, x_block_rows: int = 16) -> FwdResult:
    """Eq. (2): Y = Xhat Rhat^T + X Ls_down^T Ls_up^T + s X A^T B^T.
    ``rows`` (optional) evaluates Y only for those token rows.  ``x_block_rows`` = 1
    quantizes X group-wise 1x16 (Table 5's comparison, forward only) instead of 16x16."""
    qx = quantize_block16(x, amax_x) if x_block_rows == 16 else quantize_1x16(x, amax_x)
    Xd = bf16_f64(x)
    Xh = qx.dequantize()
    Rh = layer.qr.dequantize()
    T = Xd @ layer.down().T
    if rows is not None:
        Xh, Tr = Xh[rows], T[rows]
    else:
        Tr = T
    y = Xh @ Rh.T + Tr @ layer.up().T
    return FwdResult(y=y, t=T, qx=qx)


@dataclasses.dataclass
class BwdResult:
    dx: np.ndarray         # fp64 [M, K] (or the sampled rows)
    da: np.ndarray         # fp64 [r, K]
    db: np.ndarray         # fp64 [N, r]
    u: np.ndarray          # fp64 [M, r_s + r] = G [Ls_up, s B]
    qg: QTensor


def linear_bwd(x: torch.Tensor, dy: torch.Tensor, layer: Layer, amax_g: Optional[float] = None,
               rows: Optional[np.ndarray] = None) -> BwdResult:
    """Eq. (3) and the adapter gradients of section 3.2:
    dX = Ghat Rhat + (G [Ls_up, s B]) [Ls_down; A];  dB = s G^T (X A^T);
    dA = s (G B)^T X.  ``rows`` (optional) evaluates dX only for those rows;
    dA and dB are always full."""
    qg = quantize_block16(dy, amax_g)
    Gd = bf16_f64(dy)
    Xd = bf16_f64(x)
    Gh = qg.dequantize()
    Rh = layer.qr.dequantize()
    U = Gd @ layer.up()
    if rows is not None:
        Gh, Ur = Gh[rows], U[rows]
    else:
        Ur = U
    dx = Gh @ Rh + Ur @ layer.down()
    s = layer.lora_scale
    A = bf16_f64(layer.lora_a)
    B = bf16_f64(layer.lora_b)
    db = s * (Gd.T @ (Xd @ A.T))
    da = s * ((Gd @ B).T @ Xd)
    return BwdResult(dx=dx, da=da, db=db, u=U, qg=qg)


# ----------------------------------------------------------------------------
# GELU-tanh between the MLP linears (section 3.3 "MLP Fusion" names GeLU)
# ----------------------------------------------------------------------------

_C = math.sqrt(2.0 / math.pi)


def gelu_tanh(p: np.ndarray) -> np.ndarray:
    """0.5 p (1 + tanh(sqrt(2/pi) (p + 0.044715 p^3))), fp64.

    Evaluated as p * sigmoid(2u), the same function (0.5 (1 + tanh u) = 1 / (1 + e^{-2u})):
    written as printed, 1 + tanh(u) cancels for p below about -6.5 and loses all relative
    precision even in fp64."""
    p = np.asarray(p, dtype=np.float64)
    u = _C * (p + 0.044715 * p ** 3)
    with np.errstate(over="ignore"):
        return p / (1.0 + np.exp(-2.0 * u))


def gelu_tanh_grad(p: np.ndarray) -> np.ndarray:
    """d/dp of gelu_tanh, fp64: with s = sigmoid(2u), s + 2 p s (1 - s) u' (the product and
    chain rule of the formula above; 1 - s = sigmoid(-2u) evaluated directly)."""
    p = np.asarray(p, dtype=np.float64)
    u = _C * (p + 0.044715 * p ** 3)
    du = _C * (1.0 + 3.0 * 0.044715 * p ** 2)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-2.0 * u))
        one_minus = 1.0 / (1.0 + np.exp(2.0 * u))
    return s + 2.0 * p * s * one_minus * du


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """Round fp64 values to bf16 (torch's conversion)."""
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).to(torch.bfloat16)


def rel_frobenius(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))
