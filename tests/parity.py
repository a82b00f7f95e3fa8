"""Element-wise parity of the layer's bf16 outputs (Y, dX, dP) against the oracle.

The oracle evaluates Eq. (2) / Eq. (3) exactly in fp64 over the same dequantized
operands (FourTune sections 3.1-3.2).  The GPU accumulates the same exact products in
fp32 and rounds the result to bf16 once.  So every element must lie within one bf16 ulp
of the oracle's value rounded to bf16, plus the fp32 accumulation error, which is bounded
per element by the sum of the magnitudes of the terms it adds:

    |got - bf16(ref)| <= ulp_bf16 + n * 2^-23 * sum_k |a_k b_k|           (rule 1)

with n the number of terms (any summation order, each addition off by at most one fp32
ulp of a partial sum, which never exceeds the sum of magnitudes).  The low-rank tail adds
the error of its fp32 down-projection (same form, over the inner dimension) and of the
bf16 high + low split of its operand (2^-17 relative).  On top of that element rule, the
relative Frobenius distance from bf16(ref) measures what the rounded outputs lose against
the correctly rounded ones.

The allowance uses the oracle's own dequantized operands and factors: nothing here comes
from the CUDA path.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from oracle import fourtune_oracle as ora

U23 = 2.0 ** -23


def bf16_round(a: np.ndarray) -> np.ndarray:
    """fp64 values of bf16(a), round to nearest even (torch's conversion)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits; subnormal spacing 2^-133)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def sample_rows(M: int, group: int = 32, seed: int = 0) -> np.ndarray:
    """One random row from every `group`-row group (so every 128-row band, every TMEM lane
    quarter of every tile), plus the first and last rows."""
    rng = np.random.default_rng(seed)
    rows = np.arange(0, M, group) + rng.integers(0, group, size=M // group)
    return np.unique(np.concatenate([[0], rows, [M - 1]]))


@dataclasses.dataclass
class Stats:
    name: str
    n: int
    worst: float          # max over elements of |got - bf16(ref)| / (ulp + allowance)
    frob_rounded: float   # ||got - bf16(ref)|| / ||bf16(ref)||
    frob_exact: float     # ||got - ref|| / ||ref||
    off_by_ulps: int      # elements that differ from bf16(ref)

    def __str__(self):
        return (f"{self.name}: n={self.n} worst={self.worst:.3f} frob_vs_rounded={self.frob_rounded:.3e} "
                f"frob_vs_fp64={self.frob_exact:.3e} differing={self.off_by_ulps}")


def compare_bf16(name: str, got: np.ndarray, ref: np.ndarray, allowance: np.ndarray) -> Stats:
    got = np.asarray(got, dtype=np.float64)
    ref_r = bf16_round(ref)
    ulp = bf16_ulp(np.maximum(np.abs(ref_r), np.abs(got)))
    d = np.abs(got - ref_r)
    worst = float(np.max(d / (ulp + allowance))) if d.size else 0.0
    return Stats(name=name, n=int(got.size), worst=worst, frob_rounded=ora.rel_frobenius(got, ref_r),
                 frob_exact=ora.rel_frobenius(got, ref), off_by_ulps=int(np.count_nonzero(d)))


def assert_bf16_parity(st: Stats, frob_rounded_tol: float, frob_tol: float = 2e-3):
    assert st.worst <= 1.0, str(st)
    assert st.frob_exact <= frob_tol, str(st)
    assert st.frob_rounded <= frob_rounded_tol, str(st)


def _lowrank_allowance(inner_abs: np.ndarray, inner_len: int, t: np.ndarray, up_abs: np.ndarray) -> np.ndarray:
    """Error of the low-rank tail sum_j t_j up_j as the GPU forms it: t in fp32 from an
    fp32 accumulation of `inner_len` terms (|terms| summed in inner_abs [rows, R]), split
    into bf16 high + low (2^-17 relative), multiplied by bf16 factors and accumulated in
    fp32 with the 4-bit products."""
    R = t.shape[1]
    t_err = inner_len * U23 * inner_abs + 2.0 ** -17 * np.abs(t)
    return t_err @ up_abs.T + 2 * R * U23 * (np.abs(t) @ up_abs.T)


def fwd_allowance(x: torch.Tensor, layer: ora.Layer, fr: ora.FwdResult, rows: Optional[np.ndarray] = None):
    """Per-element allowance for Y = Xhat Rhat^T + T Up^T (rows: the sampled rows)."""
    Xh = fr.qx.dequantize()
    Rh = layer.qr.dequantize()
    Xd = ora.bf16_f64(x)
    if rows is not None:
        Xh, Xd, t = Xh[rows], Xd[rows], fr.t[rows]
    else:
        t = fr.t
    K = Xh.shape[1]
    s4 = np.abs(Xh) @ np.abs(Rh).T
    dn_abs = np.abs(layer.down())
    lr = _lowrank_allowance(np.abs(Xd) @ dn_abs.T, K, t, np.abs(layer.up()))
    y_abs = s4 + np.abs(t) @ np.abs(layer.up()).T
    # the 4-bit sum over K, the tail, and the final fp32 scaling by 1 / (g_x g_r)
    return K * U23 * s4 + lr + 2 * U23 * y_abs


def bwd_allowance(dy: torch.Tensor, layer: ora.Layer, br: ora.BwdResult, rows: Optional[np.ndarray] = None):
    """Per-element allowance for dX = Ghat Rhat + U Dn (rows: the sampled rows)."""
    Gh = br.qg.dequantize()
    Rh = layer.qr.dequantize()
    Gd = ora.bf16_f64(dy)
    if rows is not None:
        Gh, Gd, u = Gh[rows], Gd[rows], br.u[rows]
    else:
        u = br.u
    N = Gh.shape[1]
    s4 = np.abs(Gh) @ np.abs(Rh)
    up_abs = np.abs(layer.up())
    dn_abs = np.abs(layer.down())
    lr = _lowrank_allowance(np.abs(Gd) @ up_abs, N, u, dn_abs.T)
    y_abs = s4 + np.abs(u) @ dn_abs
    return N * U23 * s4 + lr + 2 * U23 * y_abs
