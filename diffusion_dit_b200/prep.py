"""Offline weight preparation (FourTune Eq. (1), section 3.1), run once per frozen weight.

W ~= R + L_stab with L_stab = Ls_up Ls_down, the top-r_s singular triplets of W
(sqrt of each singular value on either side, both factors bf16), and
R = fl32(W - Ls_up Ls_down).  The pages apply this split offline and keep the
stabilizer in high precision; it is not on the per-step path, so the SVD here is a
library routine (torch's randomized low-rank SVD in fp64 on the host).  The 4-bit
quantization of R that follows runs in the CUDA library
(``fourtune.prepare_weights``).
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass
class StabilizerSplit:
    ls_up: torch.Tensor    # bf16 [N, r_s]
    ls_down: torch.Tensor  # bf16 [r_s, K]
    residual: torch.Tensor  # fp32 [N, K]


def svd_split(w: torch.Tensor, r_s: int, niter: int = 8, oversample: int = 8, seed: int = 0) -> StabilizerSplit:
    """Split a bf16 [N, K] weight into a fp32 residual and a bf16 rank-r_s stabilizer."""
    W = w.detach().to("cpu", torch.float64)
    N, K = W.shape
    if r_s == 0:
        return StabilizerSplit(torch.zeros(N, 0, dtype=torch.bfloat16), torch.zeros(0, K, dtype=torch.bfloat16),
                               W.float())
    torch.manual_seed(seed)
    U, S, V = torch.svd_lowrank(W, q=min(r_s + oversample, min(N, K)), niter=niter)
    U, S, V = U[:, :r_s], S[:r_s], V[:, :r_s]
    root = S.sqrt()
    ls_up = (U * root).to(torch.bfloat16)
    ls_down = (V * root).T.contiguous().to(torch.bfloat16)
    L = ls_up.double() @ ls_down.double()
    return StabilizerSplit(ls_up, ls_down, (W - L).float())
