"""Seeded synthetic workloads for the W4A4G4 triple-branch linear layer.

This module only draws random inputs.  It holds none of the layer's arithmetic
(no SVD split, no quantization, no products), so the CUDA path and the CPU oracle
can both take their inputs from it without sharing any of the method.

Shapes follow the FLUX.1-dev DiT layers that the FourTune paper trains
(FourTune, section 4.1, "Customization Setup": FLUX.1-dev at 1024x1024, LoRA rank
64): 4096 image-latent tokens plus 512 text tokens, hidden size 3072, MLP width
12288, and the single-stream block's fused projections.  The pretrained weights
are not available, so weights are Gaussian with a planted low-rank outlier
component, which gives the SVD stabilizer (section 3.1, Eq. 1) something to
absorb; activations carry a few outlier input channels.

Draw order for a layer (fixed): outlier channel indices, X, W bulk, U_p, V_p,
A, B, dY.  All draws are fp32 on a CPU ``torch.Generator`` and are rounded to
bf16 with round-to-nearest-even.

Distribution parameters: ``N(0, s)`` means standard deviation ``s``, except the
LoRA down factor A, which is drawn with variance 1/fan_in (std 1/sqrt(K)).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """One W4A4G4 linear: Y[M, N] = X[M, K] W[N, K]^T (PyTorch layout)."""

    name: str
    M: int
    K: int
    N: int
    r_s: int            # stabilizer rank
    r: int              # LoRA rank
    alpha: float        # LoRA scale s = alpha / r
    n_outlier_cols: int  # input channels of X scaled by `outlier_gain`
    outlier_gain: float
    w_std: float        # bulk weight std
    plant_rank: int     # rank of the planted outlier component of W
    plant_sigma: float  # its singular values (all equal)
    b_std: float        # LoRA up factor std
    dy_std: float       # upstream gradient std

    @property
    def lora_scale(self) -> float:
        return self.alpha / self.r


@dataclasses.dataclass(frozen=True)
class QuantSpec:
    """Quantizer-only workload: a bf16 [rows, cols] matrix with heavy-tailed entries."""

    name: str
    rows: int
    cols: int
    r_down: int          # rank of the fused down-projection
    p_heavy: float       # probability that an entry is replaced by Laplace(0, b)
    laplace_b: float


def _plant_sigma(N: int, K: int) -> float:
    # Same ratio to the bulk spectral edge 0.02 (sqrt(N) + sqrt(K)) as the small
    # parity layer (sigma 5 on a 512x512 layer): 0.11 (sqrt(N) + sqrt(K)).
    return 0.11 * (math.sqrt(N) + math.sqrt(K))


def _outliers(K: int) -> int:
    return int(round(0.005 * K))


def flux_layer(name: str, M: int, K: int, N: int, r_s: int, r: int) -> LayerSpec:
    return LayerSpec(name=name, M=M, K=K, N=N, r_s=r_s, r=r, alpha=float(r),
                     n_outlier_cols=_outliers(K), outlier_gain=20.0, w_std=0.02,
                     plant_rank=8, plant_sigma=_plant_sigma(N, K), b_std=0.01,
                     dy_std=1e-3)


# The small parity layer: 256x512 -> 512, stabilizer rank 16, LoRA rank 8, alpha 8.
PARITY_SMALL = LayerSpec(name="parity_256x512x512", M=256, K=512, N=512, r_s=16, r=8,
                         alpha=8.0, n_outlier_cols=4, outlier_gain=20.0, w_std=0.02,
                         plant_rank=4, plant_sigma=5.0, b_std=0.01, dy_std=1e-2)

# FLUX attention QKV projection: 4608 tokens, 3072 -> 9216.
FLUX_QKV = flux_layer("flux_qkv_4608x3072x9216", 4608, 3072, 9216, r_s=32, r=16)

# FLUX MLP pair: up 3072 -> 12288, GELU-tanh, down 12288 -> 3072.
FLUX_MLP_UP = flux_layer("flux_mlp_up_4608x3072x12288", 4608, 3072, 12288, r_s=32, r=32)
FLUX_MLP_DOWN = flux_layer("flux_mlp_down_4608x12288x3072", 4608, 12288, 3072, r_s=32, r=32)

# FLUX single-stream block, batch 2 x 4608 tokens.
FLUX_SS_L1 = flux_layer("flux_single_l1_9216x3072x21504", 9216, 3072, 21504, r_s=32, r=64)
FLUX_SS_L2 = flux_layer("flux_single_l2_9216x15360x3072", 9216, 15360, 3072, r_s=32, r=64)

QUANT_SWEEP: List[QuantSpec] = [
    QuantSpec("quant_4608x3072", 4608, 3072, 32, 0.01, 10.0),
    QuantSpec("quant_4608x12288", 4608, 12288, 32, 0.01, 10.0),
    QuantSpec("quant_9216x15360", 9216, 15360, 32, 0.01, 10.0),
    QuantSpec("quant_36864x21504", 36864, 21504, 32, 0.01, 10.0),
]

LAYERS: Dict[str, LayerSpec] = {s.name: s for s in
                                 [PARITY_SMALL, FLUX_QKV, FLUX_MLP_UP, FLUX_MLP_DOWN,
                                  FLUX_SS_L1, FLUX_SS_L2]}


def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


def _orthonormal(gen: torch.Generator, n: int, k: int) -> torch.Tensor:
    """n x k matrix with orthonormal columns (QR of a Gaussian block, fp64)."""
    g = torch.randn(n, k, generator=gen, dtype=torch.float32).double()
    q, rr = torch.linalg.qr(g)
    # fix the sign convention so the draw is a deterministic function of the seed
    q = q * torch.sign(torch.diagonal(rr)).unsqueeze(0)
    return q


@dataclasses.dataclass
class LayerInputs:
    """Raw (pre-prep) inputs of one layer, all on the CPU."""

    spec: LayerSpec
    x: torch.Tensor        # bf16 [M, K]
    w: torch.Tensor        # bf16 [N, K]  full pretrained weight (split offline)
    lora_a: torch.Tensor   # bf16 [r, K]
    lora_b: torch.Tensor   # bf16 [N, r]
    dy: torch.Tensor       # bf16 [M, N]
    outlier_cols: torch.Tensor


def make_layer_inputs(spec: LayerSpec, seed: int = 0, rows: Optional[int] = None) -> LayerInputs:
    """Draw X, W, A, B and dY for ``spec``.  ``rows`` (optional) draws only the
    first ``rows`` token rows of X and dY (the weights are unchanged)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    M = spec.M if rows is None else rows
    cols = torch.randperm(spec.K, generator=gen)[: spec.n_outlier_cols]
    x = torch.randn(M, spec.K, generator=gen, dtype=torch.float32)
    x[:, cols] *= spec.outlier_gain
    w = torch.randn(spec.N, spec.K, generator=gen, dtype=torch.float32).double() * spec.w_std
    up = _orthonormal(gen, spec.N, spec.plant_rank)
    vp = _orthonormal(gen, spec.K, spec.plant_rank)
    w = w + spec.plant_sigma * (up @ vp.T)
    a = torch.randn(spec.r, spec.K, generator=gen, dtype=torch.float32) / math.sqrt(spec.K)
    b = torch.randn(spec.N, spec.r, generator=gen, dtype=torch.float32) * spec.b_std
    dy = torch.randn(M, spec.N, generator=gen, dtype=torch.float32) * spec.dy_std
    return LayerInputs(spec=spec, x=_bf16(x), w=_bf16(w.float()), lora_a=_bf16(a),
                       lora_b=_bf16(b), dy=_bf16(dy), outlier_cols=cols)


def make_quant_input(spec: QuantSpec, seed: int = 0, rows: Optional[int] = None):
    """bf16 [rows, cols] ~ N(0, 1) with each entry independently (p) replaced by a
    Laplace(0, b) draw, plus the fused down-projection factor [r_down, cols] with
    variance 1/cols.  Returns (x, down)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    R = spec.rows if rows is None else rows
    x = torch.randn(R, spec.cols, generator=gen, dtype=torch.float32)
    heavy = torch.rand(R, spec.cols, generator=gen) < spec.p_heavy
    u = torch.rand(R, spec.cols, generator=gen, dtype=torch.float32) - 0.5
    lap = -spec.laplace_b * torch.sign(u) * torch.log1p(-2.0 * u.abs())
    x = torch.where(heavy, lap, x)
    down = torch.randn(spec.r_down, spec.cols, generator=gen, dtype=torch.float32) / math.sqrt(spec.cols)
    return _bf16(x), _bf16(down)


def make_gaussian_bf16(shape, std: float, seed: int) -> torch.Tensor:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return _bf16(torch.randn(*shape, generator=gen, dtype=torch.float32) * std)
