"""Host-side logic of bench.py (no GPU): the algorithmic FLOP counts behind the metric,
checked against the per-config totals of the workload table (FP4: 4·M·N·K per layer for
the forward and dX GEMMs; bf16: the stabilizer and LoRA projections and the adapter
gradients), and the choice of the roofline peak."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


# (layers as (M, K, N, r_s, r), FP4 GFLOP, bf16 GFLOP) as the workload table states them
TABLE = [
    ("C1", [(256, 512, 512, 16, 8)], 0.27, 0.03),
    ("C2", [(4608, 3072, 9216, 32, 16)], 521.8, 12.7),
    ("C3", [(4608, 3072, 12288, 32, 32), (4608, 12288, 3072, 32, 32)], 1391.6, 45.3),
    ("C5", [(9216, 3072, 21504, 32, 64), (9216, 15360, 3072, 32, 64)], 4174.7, 202.9),
]


@pytest.mark.parametrize("name,layers,fp4_g,bf16_g", TABLE, ids=[t[0] for t in TABLE])
def test_step_flops_match_the_workload_table(name, layers, fp4_g, bf16_g):
    b = _bench()
    fp4 = sum(b.layer_flops(*l)[0] for l in layers) / 1e9
    bf16 = sum(b.layer_flops(*l)[1] for l in layers) / 1e9
    assert fp4 == pytest.approx(fp4_g, abs=0.06)
    assert bf16 == pytest.approx(bf16_g, abs=0.06)


@pytest.mark.parametrize("layer", [(4608, 3072, 9216, 32, 16), (9216, 15360, 3072, 32, 64), (256, 512, 512, 16, 0)])
def test_pass_flops_add_up_to_the_step(layer):
    b = _bench()
    fwd, bwd = b.pass_flops(*layer)
    fp4, bf16 = b.layer_flops(*layer)
    assert fwd + bwd == pytest.approx(fp4 + bf16, rel=1e-12)
    M, K, N, r_s, r = layer
    assert fwd == pytest.approx(2.0 * M * N * K + 2.0 * (r_s + r) * (M * K + M * N), rel=1e-12)


def test_roofline_peak_follows_the_power_state():
    b = _bench()
    hbm, burst, sustained, src = b.peaks()
    capped = b.gemm_roofline_peak({"reasons": ["sw_power_cap"]})
    free = b.gemm_roofline_peak({"reasons": []})
    assert capped[0] == pytest.approx(sustained * b.NOMINAL_FP4_OVER_BF16)
    assert free[0] == pytest.approx(burst * b.NOMINAL_FP4_OVER_BF16)
    assert capped[1] == free[1] == pytest.approx(burst * b.NOMINAL_FP4_OVER_BF16)
    assert capped[2] == free[2] == pytest.approx(sustained * b.NOMINAL_FP4_OVER_BF16)
    assert "sustained" in capped[3] and "burst" in free[3]
    assert sustained <= burst and hbm > 0


def test_gemm_traffic_is_reported_only_for_the_recorded_sources():
    b = _bench()
    rec = b.GEMM_DRAM_BYTES["single"]
    assert b.gemm_traffic("single") in (rec[0], None)
    assert (b.gemm_traffic("single") is not None) == (b.gemm_sources_hash() == rec[1])
    assert b.gemm_traffic("qkv") is None
