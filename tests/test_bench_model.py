"""The bench's layer roofline model (no GPU needed) against the figures the
method's cost model gives for each workload: tensor work 2 T k d^2 flops and
the algorithmic bytes x + y + d^2/4 (2-bit base) + 2 N (d/2) log2 d * 4
(fp32 angles) + T N 4 (fp32 logits), worked out by hand per workload."""
import pytest

import bench
from ternary_moe_butterfly_b200 import workloads as wl

# (GFLOP, MB) per workload, from the closed forms above
EXPECTED = {
    "tiny": (0.0021, 0.083),
    "headline": (4.295, 10.68),
    "many_experts": (17.18, 55.12),
    "llm_width": (549.8, 153.1),
    "vit": (26.44, 57.75),
}


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_layer_model_matches_hand_worked_figures(name):
    gflop, mb = EXPECTED[name]
    flops, bmin = bench.layer_model(wl.WORKLOADS[name])
    assert flops / 1e9 == pytest.approx(gflop, rel=3e-3)
    assert bmin / 1e6 == pytest.approx(mb, rel=3e-3)


def test_headline_roofline_times():
    # at the measured peaks the headline layer is tensor-bound: 2.570 us of
    # tensor time against 1.636 us of HBM time
    flops, bmin = bench.layer_model(wl.WORKLOADS["headline"])
    assert flops / 1670.9e12 * 1e6 == pytest.approx(2.570, abs=1e-3)
    assert bmin / 6530.6e9 * 1e6 == pytest.approx(1.636, abs=1e-3)
