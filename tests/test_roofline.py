"""The roofline arithmetic the benchmark reports against (CPU only).

The algorithmic FLOPs and bytes of each workload are checked against figures
worked out by hand from the layer sizes (rounded as printed there), and
against an enumeration of the block's GEMMs written out one by one."""
import dataclasses

import pytest

from mixture_experts_ffn_16_b200 import roofline
from mixture_experts_ffn_16_b200.inputs import CONFIGS

# (GFLOP, GB, relative rounding of the printed figure), all experts touched
HAND = {
    "prefill_softmax": (236.2, 1.652, 5e-4),
    "prefill_sigmoid": (2087.0, 9.85, 1e-3),
    "decode_sqrt_softplus": (18.0, 12.9, 5e-3),
    "large_imbalanced": (9591.0, 20.3, 5e-3),
}


def gemms(c):
    """Every GEMM of one step as (rows, cols, depth)."""
    g = [(c.T, c.E, c.d)]                                   # router
    g += [(c.T * c.k, c.f, c.d)] * 2                        # routed gate, up
    g += [(c.T * c.k, c.d, c.f)]                            # routed down
    for _ in range(c.S):
        g += [(c.T, c.fs, c.d)] * 2 + [(c.T, c.d, c.fs)]    # shared gate, up, down
    return g


@pytest.mark.parametrize("name", list(HAND))
def test_block_cost_matches_hand_figures(name):
    c = CONFIGS[name]
    flops, bytes_ = roofline.block_cost(c)
    gf, gb, rel = HAND[name]
    assert flops / 1e9 == pytest.approx(gf, rel=rel)
    assert bytes_ / 1e9 == pytest.approx(gb, rel=rel)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_flops_are_the_sum_over_gemms(name):
    c = CONFIGS[name]
    expect = sum(2.0 * m * n * k for m, n, k in gemms(c))
    flops, _ = roofline.block_cost(c)
    assert flops == expect
    kc = roofline.kernel_costs(c)
    assert kc["route"][0] + kc["gate_up"][0] + kc["down"][0] == expect


@pytest.mark.parametrize("name", list(CONFIGS))
def test_block_bytes_count_each_weight_once(name):
    c = CONFIGS[name]
    _, b_all = roofline.block_cost(c)
    weights = 2.0 * (c.E * c.d + c.E * 3 * c.f * c.d + c.S * 3 * c.fs * c.d)
    io = 2.0 * 2 * c.T * c.d + 8.0 * c.T * c.k          # x in, out, topk_idx and topk_w
    assert b_all == weights + io
    # untouched experts do not count
    _, b_half = roofline.block_cost(c, touched=c.E // 2)
    assert b_all - b_half == pytest.approx(2.0 * (c.E - c.E // 2) * 3 * c.f * c.d)


def test_fp8_weight_bytes():
    c = dataclasses.replace(CONFIGS["decode_sqrt_softplus"], fp8=True)
    assert roofline.weight_bytes(c) == 1.0 + 1.0 / 32.0
    assert roofline.weight_bytes(CONFIGS["decode_sqrt_softplus"]) == 2.0
    _, b8 = roofline.block_cost(c)
    _, b16 = roofline.block_cost(CONFIGS["decode_sqrt_softplus"])
    expert = c.E * 3 * c.f * c.d + c.S * 3 * c.fs * c.d
    assert b16 - b8 == pytest.approx(expert * (2.0 - 33.0 / 32.0))


def test_traffic_figures_only_for_known_revisions(monkeypatch):
    assert roofline.measured_traffic("prefill_softmax", "combine") is None
    assert roofline.measured_traffic("tiny", "gate_up") is None
    monkeypatch.setattr(roofline, "_gemm_source_sha", lambda: "0000000000000000")
    assert roofline.measured_traffic("prefill_softmax", "gate_up") is None
