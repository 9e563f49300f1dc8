"""The seeded synthetic inputs (CPU only): the FP8 weight recipe, the skewed
router of the large workload, and determinism of the generator."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_16_b200.inputs import CONFIGS, MoEConfig, make_inputs, quantize_mxfp8


def e4m3_table():
    """Value of every finite E4M3FN code, decoded from the bit fields here
    (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 is
    subnormal; 0x7F and 0xFF are NaN)."""
    vals = {}
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            continue
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        vals[c] = -v if s else v
    return vals


TABLE = e4m3_table()
CODES = np.array(sorted(TABLE), dtype=np.int64)
VALUES = np.array([TABLE[c] for c in CODES])


def nearest_code_value(v):
    """Nearest E4M3 value to v by exhaustive search; a tie goes to the code
    with an even mantissa."""
    d = np.abs(VALUES - v)
    best = d.min()
    cand = CODES[d == best]
    even = [c for c in cand if c & 1 == 0]
    return TABLE[int((even or list(cand))[0])]


def make_weights(seed, G=2, rows=8, K=128):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(G, rows, K, generator=g) * 0.02
    w[0, 0, :32] = 0.0                           # an all-zero block
    w[0, 1, 32:64] *= 1e-30                      # a block far below E4M3's normal range
    if G > 1 and rows > 2 and K >= 96:
        w[1, 2, 64:96] = 448.0 * 2.0 ** -3       # a block whose maximum is exactly 448 * 2^-3
    return w.to(torch.bfloat16)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_fp8_recipe_scale_is_the_smallest_that_fits(seed):
    w = make_weights(seed)
    codes, scales = quantize_mxfp8(w)
    G, rows, K = w.shape
    assert codes.shape == (G, rows, K) and scales.shape == (G, K // 32, rows)
    wf = w.float().numpy().astype(np.float64)
    u = scales.numpy().astype(np.int64)
    for g in range(G):
        for r in range(rows):
            for b in range(K // 32):
                blk = wf[g, r, 32 * b:32 * b + 32]
                amax = np.abs(blk).max()
                ub = u[g, b, r]
                if amax == 0:
                    assert ub == 127
                    continue
                s = 2.0 ** (ub - 127)
                assert amax / s <= 448.0                         # fits
                if ub > 1:
                    assert amax / (s / 2) > 448.0                # half the scale would not
    assert u[1, 2, 2] == 127 - 3                                 # 448 * 2^-3 fits exactly at 2^-3


@pytest.mark.parametrize("seed", [0, 3])
def test_fp8_recipe_codes_are_nearest_ties_to_even(seed):
    w = make_weights(seed, G=1, rows=4, K=64)
    codes, scales = quantize_mxfp8(w)
    wf = w.float().numpy().astype(np.float64)
    c = codes.numpy()
    u = scales.numpy().astype(np.int64)
    for r in range(4):
        for k in range(64):
            s = 2.0 ** (u[0, k // 32, r] - 127)
            want = nearest_code_value(wf[0, r, k] / s)
            got = TABLE[int(c[0, r, k])]
            assert got == want, (r, k, wf[0, r, k], s, got, want)


def test_fp8_recipe_plants_ties():
    """Values exactly halfway between two E4M3 values go to the even mantissa."""
    # scale 2^0 (block maximum 448): 1.0625 lies halfway between 1.0 (m=0) and 1.125 (m=1)
    w = torch.zeros(1, 1, 32)
    w[0, 0, 0] = 448.0
    w[0, 0, 1] = 1.0625
    w[0, 0, 2] = 1.1875                          # between 1.125 (m=1) and 1.25 (m=2): goes to 1.25
    codes, scales = quantize_mxfp8(w.to(torch.bfloat16))
    assert int(scales[0, 0, 0]) == 127
    assert TABLE[int(codes[0, 0, 1])] == 1.0
    assert TABLE[int(codes[0, 0, 2])] == 1.25


def test_generator_is_deterministic():
    cfg = MoEConfig("det", T=32, d=128, E=8, k=2, f=64, S=1, fs=64, seed=7)
    a = make_inputs(cfg, device="cpu")
    b = make_inputs(cfg, device="cpu")
    for key, v in a.items():
        if isinstance(v, torch.Tensor):
            assert torch.equal(v, b[key]), key


def test_large_workload_skew_lives_in_the_data():
    """The skew reading: x[:, 0] = 1 and W_router[e, 0] = bf16(0.5 ln(1/r_e)) for
    a seeded permutation r of 1..E."""
    cfg = CONFIGS["large_imbalanced"]
    assert cfg.skew == "zipf_rank"
    small = MoEConfig("skew_small", T=16, d=128, E=cfg.E, k=4, f=64, S=0, fs=0, skew="zipf_rank", seed=cfg.seed)
    inp = make_inputs(small, device="cpu")
    ranks = inp["ranks"].numpy()
    assert np.array_equal(np.sort(ranks), np.arange(1, cfg.E + 1))
    assert torch.all(inp["x"][:, 0].float() == 1.0)
    want = torch.tensor(0.5 * np.log(1.0 / ranks.astype(np.float64))).to(torch.bfloat16)
    assert torch.equal(inp["W_router"][:, 0], want)
