"""moe_route_noalloc: the routing step for callers that cannot allocate device
memory (for example an inference-engine plugin whose per-call hook may not
allocate, or a process whose device memory is reserved up front by another
allocator).  Its scratch is an array built into the library, so the caller
passes only inputs and outputs.

Checked through the C ABI against moe_route (the workspace entry point) on
two calls in a row, and against the fp64 oracle by the same index, near-tie
and weight rules as moe_route; also a shape whose partial logits would not fit
the built-in scratch (the call then sums fewer slices of d, in another order),
and that a shape beyond the built-in scratch is refused before anything is
enqueued.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_16_b200 import api
from mixture_experts_ffn_16_b200.inputs import CONFIGS, MoEConfig, bf16_bits, make_inputs, oracle_args

from parity_util import W_ATOL, W_RTOL, check_routing

pytestmark = pytest.mark.gpu


def _route_with_workspace(cfg, inp):
    shape = api.shape_of(cfg)
    ws = api.alloc_workspace(shape)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device="cuda")
    api.moe_route(shape, inp["x"], inp["W_router"], inp["expert_bias"], cfg.score_fn, cfg.norm_topk,
                  cfg.route_scale, idx, w, ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == api.MOE_OK
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("cfg", [
    CONFIGS["prefill_softmax"],
    MoEConfig("noalloc_sigmoid_bias", T=777, d=512, E=96, k=6, f=128, S=1, fs=128, score_fn="sigmoid",
              bias_std=0.1, route_scale=2.5, seed=41),
], ids=lambda c: c.name)
def test_noalloc_route_matches_workspace_route_twice(oracle_mod, cfg):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.load()
    inp = make_inputs(cfg, device="cuda")
    ref_idx, ref_w = _route_with_workspace(cfg, inp)
    shape = api.shape_of(cfg)
    for _ in range(2):
        idx = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.k), -7.0, dtype=torch.float32, device="cuda")
        api.moe_route_noalloc(shape, inp["x"], inp["W_router"], inp["expert_bias"], cfg.score_fn,
                              cfg.norm_topk, cfg.route_scale, idx, w)
        torch.cuda.synchronize()
        got_idx, got_w = idx.cpu().numpy(), w.cpu().numpy()
        assert np.array_equal(got_idx, ref_idx)
        np.testing.assert_allclose(got_w, ref_w, rtol=W_RTOL, atol=W_ATOL)
    rep = check_routing(oracle_mod, cfg, oracle_args(inp), got_idx, got_w)
    print(cfg.name, rep)


def test_noalloc_route_with_fewer_slices_matches_oracle(oracle_mod, parity_log):
    """T = 8448, d = 2048, E = 256: T * E fp32 logits (8.25 MiB) fit the 16 MiB
    scratch, but the workspace plan's two slices of d (16.5 MiB of partial
    logits) do not, so the call sums the logits over one slice: a different
    fp32 summation order than moe_route, checked against the oracle by the
    near-tie rule."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.load()
    cfg = MoEConfig("noalloc_one_slice", T=8448, d=2048, E=256, k=8, f=64, S=0, fs=0, score_fn="sigmoid",
                    bias_std=0.1, seed=42)
    shape = api.shape_of(cfg)
    off, nbytes = api.moe_workspace_region(shape, "logits")
    assert nbytes > 16 * 2**20 >= cfg.T * cfg.E * 4         # the branch that cuts the slices
    inp = {n: t for n, t in make_inputs(cfg, device="cuda").items()
           if n in ("x", "W_router", "expert_bias")}
    for _ in range(2):
        idx = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
        w = torch.full((cfg.T, cfg.k), -7.0, dtype=torch.float32, device="cuda")
        api.moe_route_noalloc(shape, inp["x"], inp["W_router"], inp["expert_bias"], cfg.score_fn,
                              cfg.norm_topk, cfg.route_scale, idx, w)
        torch.cuda.synchronize()
        host = {"x": bf16_bits(inp["x"]), "W_router": bf16_bits(inp["W_router"]),
                "expert_bias": inp["expert_bias"].cpu().numpy()}
        rep = check_routing(oracle_mod, cfg, host, idx.cpu().numpy(), w.cpu().numpy())
        assert rep["tokens"] == cfg.T
    parity_log.append(dict(case="noalloc_one_slice", check="routing", **rep))


def test_noalloc_route_refuses_shapes_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.load()
    cfg = CONFIGS["large_imbalanced"]          # T * E = 14.7M logits > 4,194,304
    shape = api.shape_of(cfg)
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((E, d), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    with pytest.raises(api.MoEError) as ei:
        api.moe_route_noalloc(shape, x, wr, None, "softmax", True, 1.0, idx, w)
    assert ei.value.status == api.MOE_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert (idx == -7).all() and (w == -7.0).all()      # nothing was enqueued
