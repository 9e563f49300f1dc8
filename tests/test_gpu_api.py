"""Behaviour of the C ABI on a B200: the step-by-step entry points, the host
buffer entry point, determinism, the permute bookkeeping (exact integers
against a brute-force counting sort), error codes and the bounded-wait status."""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_ffn_16_b200 import api
from mixture_experts_ffn_16_b200.inputs import MoEConfig, make_inputs

pytestmark = pytest.mark.gpu

CFG = MoEConfig("api_case", T=333, d=256, E=20, k=4, f=192, S=1, fs=128, score_fn="sigmoid",
                bias_std=0.1, seed=31)


@pytest.fixture(scope="module")
def case():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    api.load()
    inp = make_inputs(CFG, device="cuda")
    layer = api.MoELayer(CFG, inp)
    return inp, layer


def test_forward_is_bitwise_deterministic(case):
    inp, layer = case
    o1, i1, w1 = [t.clone() for t in layer()]
    layer.workspace.fill_(0xA5)            # stale workspace contents must not matter
    o2, i2, w2 = [t.clone() for t in layer()]
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(i1, i2) and torch.equal(w1, w2)


def test_steps_equal_forward(case):
    inp, layer = case
    o1, i1, w1 = [t.clone() for t in layer()]
    o2, i2, w2 = [t.clone() for t in layer.steps()]
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(i1, i2) and torch.equal(w1, w2)


def test_host_entry_point_equals_device_entry_point(case):
    inp, layer = case
    o1, i1, w1 = [t.clone() for t in layer()]
    T, d, k = CFG.T, CFG.d, CFG.k
    xh = inp["x"].cpu().pin_memory()
    oh = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    ih = torch.empty((T, k), dtype=torch.int32).pin_memory()
    wh = torch.empty((T, k), dtype=torch.float32).pin_memory()
    api.moe_forward_host(layer.shape, xh, inp["W_router"], inp["expert_bias"], inp["W_gate"], inp["W_up"],
                         inp["W_down"], inp["W_shared_gate"], inp["W_shared_up"], inp["W_shared_down"],
                         CFG.score_fn, CFG.norm_topk, CFG.route_scale, oh, ih, wh, layer.workspace)
    torch.cuda.synchronize()
    assert torch.equal(o1.cpu().view(torch.int16), oh.view(torch.int16))
    assert torch.equal(i1.cpu(), ih) and torch.equal(w1.cpu(), wh)


def test_row_permutation_does_not_change_output(case):
    """Permuting the tokens permutes the outputs bit for bit (rows are
    independent in every kernel and the combine order is fixed per token)."""
    inp, layer = case
    o1, i1, _ = [t.clone() for t in layer()]
    perm = torch.randperm(CFG.T, generator=torch.Generator().manual_seed(3)).cuda()
    o2, i2, _ = layer(inp["x"][perm].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(o1[perm].view(torch.int16), o2.view(torch.int16))
    assert torch.equal(i1[perm], i2)


def _synthetic_routing(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    w = torch.rand((T, k), generator=g, dtype=torch.float32)
    return idx, w


@pytest.mark.parametrize("T,E,k", [(333, 20, 4), (1, 8, 8), (1000, 64, 8), (257, 2048, 32), (600, 3, 1)])
def test_permute_matches_brute_force_counting_sort(T, E, k):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    shape = api.make_shape(T, 128, E, k, 128, 1, 128)
    ws = api.alloc_workspace(shape)
    ws.zero_()       # the error word is cleared by moe_route, which this test skips
    idx, w = _synthetic_routing(T, E, k, seed=T + E + k)
    api.moe_permute(shape, idx.cuda(), w.cuda(), ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == api.MOE_OK
    counts = api.workspace_view(ws, shape, "counts", torch.int32, (E,)).cpu().numpy()
    roff = api.workspace_view(ws, shape, "offsets", torch.int32, (E + 1,)).cpu().numpy()
    idx_n = idx.numpy()
    exp_counts = np.bincount(idx_n.ravel(), minlength=E)
    assert np.array_equal(counts, exp_counts)
    # segments are padded to 16 rows, or to 32 when the expert GEMMs run on CTA pairs
    ok_pads = []
    for P in (16, 32):
        pad = (exp_counts + P - 1) // P * P
        if np.array_equal(roff, np.concatenate([[0], np.cumsum(pad)])):
            ok_pads.append(P)
    assert len(ok_pads) >= 1, roff
    exp_roff = roff.astype(np.int64)
    rows = int(exp_roff[-1])
    perm = api.workspace_view(ws, shape, "perm", torch.int32, (rows,)).cpu().numpy()
    roww = api.workspace_view(ws, shape, "row_w", torch.float32, (rows,)).cpu().numpy()
    inv = api.workspace_view(ws, shape, "inv", torch.int32, (T, k)).cpu().numpy()
    for e in range(E):
        toks = [t for t in range(T) if e in idx_n[t]]          # ascending token order
        seg = perm[exp_roff[e]:exp_roff[e] + exp_counts[e]]
        assert seg.tolist() == toks
        assert (perm[exp_roff[e] + exp_counts[e]:exp_roff[e + 1]] == 0).all()
        assert (roww[exp_roff[e] + exp_counts[e]:exp_roff[e + 1]] == 0).all()
    for t in range(T):
        for j in range(k):
            r = inv[t, j]
            assert perm[r] == t and roww[r] == w[t, j].item()
            assert exp_roff[idx_n[t, j]] <= r < exp_roff[idx_n[t, j]] + exp_counts[idx_n[t, j]]


def _skewed_routing(T, E, k, seed):
    """k distinct experts per token, drawn with probability proportional to
    rank^-1.1 over a shuffled ranking, so that expert sizes vary by an order
    of magnitude and some experts get no token."""
    rng = np.random.default_rng(seed)
    p = 1.0 / (1.0 + rng.permutation(E)) ** 1.1
    p /= p.sum()
    idx = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    w = rng.random((T, k), dtype=np.float32)
    return torch.from_numpy(idx), torch.from_numpy(w)


def _check_work_list(units, E, seg, label):
    """units: int [U, 4] {group, weight block, first row, rows}; seg(g) = the
    group's row range.  Every group's runs tile its range once for each weight
    block, the shared groups (>= E) come first, each routed group's units are
    contiguous; returns the routed groups in list order."""
    groups = units[:, 0]
    shared = groups >= E
    if shared.any():
        assert shared[:shared.sum()].all(), label + ": shared units first"
    order, seen = [], set()
    prev = None
    for g in groups[~shared]:
        g = int(g)
        if g != prev:
            assert g not in seen, f"{label}: expert {g}'s units are not contiguous"
            seen.add(g)
            order.append(g)
            prev = g
    nwb = None
    for g in np.unique(groups):
        sel = units[groups == g]
        lo, hi = seg(int(g))
        wbs = np.unique(sel[:, 1])
        assert np.array_equal(wbs, np.arange(len(wbs))), f"{label}: group {g} weight blocks {wbs}"
        if g < E:
            nwb = len(wbs) if nwb is None else nwb
            assert len(wbs) == nwb, f"{label}: routed groups with different weight-block counts"
        for wb in wbs:
            runs = sel[sel[:, 1] == wb]
            runs = runs[np.argsort(runs[:, 2])]
            assert runs[0, 2] == lo and (runs[:-1, 2] + runs[:-1, 3] == runs[1:, 2]).all() \
                and runs[-1, 2] + runs[-1, 3] == hi, f"{label}: group {g} block {wb} runs {runs.tolist()} vs [{lo}, {hi})"
            assert (runs[:, 3] > 0).all() and (runs[:, 3] % 16 == 0).all()
    return order


@pytest.mark.parametrize("T,E,k,S", [(3000, 40, 4, 2), (500, 64, 2, 1), (200, 300, 6, 0)])
def test_work_lists_tile_every_segment_in_interleaved_size_order(T, E, k, S):
    """After moe_permute, the gate/up and down work lists cover each expert's
    padded row segment once per weight block with runs of at most 256 rows,
    the shared experts' rows [0, Tp) likewise and first, and the
    routed experts in the order largest, smallest, 2nd largest, 2nd smallest,
    ... by padded rows (ties: lower expert index first), each expert's units
    together.  Cases: CTA pairs (300 rows per expert), single CTAs, and many
    empty experts."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    shape = api.make_shape(T, 256, E, k, 384, S, 256 if S else 0)
    ws = api.alloc_workspace(shape)
    ws.zero_()
    idx, w = _skewed_routing(T, E, k, seed=T + E)
    api.moe_permute(shape, idx.cuda(), w.cuda(), ws)
    torch.cuda.synchronize()
    assert api.moe_device_status(ws) == api.MOE_OK
    nun = api.workspace_view(ws, shape, "work_counts", torch.int32, (4,)).cpu().numpy()
    roff = api.workspace_view(ws, shape, "offsets", torch.int32, (E + 1,)).cpu().numpy().astype(np.int64)
    pad = roff[1:] - roff[:-1]
    assert nun[2] == roff[E]
    for name, n in (("work_gate_up", nun[0]), ("work_down", nun[1])):
        units = api.workspace_view(ws, shape, name, torch.int32, (int(n), 4)).cpu().numpy().astype(np.int64)
        assert units[:, 3].max() <= 256
        sh = units[units[:, 0] >= E]
        assert set(np.unique(sh[:, 0]).tolist()) == set(range(E, E + S))
        tp = int((sh[:, 2] + sh[:, 3]).max()) if S else 0          # T rounded up to the row padding
        assert S == 0 or tp in (-(-T // 16) * 16, -(-T // 32) * 32)
        seg = lambda g: (0, tp) if g >= E else (int(roff[g]), int(roff[g + 1]))
        order = _check_work_list(units, E, seg, name)
        rank = sorted(range(E), key=lambda e: (-pad[e], e))
        pos = [2 * r if r < (E + 1) // 2 else 2 * (E - 1 - r) + 1 for r in range(E)]
        expect = [None] * E
        for r, e in enumerate(rank):
            expect[pos[r]] = e
        assert order == [e for e in expect if pad[e] > 0], name


def test_invalid_routing_is_reported_not_faulted():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    T, E, k = 40, 8, 2
    shape = api.make_shape(T, 128, E, k, 128, 0, 0)
    ws = api.alloc_workspace(shape)
    ws.zero_()
    idx = torch.zeros((T, k), dtype=torch.int32)
    idx[:, 1] = 1
    idx[3, 1] = 0          # repeated expert
    idx[7, 0] = 99         # out of range
    api.moe_permute(shape, idx.cuda(), torch.ones((T, k)).cuda(), ws)
    assert api.moe_device_status(ws) == api.MOE_ERR_INVALID_ARG


def test_nonfinite_router_inputs_stay_in_range_and_are_reported(case):
    """A token row of x that is all NaN, and a NaN expert bias: every token
    still gets k distinct experts in [0, E) (a NaN key ranks with -inf, below
    every other key, ties to the lower index), the other tokens' routing and
    outputs are those of a run without the NaN row, and moe_device_status
    reports MOE_ERR_NONFINITE."""
    inp, layer = case
    T, E, k = CFG.T, CFG.E, CFG.k
    bad_t = 5
    x_clean = inp["x"].clone()
    x_clean[bad_t] = 0.0
    o_ref, i_ref, w_ref = [t.clone() for t in layer(x_clean)]
    assert api.moe_device_status(layer.workspace) == api.MOE_OK
    x_nan = x_clean.clone()
    x_nan[bad_t] = float("nan")
    o, i, w = [t.clone() for t in layer(x_nan)]
    assert api.moe_device_status(layer.workspace) == api.MOE_ERR_NONFINITE
    idx = i.cpu().numpy()
    assert ((idx >= 0) & (idx < E)).all()
    assert all(len(set(r)) == k for r in idx.tolist())
    assert idx[bad_t].tolist() == list(range(k))          # all keys NaN: the lowest indices
    keep = torch.ones(T, dtype=torch.bool)
    keep[bad_t] = False
    assert torch.equal(i[keep.cuda()], i_ref[keep.cuda()])
    assert torch.equal(w[keep.cuda()], w_ref[keep.cuda()])
    assert torch.equal(o[keep.cuda()].view(torch.int16), o_ref[keep.cuda()].view(torch.int16))
    # a NaN selection bias: that expert ranks last for every token
    bias = inp["expert_bias"].clone()
    bias[3] = float("nan")
    api.moe_route(layer.shape, x_clean, inp["W_router"], bias, CFG.score_fn, CFG.norm_topk, CFG.route_scale,
                  layer.topk_idx, layer.topk_w, layer.workspace)
    assert api.moe_device_status(layer.workspace) == api.MOE_ERR_NONFINITE
    idx = layer.topk_idx.cpu().numpy()
    assert ((idx >= 0) & (idx < E)).all() and not (idx == 3).any()
    assert torch.isfinite(layer.topk_w).all()
    layer()
    assert api.moe_device_status(layer.workspace) == api.MOE_OK


def test_status_ok_then_bounded_wait_timeout_then_usable(case):
    inp, layer = case
    layer()
    assert api.moe_device_status(layer.workspace) == api.MOE_OK
    api.moe_debug_wait_timeout(layer.workspace, 5_000_000)      # 5 ms, nothing ever arrives
    assert api.moe_device_status(layer.workspace) == api.MOE_ERR_DEVICE_TIMEOUT
    out, _, _ = layer()                                         # context still usable
    assert api.moe_device_status(layer.workspace) == api.MOE_OK
    assert torch.isfinite(out.float()).all()


def test_error_codes_enqueue_nothing(case):
    inp, layer = case
    s = layer.shape
    out = torch.full((CFG.T, CFG.d), 7.0, dtype=torch.bfloat16, device="cuda")
    lib = api.load()

    def call(shape=s, x=inp["x"], ws=layer.workspace, ws_bytes=None, score=1, out_t=out):
        return lib.moe_forward(ctypes.byref(shape), ctypes.c_void_p(x if isinstance(x, int) else x.data_ptr()),
                               ctypes.c_void_p(inp["W_router"].data_ptr()),
                               ctypes.c_void_p(inp["expert_bias"].data_ptr()),
                               ctypes.c_void_p(inp["W_gate"].data_ptr()), ctypes.c_void_p(inp["W_up"].data_ptr()),
                               ctypes.c_void_p(inp["W_down"].data_ptr()),
                               ctypes.c_void_p(inp["W_shared_gate"].data_ptr()),
                               ctypes.c_void_p(inp["W_shared_up"].data_ptr()),
                               ctypes.c_void_p(inp["W_shared_down"].data_ptr()), None, score, 1, 1.0,
                               ctypes.c_void_p(out_t.data_ptr()), ctypes.c_void_p(layer.topk_idx.data_ptr()),
                               ctypes.c_void_p(layer.topk_w.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                               ws.numel() if ws_bytes is None else ws_bytes, None)

    assert call(x=0) == api.MOE_ERR_INVALID_ARG
    assert call(score=7) == api.MOE_ERR_INVALID_ARG
    assert call(x=inp["x"].data_ptr() + 2) == api.MOE_ERR_UNSUPPORTED
    assert call(ws_bytes=16) == api.MOE_ERR_WORKSPACE
    bad = api.make_shape(CFG.T, CFG.d, CFG.E, CFG.E + 1, CFG.f, CFG.S, CFG.fs)
    assert call(shape=bad) == api.MOE_ERR_INVALID_ARG
    bad = api.make_shape(CFG.T, 100, CFG.E, CFG.k, CFG.f, CFG.S, CFG.fs)
    assert call(shape=bad) == api.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (out.float() == 7.0).all()        # nothing was enqueued
    assert call() == api.MOE_OK
    torch.cuda.synchronize()
