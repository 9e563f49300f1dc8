"""Comparison of the CUDA path with the fp64 oracle.

TEST INFRASTRUCTURE ONLY, like the rest of this package: used by the tests
and by the benchmark's CPU-baseline leg (which compares the GPU's results of
its token sample with the oracle's).  Takes numpy arrays; imports nothing of
the CUDA path.

Rules (from the block's specification):
  * top-k indices match exactly, except tokens whose oracle k-th and (k+1)-th
    selection keys differ by less than 1e-5 relative (|a-b|/max(|a|,|b|));
    such a token may pick any experts of that near-tie group, and it is
    counted.  Inside the picked set the order may differ only between
    neighbours whose oracle keys are within 1e-5 relative (also counted).
  * combine weights match the oracle's for the same experts within
    rtol 1e-5 (+ atol 1e-6 for tiny softmax probabilities).
  * outputs: max |out - oracle| <= 2e-2 * max |oracle| over the checked tokens,
    with bf16 inputs and fp32 accumulation on the GPU.
For a near-tie token the oracle itself is re-run with the alternative set of
experts that the oracle's own keys allow (built from the oracle's ordering,
never from the GPU's output); the GPU's set must be one of those sets, and
its output is compared with that run.
"""
from __future__ import annotations

import itertools

import numpy as np

TIE_REL = 1e-5
W_RTOL = 1e-5
W_ATOL = 1e-6
OUT_TOL = 2e-2


def rel_gap(a, b):
    m = max(abs(a), abs(b))
    return 0.0 if m == 0 else abs(a - b) / m


def oracle_candidates(keys_row, order_row, k, max_group=6):
    """Index sets the rule allows, from the oracle's keys of one token: the
    oracle's own top-k first, then sets that swap members of the near-tie group
    at the k-th place."""
    E = keys_row.shape[0]
    base = [int(e) for e in order_row[:k]]
    if k >= E:
        return [base]
    ck = keys_row[base[-1]]
    group = [e for e in range(E) if rel_gap(keys_row[e], ck) < TIE_REL]
    if len(group) <= 1:
        return [base]
    fixed = [e for e in base if e not in group]
    need = k - len(fixed)
    cands = [base]
    if len(group) <= max_group:
        for combo in itertools.combinations(sorted(group), need):
            s = fixed + list(combo)
            if sorted(s) != sorted(base):
                cands.append(s)
    return cands


def check_parity(oracle_mod, cfg, host_inputs, gpu_out, gpu_idx, gpu_w, tokens=None, n_threads=None,
                 ref=None):
    """Compare GPU results (host numpy arrays over `tokens`, or all T) with the
    oracle.  `ref`: the oracle's result for those tokens if already computed
    (oracle_mod.forward with want_logits=True).  Returns a report dict; raises
    AssertionError on a violation."""
    o = ref if ref is not None else oracle_mod.forward(
        **host_inputs, k=cfg.k, score_fn=cfg.score_fn, norm_topk=cfg.norm_topk, route_scale=cfg.route_scale,
        tokens=tokens, want_logits=True, n_threads=n_threads)
    n, k = o["topk_idx"].shape
    gpu_idx = np.asarray(gpu_idx)
    gpu_w = np.asarray(gpu_w, np.float64)
    gpu_out = np.asarray(gpu_out, np.float64)
    assert gpu_idx.shape == (n, k) and gpu_w.shape == (n, k) and gpu_out.shape[0] == n
    ref_out = o["out"].copy()
    ref_w = o["topk_w"].copy()
    ref_idx = o["topk_idx"].copy()
    boundary_ties = 0
    order_swaps = 0
    alt_rows = {}
    for t in range(n):
        g = [int(e) for e in gpu_idx[t]]
        assert len(set(g)) == k, f"token {t}: repeated expert in {g}"
        keys = o["keys"][t]
        if sorted(g) != sorted(ref_idx[t].tolist()):
            cands = oracle_candidates(keys, o["sel_order"][t], k)
            match = [c for c in cands[1:] if sorted(c) == sorted(g)]
            assert match, (f"token {t}: GPU experts {sorted(g)} != oracle {sorted(ref_idx[t].tolist())} "
                           f"and not a near-tie alternative (k-th/k+1-th keys "
                           f"{o['sel_keys'][t][k - 1]!r} {o['sel_keys'][t][k]!r})")
            boundary_ties += 1
            alt_rows[t] = match[0]
        # order: GPU keys non-increasing up to near-ties
        gk = [keys[e] for e in g]
        for j in range(k - 1):
            if gk[j] < gk[j + 1]:
                assert rel_gap(gk[j], gk[j + 1]) < TIE_REL, f"token {t}: order {g} keys {gk}"
        if g != sorted(g, key=lambda e: (-keys[e], e)):
            order_swaps += 1
    if alt_rows:
        rows = sorted(alt_rows)
        forced = np.array([sorted(alt_rows[t], key=lambda e: (-o["keys"][t][e], e)) for t in rows],
                          np.int32)
        tok_ids = np.asarray(tokens if tokens is not None else np.arange(n))[rows]
        oa = oracle_mod.forward(**host_inputs, k=cfg.k, score_fn=cfg.score_fn, norm_topk=cfg.norm_topk,
                                route_scale=cfg.route_scale, tokens=tok_ids, forced_idx=forced,
                                n_threads=n_threads)
        for i, t in enumerate(rows):
            ref_out[t] = oa["out"][i]
            ref_w[t] = oa["topk_w"][i]
            ref_idx[t] = oa["topk_idx"][i]
    # weights, matched by expert id
    max_w_rel = 0.0
    for t in range(n):
        wmap = {int(e): ref_w[t, j] for j, e in enumerate(ref_idx[t])}
        for j, e in enumerate(gpu_idx[t]):
            ref = wmap[int(e)]
            err = abs(gpu_w[t, j] - ref)
            assert err <= W_RTOL * abs(ref) + W_ATOL, f"token {t} expert {e}: w {gpu_w[t, j]} vs {ref}"
            if ref != 0:
                max_w_rel = max(max_w_rel, err / abs(ref))
    scale = float(np.max(np.abs(ref_out))) if ref_out.size else 0.0
    err = float(np.max(np.abs(gpu_out - ref_out))) if ref_out.size else 0.0
    assert np.isfinite(gpu_out).all(), "non-finite GPU output"
    assert err <= OUT_TOL * scale, f"max|out-oracle| {err:.4g} > {OUT_TOL} * {scale:.4g}"
    return {"tokens": n, "boundary_ties": boundary_ties, "order_swaps": order_swaps,
            "max_abs_err": err, "max_abs_ref": scale, "err_ratio": err / scale if scale else 0.0,
            "max_w_rel": max_w_rel}


def check_routing(oracle_mod, cfg, host_inputs, gpu_idx, gpu_w, tokens=None, n_threads=None):
    """Routing only (steps a1-a2): compare topk_idx / topk_w of the GPU with the
    oracle's route_only pass over `tokens` (or all T), by the same index,
    near-tie and weight rules as check_parity.  Near-tie tokens are counted;
    for them the weights are compared with the oracle's weights for the GPU's
    experts (the oracle re-run with those experts forced).  Returns a report;
    raises AssertionError on a violation."""
    o = oracle_mod.forward(host_inputs["x"], host_inputs["W_router"], expert_bias=host_inputs.get("expert_bias"),
                           k=cfg.k, score_fn=cfg.score_fn, norm_topk=cfg.norm_topk, route_scale=cfg.route_scale,
                           tokens=tokens, route_only=True, want_logits=True, n_threads=n_threads)
    n, k = o["topk_idx"].shape
    gpu_idx = np.asarray(gpu_idx)
    gpu_w = np.asarray(gpu_w, np.float64)
    assert gpu_idx.shape == (n, k) and gpu_w.shape == (n, k)
    ref_idx = o["topk_idx"]
    # fast path: rows whose experts and order equal the oracle's exactly
    same = (gpu_idx == ref_idx).all(1)
    boundary_ties = 0
    order_swaps = 0
    alt_rows = {}
    for t in np.nonzero(~same)[0]:
        t = int(t)
        g = [int(e) for e in gpu_idx[t]]
        assert len(set(g)) == k, f"token {t}: repeated expert in {g}"
        assert all(0 <= e < cfg.E for e in g), f"token {t}: expert out of range in {g}"
        keys = o["keys"][t]
        if sorted(g) != sorted(ref_idx[t].tolist()):
            cands = oracle_candidates(keys, o["sel_order"][t], k)
            match = [c for c in cands[1:] if sorted(c) == sorted(g)]
            assert match, (f"token {t}: GPU experts {sorted(g)} != oracle {sorted(ref_idx[t].tolist())} "
                           f"and not a near-tie alternative (k-th/k+1-th keys "
                           f"{o['sel_keys'][t][k - 1]!r} {o['sel_keys'][t][k]!r})")
            boundary_ties += 1
            alt_rows[t] = match[0]
        gk = [keys[e] for e in g]
        for j in range(k - 1):
            if gk[j] < gk[j + 1]:
                assert rel_gap(gk[j], gk[j + 1]) < TIE_REL, f"token {t}: order {g} keys {gk}"
        if g != sorted(g, key=lambda e: (-keys[e], e)):
            order_swaps += 1
    ref_w = o["topk_w"].copy()
    ref_idx = ref_idx.copy()
    if alt_rows:
        rows = sorted(alt_rows)
        forced = np.array([sorted(alt_rows[t], key=lambda e: (-o["keys"][t][e], e)) for t in rows], np.int32)
        tok_ids = np.asarray(tokens if tokens is not None else np.arange(n))[rows]
        oa = oracle_mod.forward(host_inputs["x"], host_inputs["W_router"],
                                expert_bias=host_inputs.get("expert_bias"), k=cfg.k, score_fn=cfg.score_fn,
                                norm_topk=cfg.norm_topk, route_scale=cfg.route_scale, tokens=tok_ids,
                                forced_idx=forced, route_only=True, n_threads=n_threads)
        for i, t in enumerate(rows):
            ref_w[t] = oa["topk_w"][i]
            ref_idx[t] = oa["topk_idx"][i]
    # weights matched by expert id: sort both rows by expert
    go = np.argsort(gpu_idx, 1)
    ro = np.argsort(ref_idx, 1)
    gi = np.take_along_axis(gpu_idx, go, 1)
    ri = np.take_along_axis(ref_idx, ro, 1)
    assert np.array_equal(gi, ri)
    gw = np.take_along_axis(gpu_w, go, 1)
    rw = np.take_along_axis(ref_w, ro, 1)
    err = np.abs(gw - rw)
    bad = err > W_RTOL * np.abs(rw) + W_ATOL
    assert not bad.any(), f"{int(bad.sum())} weights off, first at {np.argwhere(bad)[0].tolist()}"
    with np.errstate(invalid="ignore", divide="ignore"):
        rel = np.where(rw != 0, err / np.abs(np.where(rw != 0, rw, 1.0)), 0.0)
    return {"tokens": n, "boundary_ties": boundary_ties, "order_swaps": order_swaps,
            "max_w_rel": float(rel.max()) if rel.size else 0.0}
