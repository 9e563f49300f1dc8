"""The C ABI on a machine without a GPU: the library loads, exports every
function include/moe.h declares, and its host-side logic (workspace sizing,
region layout, argument checks) behaves; nothing here launches a kernel."""
import ctypes
import os
import re

import pytest

from mixture_experts_ffn_16_b200 import api, build
from mixture_experts_ffn_16_b200.inputs import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return api.load()


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if fn.endswith(".h"):
            with open(os.path.join(inc, fn)) as fh:
                src = fh.read()
            names += re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", src)
    return names


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert len(names) >= 13
    assert sorted(names) == sorted(api.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.moe_version() >= 100
    for code in (0, -1, -2, -3, -4, -5):
        assert lib.moe_status_string(code)
    assert b"unknown" in lib.moe_status_string(42)


@pytest.mark.parametrize("name", list(CONFIGS))
def test_workspace_sizes_of_workloads(lib, name):
    c = CONFIGS[name]
    s = api.shape_of(c)
    n = api.moe_workspace_bytes(s)
    assert n > 0
    # must at least hold the routed hidden and output rows (T*k of each) and the logits
    assert n >= c.T * c.k * (c.f + c.d) * 2 + c.T * c.E * 4
    # regions are disjoint, 256-byte aligned and inside the workspace
    spans = []
    for r in api.WS_REGIONS:
        off, nb = api.moe_workspace_region(s, r)
        assert off % 256 == 0 and off + nb <= n
        spans.append((off, off + nb))
    spans.sort()
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0 or a0 == a1 or b0 == b1


@pytest.mark.parametrize("bad,code", [
    (dict(T=0), api.MOE_ERR_INVALID_ARG), (dict(k=0), api.MOE_ERR_INVALID_ARG),
    (dict(k=9, E=8), api.MOE_ERR_INVALID_ARG), (dict(E=0), api.MOE_ERR_INVALID_ARG),
    (dict(d_model=100), api.MOE_ERR_UNSUPPORTED), (dict(d_ff=96), api.MOE_ERR_UNSUPPORTED),
    (dict(n_shared=1, d_ff_shared=80), api.MOE_ERR_UNSUPPORTED), (dict(E=4096), api.MOE_ERR_UNSUPPORTED),
    (dict(k=33, E=64), api.MOE_ERR_UNSUPPORTED), (dict(n_shared=9, d_ff_shared=64), api.MOE_ERR_UNSUPPORTED),
    (dict(T=(1 << 22) + 1), api.MOE_ERR_UNSUPPORTED), (dict(d_model=65536 + 64), api.MOE_ERR_UNSUPPORTED),
    (dict(d_ff=65536 + 64), api.MOE_ERR_UNSUPPORTED), (dict(d_ff_shared=65536 + 64), api.MOE_ERR_UNSUPPORTED),
    (dict(n_shared=-1), api.MOE_ERR_INVALID_ARG), (dict(n_shared=1, d_ff_shared=0), api.MOE_ERR_INVALID_ARG),
])
def test_invalid_shapes(lib, bad, code):
    base = dict(T=16, d_model=128, E=8, k=2, d_ff=128, n_shared=1, d_ff_shared=128)
    base.update(bad)
    s = api.make_shape(**base)
    assert api.moe_workspace_bytes(s) == 0
    st = lib.moe_forward(ctypes.byref(s), *([ctypes.c_void_p(256)] * 9), None, 0, 1, 1.0,
                         *([ctypes.c_void_p(256)] * 4), 1 << 30, None)
    assert st == code


def test_largest_supported_shape_plans(lib):
    """The limits themselves are accepted: T = 2^22, d = f = fs = 65536."""
    s = api.make_shape(1 << 22, 65536, 8, 2, 65536, 1, 65536)
    assert api.moe_workspace_bytes(s) > 0


def test_argument_checks_before_any_device_work(lib):
    s = api.make_shape(16, 128, 8, 2, 128, 1, 128)
    n = api.moe_workspace_bytes(s)
    P = ctypes.c_void_p
    good = [P(4096)] * 9
    # null x
    st = lib.moe_forward(ctypes.byref(s), None, *good[1:], None, 0, 1, 1.0, P(4096), P(4096), P(4096), P(4096),
                         n, None)
    assert st == api.MOE_ERR_INVALID_ARG
    # bad score function / norm flag / non-finite scale
    for sf, nt, sc in [(3, 1, 1.0), (0, 2, 1.0), (0, 1, float("inf"))]:
        st = lib.moe_forward(ctypes.byref(s), *good, None, sf, nt, sc, P(4096), P(4096), P(4096), P(4096), n, None)
        assert st == api.MOE_ERR_INVALID_ARG
    # misaligned pointer
    st = lib.moe_forward(ctypes.byref(s), P(4098), *good[1:], None, 0, 1, 1.0, P(4096), P(4096), P(4096), P(4096),
                         n, None)
    assert st == api.MOE_ERR_UNSUPPORTED
    # shared weights given with S == 0
    s0 = api.make_shape(16, 128, 8, 2, 128, 0, 0)
    st = lib.moe_forward(ctypes.byref(s0), *good, None, 0, 1, 1.0, P(4096), P(4096), P(4096), P(4096),
                         api.moe_workspace_bytes(s0), None)
    assert st == api.MOE_ERR_INVALID_ARG
    # shared-expert gate vector given with S == 0, or misaligned
    st = lib.moe_forward(ctypes.byref(s0), *good[:6], None, None, None, P(4096), 0, 1, 1.0,
                         P(4096), P(4096), P(4096), P(4096), api.moe_workspace_bytes(s0), None)
    assert st == api.MOE_ERR_INVALID_ARG
    st = lib.moe_forward(ctypes.byref(s), *good, P(4100), 0, 1, 1.0, P(4096), P(4096), P(4096), P(4096),
                         n, None)
    assert st == api.MOE_ERR_UNSUPPORTED
    # workspace too small / misaligned
    st = lib.moe_forward(ctypes.byref(s), *good, None, 0, 1, 1.0, P(4096), P(4096), P(4096), P(4096), n - 1, None)
    assert st == api.MOE_ERR_WORKSPACE
    st = lib.moe_forward(ctypes.byref(s), *good, None, 0, 1, 1.0, P(4096), P(4096), P(4096), P(4128), n, None)
    assert st == api.MOE_ERR_WORKSPACE


def test_region_query_rejects_bad_region(lib):
    s = api.make_shape(16, 128, 8, 2, 128, 1, 128)
    off, nb = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.moe_workspace_region(ctypes.byref(s), 99, ctypes.byref(off), ctypes.byref(nb)) == api.MOE_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(api, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        api.load()


def test_experts_forward_argument_checks(lib):
    """External-indices entry: null or misaligned routing arrays and a gate
    vector with no shared expert are refused before any device work."""
    s = api.make_shape(16, 128, 8, 2, 128, 1, 128)
    n = api.moe_workspace_bytes(s)
    P = ctypes.c_void_p
    w6 = [P(4096)] * 6

    def call(shape=s, x=P(4096), idx=P(4096), wt=P(4096), gv=None, out=P(4096), ws_bytes=n, weights=w6):
        return lib.moe_experts_forward(ctypes.byref(shape), x, idx, wt, *weights, gv, out, P(4096), ws_bytes, None)

    assert call(idx=None) == api.MOE_ERR_INVALID_ARG
    assert call(wt=None) == api.MOE_ERR_INVALID_ARG
    assert call(out=None) == api.MOE_ERR_INVALID_ARG
    assert call(idx=P(4100)) == api.MOE_ERR_UNSUPPORTED
    assert call(gv=P(4104)) == api.MOE_ERR_UNSUPPORTED
    assert call(weights=w6[:3] + [None] * 3) == api.MOE_ERR_INVALID_ARG
    s0 = api.make_shape(16, 128, 8, 2, 128, 0, 0)
    assert call(shape=s0, weights=w6[:3] + [None] * 3, gv=P(4096),
                ws_bytes=api.moe_workspace_bytes(s0)) == api.MOE_ERR_INVALID_ARG
    assert call(ws_bytes=n - 1) == api.MOE_ERR_WORKSPACE


def test_prenorm_and_rmsnorm_argument_checks(lib):
    s = api.make_shape(16, 128, 8, 2, 128, 1, 128)
    n = api.moe_workspace_bytes(s)
    P = ctypes.c_void_p
    good = [P(4096)] * 9

    def fwd(gain=P(4096), eps=1e-6, x=P(4096)):
        return lib.moe_forward_prenorm(ctypes.byref(s), x, gain, eps, *good[1:], None, 0, 1, 1.0,
                                       P(4096), P(4096), P(4096), P(4096), n, None)

    assert fwd(gain=None) == api.MOE_ERR_INVALID_ARG
    assert fwd(eps=-1.0) == api.MOE_ERR_INVALID_ARG
    assert fwd(eps=float("nan")) == api.MOE_ERR_INVALID_ARG
    assert fwd(eps=float("inf")) == api.MOE_ERR_INVALID_ARG
    assert fwd(x=None) == api.MOE_ERR_INVALID_ARG
    assert fwd(gain=P(4098)) == api.MOE_ERR_UNSUPPORTED
    assert lib.moe_rmsnorm(ctypes.byref(s), P(4096), None, 1e-6, P(4096), None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm(ctypes.byref(s), P(4096), P(4096), -1.0, P(4096), None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm(ctypes.byref(s), P(4096), P(4096), 1e-6, P(4100), None) == api.MOE_ERR_UNSUPPORTED
    bad = api.make_shape(16, 100, 8, 2, 128, 1, 128)
    assert lib.moe_rmsnorm(ctypes.byref(bad), P(4096), P(4096), 1e-6, P(4096), None) == api.MOE_ERR_UNSUPPORTED


def test_x_stage_region(lib):
    s = api.make_shape(16, 128, 8, 2, 128, 1, 128)
    off, nb = api.moe_workspace_region(s, "x_stage")
    assert nb == 16 * 128 * 2 and off % 256 == 0 and off + nb <= api.moe_workspace_bytes(s)


def test_fp8_argument_checks(lib):
    """FP8 entry points refuse null or half-given weights and misalignment before any device work."""
    s = api.make_shape(16, 128, 8, 2, 128, 1, 128)
    n = api.moe_workspace_bytes(s)
    P = ctypes.c_void_p
    W = api.MoeFp8Weight
    good = W(P(4096), P(8192))

    def fwd(ws6=None, shape=s, nb=n):
        ws6 = ws6 if ws6 is not None else [good] * 6
        ptrs = [None if w is None else ctypes.pointer(w) for w in ws6]
        return lib.moe_forward_fp8(ctypes.byref(shape), P(4096), P(4096), None, *ptrs, None, 0, 1, 1.0,
                                   P(4096), P(4096), P(4096), P(4096), nb, None)

    assert fwd([None] + [good] * 5) == api.MOE_ERR_INVALID_ARG
    assert fwd([W(P(4096), None)] + [good] * 5) == api.MOE_ERR_INVALID_ARG      # codes without scales
    assert fwd([good] * 3 + [None] * 3) == api.MOE_ERR_INVALID_ARG              # S = 1 needs shared weights
    assert fwd([W(P(4100), P(8192))] + [good] * 5) == api.MOE_ERR_UNSUPPORTED
    assert fwd([good] * 2 + [W(P(4096), P(8200))] + [good] * 3) == api.MOE_ERR_UNSUPPORTED
    s0 = api.make_shape(16, 128, 8, 2, 128, 0, 0)
    assert fwd([good] * 6, shape=s0, nb=api.moe_workspace_bytes(s0)) == api.MOE_ERR_INVALID_ARG
    assert fwd(nb=n - 1) == api.MOE_ERR_WORKSPACE
    pg = ctypes.pointer(good)
    assert lib.moe_expert_gate_up_fp8(ctypes.byref(s), P(4096), pg, None, pg, pg, P(4096), n, None) == \
        api.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_down_fp8(ctypes.byref(s), pg, None, P(4096), n, None) == api.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("name", list(CONFIGS))
def test_router_logit_slices(lib, name):
    """The logits region holds P whole [T, E] fp32 arrays, one per K slice of
    the router GEMM: at least one, at most 16, never more than d / 64."""
    c = CONFIGS[name]
    s = api.shape_of(c)
    _, nb = api.moe_workspace_region(s, "logits")
    one = c.T * c.E * 4
    assert nb % one == 0
    slices = nb // one
    assert 1 <= slices <= min(16, c.d // 64)


# The router tiling each workload gets (K slices of d): small batches split d
# to fill the SMs (tiny, decode); prefill_softmax reads fewer W_router bytes
# per SM with two slices of single-CTA units; prefill_sigmoid and
# large_imbalanced run on CTA pairs of 256 experts x 256 tokens, the latter in
# two slices to spread its 256 pair-units over the pairs evenly.
ROUTER_SLICES = {"tiny": 4, "prefill_softmax": 2, "prefill_sigmoid": 1, "decode_sqrt_softplus": 8,
                 "large_imbalanced": 2}


@pytest.mark.parametrize("name", list(ROUTER_SLICES))
def test_router_plan_of_each_workload(lib, name):
    c = CONFIGS[name]
    _, nb = api.moe_workspace_region(api.shape_of(c), "logits")
    assert nb // (c.T * c.E * 4) == ROUTER_SLICES[name]


def test_work_list_regions_hold_the_largest_lists():
    """The work-list regions hold the most units any routing can produce:
    every routed row in its own run plus one partial run per expert, per
    weight block, plus the shared experts' runs."""
    c = CONFIGS["large_imbalanced"]
    s = api.shape_of(c)
    assert api.moe_workspace_region(s, "work_counts")[1] == 16
    rows_cap = c.T * c.k + c.E * 31
    for name, nwb, nwbs in (("work_gate_up", c.f // 128, c.fs // 128), ("work_down", c.d // 256, c.d // 256)):
        _, nb = api.moe_workspace_region(s, name)
        assert nb % 16 == 0
        assert nb // 16 >= nwb * (rows_cap // 128) + c.S * nwbs * (c.T // 128)


def test_binding_marshalling_checks():
    """The Python binding checks device, dtype, shape and layout before it
    hands a pointer to the library."""
    import torch
    bf = torch.bfloat16
    t = torch.zeros(4, 8, dtype=bf)
    assert api._p(None) is None
    assert api._p(256).value == 256
    with pytest.raises(TypeError):
        api._p([1, 2], bf, (4, 8), "x")
    with pytest.raises(ValueError, match="CUDA"):
        api._p(t, bf, (4, 8), "x")                      # a host tensor where device memory is expected
    assert api._p(t, bf, (4, 8), "x", host=True).value == t.data_ptr()
    with pytest.raises(TypeError, match="bfloat16"):
        api._p(t.float(), bf, (4, 8), "x", host=True)
    with pytest.raises(ValueError, match="shape"):
        api._p(t, bf, (8, 4), "x", host=True)
    with pytest.raises(ValueError, match="contiguous"):
        api._p(t.t(), bf, (8, 4), "x", host=True)
    s = api.make_shape(4, 8, 2, 1, 64, 0, 0)
    with pytest.raises(ValueError, match="CUDA"):
        api.moe_forward(s, t, torch.zeros(2, 8, dtype=bf), None, None, None, None, None, None, None,
                        "softmax", True, 1.0, torch.zeros(4, 8, dtype=bf), torch.zeros(4, 1, dtype=torch.int32),
                        torch.zeros(4, 1), None, stream=0)
