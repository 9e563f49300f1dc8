"""ctypes binding of libmoe.so (C ABI in include/moe.h).

Argument marshalling only: each function checks the tensors it is given
(device, dtype, shape, contiguity), passes their device pointers and the
current CUDA stream to the function of the same name in libmoe.so, and raises
MoEError on a non-zero status.  Every step of the block runs in the library's
CUDA kernels; there is no CPU path, and a missing library raises at load time.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE_TIMEOUT = -5
MOE_ERR_SCRATCH_LIMIT = -6
MOE_ERR_NONFINITE = -7

SCORE_FNS = {"softmax": 0, "sigmoid": 1, "sqrt_softplus": 2}

WS_REGIONS = {"logits": 0, "counts": 1, "offsets": 2, "perm": 3, "row_w": 4, "inv": 5,
              "h": 6, "h_shared": 7, "y": 8, "y_shared": 9, "x_stage": 10,
              "work_counts": 11, "work_gate_up": 12, "work_down": 13}

EXPORTED = ["moe_version", "moe_status_string", "moe_workspace_bytes", "moe_forward",
            "moe_forward_host", "moe_route", "moe_permute", "moe_expert_gate_up", "moe_expert_down",
            "moe_combine", "moe_workspace_region", "moe_device_status", "moe_debug_wait_timeout",
            "moe_route_noalloc", "moe_experts_forward", "moe_rmsnorm", "moe_forward_prenorm",
            "moe_forward_fp8", "moe_expert_gate_up_fp8", "moe_expert_down_fp8", "moe_permute_fp8"]


class MoEError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("d_ff_shared", ctypes.c_int32)]


class MoeFp8Weight(ctypes.Structure):
    """moe_fp8_weight: E4M3 codes [G, rows, K] and UE8M0 block scales [G, K/32, rows]."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_lib = None


def load():
    """Load libmoe.so (raises if it has not been built: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libmoe.so not found at {LIB_PATH}: build it with "
                           "`python -m mixture_experts_ffn_16_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    SH = ctypes.POINTER(MoeShape)
    lib.moe_version.restype = I
    lib.moe_version.argtypes = []
    lib.moe_status_string.restype = ctypes.c_char_p
    lib.moe_status_string.argtypes = [I]
    lib.moe_workspace_bytes.restype = SZ
    lib.moe_workspace_bytes.argtypes = [SH]
    fwd = [SH, P, P, P, P, P, P, P, P, P, P, I, I, ctypes.c_float, P, P, P, P, SZ, P]
    lib.moe_forward.restype = I
    lib.moe_forward.argtypes = fwd
    lib.moe_forward_host.restype = I
    lib.moe_forward_host.argtypes = fwd
    lib.moe_forward_prenorm.restype = I
    lib.moe_forward_prenorm.argtypes = [SH, P, P, ctypes.c_float] + fwd[2:]
    F8 = ctypes.POINTER(MoeFp8Weight)
    lib.moe_forward_fp8.restype = I
    lib.moe_forward_fp8.argtypes = [SH, P, P, P, F8, F8, F8, F8, F8, F8] + fwd[10:]
    lib.moe_permute_fp8.restype = I
    lib.moe_permute_fp8.argtypes = [SH, P, P, P, SZ, P]
    lib.moe_expert_gate_up_fp8.restype = I
    lib.moe_expert_gate_up_fp8.argtypes = [SH, P, F8, F8, F8, F8, P, SZ, P]
    lib.moe_expert_down_fp8.restype = I
    lib.moe_expert_down_fp8.argtypes = [SH, F8, F8, P, SZ, P]
    lib.moe_rmsnorm.restype = I
    lib.moe_rmsnorm.argtypes = [SH, P, P, ctypes.c_float, P, P]
    lib.moe_route.restype = I
    lib.moe_route.argtypes = [SH, P, P, P, I, I, ctypes.c_float, P, P, P, SZ, P]
    lib.moe_permute.restype = I
    lib.moe_permute.argtypes = [SH, P, P, P, SZ, P]
    lib.moe_expert_gate_up.restype = I
    lib.moe_expert_gate_up.argtypes = [SH, P, P, P, P, P, P, SZ, P]
    lib.moe_expert_down.restype = I
    lib.moe_expert_down.argtypes = [SH, P, P, P, SZ, P]
    lib.moe_combine.restype = I
    lib.moe_combine.argtypes = [SH, P, P, P, P, SZ, P]
    lib.moe_experts_forward.restype = I
    lib.moe_experts_forward.argtypes = [SH, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    lib.moe_workspace_region.restype = I
    lib.moe_workspace_region.argtypes = [SH, I, ctypes.POINTER(SZ), ctypes.POINTER(SZ)]
    lib.moe_device_status.restype = I
    lib.moe_device_status.argtypes = [P, P]
    lib.moe_debug_wait_timeout.restype = I
    lib.moe_debug_wait_timeout.argtypes = [P, SZ, ctypes.c_uint64, P]
    lib.moe_route_noalloc.restype = I
    lib.moe_route_noalloc.argtypes = [SH, P, P, P, I, I, ctypes.c_float, P, P, P]
    _lib = lib
    return lib


def status_string(status):
    try:
        return load().moe_status_string(int(status)).decode()
    except Exception:  # noqa: BLE001 - message formatting only
        return "status"


def make_shape(T, d_model, E, k, d_ff, n_shared=0, d_ff_shared=0):
    return MoeShape(int(T), int(d_model), int(E), int(k), int(d_ff), int(n_shared), int(d_ff_shared))


def shape_of(cfg):
    """moe_shape of a MoEConfig (inputs.MoEConfig)."""
    return make_shape(cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.S, cfg.fs)


def moe_workspace_bytes(shape) -> int:
    return int(load().moe_workspace_bytes(ctypes.byref(shape)))


def moe_workspace_region(shape, region):
    """(offset, bytes) of a named workspace region (see WS_REGIONS)."""
    off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    r = WS_REGIONS[region] if isinstance(region, str) else int(region)
    st = load().moe_workspace_region(ctypes.byref(shape), r, ctypes.byref(off), ctypes.byref(nb))
    if st != MOE_OK:
        raise MoEError(st, "moe_workspace_region")
    return off.value, nb.value


def alloc_workspace(shape, device=None):
    """A device byte tensor large enough for `shape` (256-byte aligned by torch's allocator)."""
    n = moe_workspace_bytes(shape)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    assert ws.data_ptr() % 256 == 0
    return ws


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _p(t, dtype=None, shape=None, name="", host=False):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if host != (t.device.type == "cpu"):
        raise ValueError(f"{name}: expected a {'host' if host else 'CUDA'} tensor, got {t.device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _check(st, where):
    if st != MOE_OK:
        raise MoEError(st, where)


def _score(score_fn):
    return SCORE_FNS[score_fn] if isinstance(score_fn, str) else int(score_fn)


def _weights(shape, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down):
    E, f, d, S, fs = shape.E, shape.d_ff, shape.d_model, shape.n_shared, shape.d_ff_shared
    bf = torch.bfloat16
    return [_p(W_gate, bf, (E, f, d), "W_gate"), _p(W_up, bf, (E, f, d), "W_up"),
            _p(W_down, bf, (E, d, f), "W_down"),
            _p(W_shared_gate, bf, (S, fs, d), "W_shared_gate") if S else None,
            _p(W_shared_up, bf, (S, fs, d), "W_shared_up") if S else None,
            _p(W_shared_down, bf, (S, d, fs), "W_shared_down") if S else None]


def _f8(w, G, rows, K, name):
    """(codes, scales) tensors -> a MoeFp8Weight (None when w is None)."""
    if w is None:
        return None
    codes, scales = w
    return MoeFp8Weight(_p(codes, torch.uint8, (G, rows, K), name + ".codes"),
                        _p(scales, torch.uint8, (G, K // 32, rows), name + ".scales"))


def _f8_weights(shape, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down):
    E, f, d, S, fs = shape.E, shape.d_ff, shape.d_model, shape.n_shared, shape.d_ff_shared
    ws = [_f8(W_gate, E, f, d, "W_gate"), _f8(W_up, E, f, d, "W_up"), _f8(W_down, E, d, f, "W_down"),
          _f8(W_shared_gate, S, fs, d, "W_shared_gate") if S else None,
          _f8(W_shared_up, S, fs, d, "W_shared_up") if S else None,
          _f8(W_shared_down, S, d, fs, "W_shared_down") if S else None]
    return [None if w is None else ctypes.pointer(w) for w in ws]


def _gate_vec(shape, W_shared_gate_vec):
    if W_shared_gate_vec is None:
        return None
    return _p(W_shared_gate_vec, torch.bfloat16, (shape.n_shared, shape.d_model), "W_shared_gate_vec")


def moe_forward(shape, x, W_router, expert_bias, W_gate, W_up, W_down, W_shared_gate, W_shared_up,
                W_shared_down, score_fn, norm_topk, route_scale, out, topk_idx, topk_w, workspace,
                stream=None, W_shared_gate_vec=None):
    T, d, E, k = shape.T, shape.d_model, shape.E, shape.k
    bf = torch.bfloat16
    st = load().moe_forward(
        ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(W_router, bf, (E, d), "W_router"),
        _p(expert_bias, torch.float32, (E,), "expert_bias"),
        *_weights(shape, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down),
        _gate_vec(shape, W_shared_gate_vec), _score(score_fn), int(bool(norm_topk)), float(route_scale),
        _p(out, bf, (T, d), "out"), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
        _p(topk_w, torch.float32, (T, k), "topk_w"),
        _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_forward")


def moe_forward_prenorm(shape, x, norm_gain, norm_eps, W_router, expert_bias, W_gate, W_up, W_down,
                        W_shared_gate, W_shared_up, W_shared_down, score_fn, norm_topk, route_scale, out,
                        topk_idx, topk_w, workspace, stream=None, W_shared_gate_vec=None):
    """moe_forward behind the pre-norm RMSNorm (zero-centred gains): x is the raw
    residual stream; the normalised rows are left in the workspace region "x_stage"."""
    T, d, E, k = shape.T, shape.d_model, shape.E, shape.k
    bf = torch.bfloat16
    st = load().moe_forward_prenorm(
        ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(norm_gain, bf, (d,), "norm_gain"), float(norm_eps),
        _p(W_router, bf, (E, d), "W_router"), _p(expert_bias, torch.float32, (E,), "expert_bias"),
        *_weights(shape, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down),
        _gate_vec(shape, W_shared_gate_vec), _score(score_fn), int(bool(norm_topk)), float(route_scale),
        _p(out, bf, (T, d), "out"), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
        _p(topk_w, torch.float32, (T, k), "topk_w"),
        _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_forward_prenorm")


def moe_forward_fp8(shape, x, W_router, expert_bias, W_gate, W_up, W_down, W_shared_gate, W_shared_up,
                    W_shared_down, score_fn, norm_topk, route_scale, out, topk_idx, topk_w, workspace,
                    stream=None, W_shared_gate_vec=None):
    """moe_forward with block-scaled FP8 expert weights: each W_* is a
    (codes uint8 [G, rows, K], scales uint8 [G, K/32, rows]) pair, or None for
    the shared ones when n_shared == 0."""
    T, d, E, k = shape.T, shape.d_model, shape.E, shape.k
    bf = torch.bfloat16
    st = load().moe_forward_fp8(
        ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(W_router, bf, (E, d), "W_router"),
        _p(expert_bias, torch.float32, (E,), "expert_bias"),
        *_f8_weights(shape, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down),
        _gate_vec(shape, W_shared_gate_vec), _score(score_fn), int(bool(norm_topk)), float(route_scale),
        _p(out, bf, (T, d), "out"), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
        _p(topk_w, torch.float32, (T, k), "topk_w"),
        _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_forward_fp8")


def moe_permute_fp8(shape, topk_idx, topk_w, workspace, stream=None):
    """The permute for the FP8 expert steps (their work lists differ from the bf16 ones)."""
    T, k = shape.T, shape.k
    st = load().moe_permute_fp8(ctypes.byref(shape), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
                                _p(topk_w, torch.float32, (T, k), "topk_w"),
                                _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_permute_fp8")


def moe_expert_gate_up_fp8(shape, x, W_gate, W_up, W_shared_gate, W_shared_up, workspace, stream=None):
    w = _f8_weights(shape, W_gate, W_up, None, W_shared_gate, W_shared_up, None)
    st = load().moe_expert_gate_up_fp8(ctypes.byref(shape), _p(x, torch.bfloat16, (shape.T, shape.d_model), "x"),
                                       w[0], w[1], w[3], w[4], _p(workspace, torch.uint8, None, "workspace"),
                                       workspace.numel(), _stream(stream))
    _check(st, "moe_expert_gate_up_fp8")


def moe_expert_down_fp8(shape, W_down, W_shared_down, workspace, stream=None):
    w = _f8_weights(shape, None, None, W_down, None, None, W_shared_down)
    st = load().moe_expert_down_fp8(ctypes.byref(shape), w[2], w[5], _p(workspace, torch.uint8, None, "workspace"),
                                    workspace.numel(), _stream(stream))
    _check(st, "moe_expert_down_fp8")


def moe_rmsnorm(shape, x, norm_gain, eps, x_norm, stream=None):
    """x_norm = bf16(x / sqrt(mean(x^2) + eps) * (1 + norm_gain)), computed in double."""
    T, d = shape.T, shape.d_model
    bf = torch.bfloat16
    st = load().moe_rmsnorm(ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(norm_gain, bf, (d,), "norm_gain"),
                            float(eps), _p(x_norm, bf, (T, d), "x_norm"), _stream(stream))
    _check(st, "moe_rmsnorm")


def moe_forward_host(shape, x_host, W_router, expert_bias, W_gate, W_up, W_down, W_shared_gate,
                     W_shared_up, W_shared_down, score_fn, norm_topk, route_scale, out_host,
                     topk_idx_host, topk_w_host, workspace, stream=None, W_shared_gate_vec=None):
    T, d, E, k = shape.T, shape.d_model, shape.E, shape.k
    bf = torch.bfloat16
    st = load().moe_forward_host(
        ctypes.byref(shape), _p(x_host, bf, (T, d), "x_host", host=True),
        _p(W_router, bf, (E, d), "W_router"), _p(expert_bias, torch.float32, (E,), "expert_bias"),
        *_weights(shape, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down),
        _gate_vec(shape, W_shared_gate_vec), _score(score_fn), int(bool(norm_topk)), float(route_scale),
        _p(out_host, bf, (T, d), "out_host", host=True),
        _p(topk_idx_host, torch.int32, (T, k), "topk_idx_host", host=True),
        _p(topk_w_host, torch.float32, (T, k), "topk_w_host", host=True),
        _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_forward_host")


def moe_route(shape, x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w,
              workspace, stream=None):
    T, d, E, k = shape.T, shape.d_model, shape.E, shape.k
    bf = torch.bfloat16
    st = load().moe_route(
        ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(W_router, bf, (E, d), "W_router"),
        _p(expert_bias, torch.float32, (E,), "expert_bias"), _score(score_fn), int(bool(norm_topk)),
        float(route_scale), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
        _p(topk_w, torch.float32, (T, k), "topk_w"), _p(workspace, torch.uint8, None, "workspace"),
        workspace.numel(), _stream(stream))
    _check(st, "moe_route")


def moe_route_noalloc(shape, x, W_router, expert_bias, score_fn, norm_topk, route_scale, topk_idx, topk_w,
                      stream=None):
    """moe_route without a workspace, for callers that cannot allocate device
    memory (the library's built-in 16 MiB scratch holds the logits; T * E must
    not exceed 4,194,304).  Calls that overlap on the GPU race."""
    T, d, E, k = shape.T, shape.d_model, shape.E, shape.k
    bf = torch.bfloat16
    st = load().moe_route_noalloc(
        ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(W_router, bf, (E, d), "W_router"),
        _p(expert_bias, torch.float32, (E,), "expert_bias"), _score(score_fn), int(bool(norm_topk)),
        float(route_scale), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
        _p(topk_w, torch.float32, (T, k), "topk_w"), _stream(stream))
    _check(st, "moe_route_noalloc")


def moe_permute(shape, topk_idx, topk_w, workspace, stream=None):
    T, k = shape.T, shape.k
    st = load().moe_permute(ctypes.byref(shape), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
                            _p(topk_w, torch.float32, (T, k), "topk_w"),
                            _p(workspace, torch.uint8, None, "workspace"), workspace.numel(),
                            _stream(stream))
    _check(st, "moe_permute")


def moe_expert_gate_up(shape, x, W_gate, W_up, W_shared_gate, W_shared_up, workspace, stream=None):
    T, d, E, f, S, fs = shape.T, shape.d_model, shape.E, shape.d_ff, shape.n_shared, shape.d_ff_shared
    bf = torch.bfloat16
    st = load().moe_expert_gate_up(
        ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(W_gate, bf, (E, f, d), "W_gate"),
        _p(W_up, bf, (E, f, d), "W_up"),
        _p(W_shared_gate, bf, (S, fs, d), "W_shared_gate") if S else None,
        _p(W_shared_up, bf, (S, fs, d), "W_shared_up") if S else None,
        _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_expert_gate_up")


def moe_expert_down(shape, W_down, W_shared_down, workspace, stream=None):
    d, E, f, S, fs = shape.d_model, shape.E, shape.d_ff, shape.n_shared, shape.d_ff_shared
    bf = torch.bfloat16
    st = load().moe_expert_down(
        ctypes.byref(shape), _p(W_down, bf, (E, d, f), "W_down"),
        _p(W_shared_down, bf, (S, d, fs), "W_shared_down") if S else None,
        _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_expert_down")


def moe_combine(shape, out, workspace, stream=None, x=None, W_shared_gate_vec=None):
    T, d = shape.T, shape.d_model
    st = load().moe_combine(ctypes.byref(shape), _p(x, torch.bfloat16, (T, d), "x"),
                            _gate_vec(shape, W_shared_gate_vec), _p(out, torch.bfloat16, (T, d), "out"),
                            _p(workspace, torch.uint8, None, "workspace"), workspace.numel(),
                            _stream(stream))
    _check(st, "moe_combine")


def moe_experts_forward(shape, x, topk_idx, topk_w, W_gate, W_up, W_down, W_shared_gate, W_shared_up,
                        W_shared_down, out, workspace, stream=None, W_shared_gate_vec=None):
    """Steps a3..a7 on a caller-supplied routing (external-indices mode)."""
    T, d, k = shape.T, shape.d_model, shape.k
    bf = torch.bfloat16
    st = load().moe_experts_forward(
        ctypes.byref(shape), _p(x, bf, (T, d), "x"), _p(topk_idx, torch.int32, (T, k), "topk_idx"),
        _p(topk_w, torch.float32, (T, k), "topk_w"),
        *_weights(shape, W_gate, W_up, W_down, W_shared_gate, W_shared_up, W_shared_down),
        _gate_vec(shape, W_shared_gate_vec), _p(out, bf, (T, d), "out"),
        _p(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream))
    _check(st, "moe_experts_forward")


def moe_device_status(workspace, stream=None) -> int:
    """Synchronises the stream and returns the workspace's device status code."""
    return int(load().moe_device_status(_p(workspace, torch.uint8, None, "workspace"), _stream(stream)))


def moe_debug_wait_timeout(workspace, timeout_ns, stream=None):
    st = load().moe_debug_wait_timeout(_p(workspace, torch.uint8, None, "workspace"), workspace.numel(),
                                       int(timeout_ns), _stream(stream))
    _check(st, "moe_debug_wait_timeout")


def workspace_view(workspace, shape, region, dtype, dims):
    """A typed view of one workspace region (tests and debugging)."""
    off, nbytes = moe_workspace_region(shape, region)
    itemsize = torch.empty((), dtype=dtype).element_size()
    n = 1
    for x in dims:
        n *= int(x)
    assert n * itemsize <= nbytes, (region, dims, nbytes)
    return workspace[off:off + n * itemsize].view(dtype).view(*dims)


class MoELayer:
    """Convenience holder: weights + workspace for one shape; __call__ runs moe_forward."""

    def __init__(self, cfg, tensors, device="cuda"):
        self.cfg = cfg
        self.shape = shape_of(cfg)
        self.t = tensors
        self.workspace = alloc_workspace(self.shape, device)
        T, d, k = cfg.T, cfg.d, cfg.k
        self.out = torch.empty((T, d), dtype=torch.bfloat16, device=device)
        self.topk_idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.topk_w = torch.empty((T, k), dtype=torch.float32, device=device)
        if cfg.fp8 and cfg.prenorm:
            raise ValueError("MoELayer: the FP8 and pre-norm forms are separate entry points")

    def __call__(self, x=None, stream=None):
        t, c = self.t, self.cfg
        if c.fp8:
            moe_forward_fp8(self.shape, t["x"] if x is None else x, t["W_router"], t["expert_bias"],
                            t["W_gate_f8"], t["W_up_f8"], t["W_down_f8"], t["W_shared_gate_f8"],
                            t["W_shared_up_f8"], t["W_shared_down_f8"], c.score_fn, c.norm_topk, c.route_scale,
                            self.out, self.topk_idx, self.topk_w, self.workspace, stream,
                            W_shared_gate_vec=t.get("W_shared_gate_vec"))
            return self.out, self.topk_idx, self.topk_w
        if c.prenorm:
            moe_forward_prenorm(self.shape, t["x"] if x is None else x, t["norm_gain"], c.norm_eps, t["W_router"],
                                t["expert_bias"], t["W_gate"], t["W_up"], t["W_down"], t["W_shared_gate"],
                                t["W_shared_up"], t["W_shared_down"], c.score_fn, c.norm_topk, c.route_scale,
                                self.out, self.topk_idx, self.topk_w, self.workspace, stream,
                                W_shared_gate_vec=t.get("W_shared_gate_vec"))
            return self.out, self.topk_idx, self.topk_w
        moe_forward(self.shape, t["x"] if x is None else x, t["W_router"], t["expert_bias"],
                    t["W_gate"], t["W_up"], t["W_down"], t["W_shared_gate"], t["W_shared_up"],
                    t["W_shared_down"], c.score_fn, c.norm_topk, c.route_scale, self.out,
                    self.topk_idx, self.topk_w, self.workspace, stream,
                    W_shared_gate_vec=t.get("W_shared_gate_vec"))
        return self.out, self.topk_idx, self.topk_w

    def steps(self, stream=None, events=None):
        """The same pass as __call__, one step at a time; when `events` (6 CUDA
        events) is given, records them around the steps on `stream`."""
        t, c, s = self.t, self.cfg, self.shape
        st = stream
        rec = (lambda i: events[i].record(st)) if events is not None else (lambda i: None)
        rec(0)
        x = t["x"]
        if c.prenorm:
            x = workspace_view(self.workspace, s, "x_stage", torch.bfloat16, (c.T, c.d))
            moe_rmsnorm(s, t["x"], t["norm_gain"], c.norm_eps, x, st)
        moe_route(s, x, t["W_router"], t["expert_bias"], c.score_fn, c.norm_topk, c.route_scale,
                  self.topk_idx, self.topk_w, self.workspace, st)
        rec(1)
        (moe_permute_fp8 if c.fp8 else moe_permute)(s, self.topk_idx, self.topk_w, self.workspace, st)
        rec(2)
        if c.fp8:
            moe_expert_gate_up_fp8(s, x, t["W_gate_f8"], t["W_up_f8"], t["W_shared_gate_f8"],
                                   t["W_shared_up_f8"], self.workspace, st)
        else:
            moe_expert_gate_up(s, x, t["W_gate"], t["W_up"], t["W_shared_gate"], t["W_shared_up"],
                               self.workspace, st)
        rec(3)
        if c.fp8:
            moe_expert_down_fp8(s, t["W_down_f8"], t["W_shared_down_f8"], self.workspace, st)
        else:
            moe_expert_down(s, t["W_down"], t["W_shared_down"], self.workspace, st)
        rec(4)
        moe_combine(s, self.out, self.workspace, st, x=x, W_shared_gate_vec=t.get("W_shared_gate_vec"))
        rec(5)
        return self.out, self.topk_idx, self.topk_w
