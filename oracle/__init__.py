"""fp64 CPU oracle of the mixture-of-experts FFN block.

TEST INFRASTRUCTURE ONLY.  The parity reference for the CUDA path: only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA library, and the library
never calls it.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, one loop per token over
the selected experts); this module builds it with gcc and marshals numpy arrays.
bf16 tensors are passed as their raw 16-bit patterns (numpy ``uint16``).

Parity pins (what fixes this oracle other than itself) are in
``tests/test_oracle_pins.py``.  Value-level parity against the pages is
unpinned: the pages print no worked numerical example for the block, so the
values are pinned by closed forms, special cases and invariants only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SOFTMAX, SIGMOID, SQRT_SOFTPLUS = 0, 1, 2
SCORE_FNS = {"softmax": SOFTMAX, "sigmoid": SIGMOID, "sqrt_softplus": SQRT_SOFTPLUS}

# A prebuilt library loaded instead of liboracle.so.  Only the planted-mistake
# tests set it, to run the pins against mutated copies of moe_oracle.c.
_OVERRIDE = os.environ.get("MOE_ORACLE_LIB") or None

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc, -O2, no fast-math)."""
    if _OVERRIDE:
        return _OVERRIDE
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i = ctypes.c_int
            lib.oracle_moe_forward.restype = i
            lib.oracle_moe_forward.argtypes = (
                [i] * 7 + [P] * 3 + [P] * 6 + [i, i, ctypes.c_double] + [P, i, P, P, P, i] + [P] * 8 + [i])
            lib.oracle_rmsnorm.restype = i
            lib.oracle_rmsnorm.argtypes = [i, i, P, P, ctypes.c_double, P, P]
            lib.oracle_double_to_bf16.restype = ctypes.c_uint16
            lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
            lib.oracle_e4m3_to_double.restype = ctypes.c_double
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_dequant_mxfp8.restype = i
            lib.oracle_dequant_mxfp8.argtypes = [i, i, i, P, P, P]
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _u16(a, shape, name):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"{name}: expected raw bf16 bits as uint16, got {a.dtype}")
    if tuple(a.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(a.shape)}")
    return a


def forward(x, W_router, W_gate=None, W_up=None, W_down=None,
            W_shared_gate=None, W_shared_up=None, W_shared_down=None,
            expert_bias=None, *, k, score_fn="softmax", norm_topk=True, route_scale=1.0,
            tokens=None, forced_idx=None, forced_w=None, shared_gate=None, route_only=False,
            want_logits=False, n_threads=None):
    """Run the oracle.

    Shapes (bf16 bit patterns as uint16): x [T,d], W_router [E,d],
    W_gate/W_up [E,f,d], W_down [E,d,f], W_shared_gate/up [S,fs,d],
    W_shared_down [S,d,fs]; expert_bias fp32 [E] or None.

    ``tokens`` restricts evaluation to those token ids (outputs are in that
    order); ``forced_idx`` [n,k] replaces the router's choice of experts (the
    weights are then the scores of the forced experts, renormalised the same
    way) unless ``forced_w`` [n,k] gives the weights as well (external
    routing).  ``shared_gate`` [S,d] (bf16 bits) scales shared expert s by
    sigma(shared_gate[s] . x) per token.  Returns a dict of float64/int32 numpy arrays: ``out`` [n,d],
    ``topk_idx`` [n,k], ``topk_w`` [n,k], ``sel_keys`` / ``sel_order`` [n,k+1]
    (selection keys and experts of the first k+1 in selection order; -inf / -1
    past E), and with ``want_logits`` also ``logits``, ``scores`` and the
    selection ``keys`` [n,E].
    """
    lib = _load()
    T, d = x.shape
    E = W_router.shape[0]
    x = _u16(x, (T, d), "x")
    W_router = _u16(W_router, (E, d), "W_router")
    if route_only:
        f, S, fs = 1, 0, 1
    else:
        f = W_gate.shape[1]
        W_gate = _u16(W_gate, (E, f, d), "W_gate")
        W_up = _u16(W_up, (E, f, d), "W_up")
        W_down = _u16(W_down, (E, d, f), "W_down")
        S = 0 if W_shared_gate is None else W_shared_gate.shape[0]
        fs = 1 if S == 0 else W_shared_gate.shape[1]
        if S:
            W_shared_gate = _u16(W_shared_gate, (S, fs, d), "W_shared_gate")
            W_shared_up = _u16(W_shared_up, (S, fs, d), "W_shared_up")
            W_shared_down = _u16(W_shared_down, (S, d, fs), "W_shared_down")
    if expert_bias is not None:
        expert_bias = np.ascontiguousarray(expert_bias, dtype=np.float32)
        if expert_bias.shape != (E,):
            raise ValueError("expert_bias must be fp32 [E]")
    if tokens is None:
        tok = None
        n = T
    else:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        n = int(tok.shape[0])
    forced = None if forced_idx is None else np.ascontiguousarray(forced_idx, dtype=np.int32)
    if forced is not None and forced.shape != (n, k):
        raise ValueError("forced_idx must be [n_tokens, k]")
    fw = None if forced_w is None else np.ascontiguousarray(forced_w, dtype=np.float64)
    if fw is not None and (forced is None or fw.shape != (n, k)):
        raise ValueError("forced_w needs forced_idx and must be [n_tokens, k]")
    sg = None
    if shared_gate is not None:
        if route_only or S == 0:
            raise ValueError("shared_gate needs shared experts")
        sg = _u16(shared_gate, (S, d), "shared_gate")

    out = None if route_only else np.zeros((n, d), np.float64)
    topk_idx = np.zeros((n, k), np.int32)
    topk_w = np.zeros((n, k), np.float64)
    sel_keys = np.zeros((n, k + 1), np.float64)
    sel_order = np.zeros((n, k + 1), np.int32)
    logits = np.zeros((n, E), np.float64) if want_logits else None
    scores = np.zeros((n, E), np.float64) if want_logits else None
    keys = np.zeros((n, E), np.float64) if want_logits else None
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    st = lib.oracle_moe_forward(
        T, d, E, k, f, S, fs,
        _ptr(x), _ptr(W_router), _ptr(expert_bias),
        _ptr(W_gate), _ptr(W_up), _ptr(W_down),
        _ptr(W_shared_gate), _ptr(W_shared_up), _ptr(W_shared_down),
        SCORE_FNS[score_fn] if isinstance(score_fn, str) else int(score_fn),
        int(bool(norm_topk)), float(route_scale),
        _ptr(tok), n, _ptr(forced), _ptr(fw), _ptr(sg), int(bool(route_only)),
        _ptr(out), _ptr(topk_idx), _ptr(topk_w), _ptr(sel_keys), _ptr(sel_order),
        _ptr(logits), _ptr(scores), _ptr(keys), int(n_threads))
    if st != 0:
        raise ValueError(f"oracle_moe_forward failed with status {st}")
    res = {"out": out, "topk_idx": topk_idx, "topk_w": topk_w, "sel_keys": sel_keys,
           "sel_order": sel_order}
    if want_logits:
        res["logits"] = logits
        res["scores"] = scores
        res["keys"] = keys
    return res


def rel_gap(a, b):
    """|a-b| / max(|a|,|b|), elementwise, 0 where both are 0."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    m = np.maximum(np.abs(a), np.abs(b))
    with np.errstate(invalid="ignore", divide="ignore"):
        g = np.where(m > 0, np.abs(a - b) / np.where(m > 0, m, 1.0), 0.0)
    return g


def to_bf16_bits(values):
    """fp64 values -> raw bf16 bits (nearest, ties to even), element by element."""
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    flat, of = v.ravel(), out.ravel()
    for n in range(flat.size):
        of[n] = lib.oracle_double_to_bf16(float(flat[n]))
    return out


def rmsnorm(x, gain, eps):
    """Pre-norm RMSNorm with zero-centred gains: y = x / sqrt(mean(x^2) + eps) * (1 + g).

    x: [T, d] raw bf16 bits (uint16); gain: [d] raw bf16 bits; eps: float.
    Returns {"y": fp64 [T, d], "y_bits": bf16 bits [T, d] (y rounded to nearest even)}.
    """
    lib = _load()
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16 or x.ndim != 2:
        raise TypeError("x: expected [T, d] raw bf16 bits (uint16)")
    T, d = x.shape
    gain = _u16(gain, (d,), "gain")
    y = np.empty((T, d), dtype=np.float64)
    yb = np.empty((T, d), dtype=np.uint16)
    rc = lib.oracle_rmsnorm(T, d, _ptr(x), _ptr(gain), float(eps), _ptr(y), _ptr(yb))
    if rc != 0:
        raise ValueError(f"oracle_rmsnorm: invalid arguments ({rc})")
    return {"y": y, "y_bits": yb}


def e4m3_value(code):
    """Value of one E4M3 (OCP E4M3FN) code, as a Python float."""
    return float(_load().oracle_e4m3_to_double(int(code) & 0xFF))


def dequant_mxfp8(q, scale):
    """Block-scaled FP8 weights -> raw bf16 bits.

    q: uint8 [G, rows, K] E4M3 codes; scale: uint8 [G, K/32, rows] UE8M0
    exponents (2^(s-127)) of the 32-element blocks along K.  Raises if a value
    is NaN or has no exact bf16 form."""
    q = np.ascontiguousarray(q)
    scale = np.ascontiguousarray(scale)
    if q.dtype != np.uint8 or scale.dtype != np.uint8 or q.ndim != 3:
        raise TypeError("q: uint8 [G, rows, K]; scale: uint8 [G, K/32, rows]")
    G, rows, K = q.shape
    if K % 32 or scale.shape != (G, K // 32, rows):
        raise ValueError(f"scale: expected shape {(G, K // 32, rows)}, got {scale.shape}")
    out = np.empty((G, rows, K), dtype=np.uint16)
    rc = _load().oracle_dequant_mxfp8(G, rows, K, _ptr(q), _ptr(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_dequant_mxfp8: {'bad arguments' if rc == -1 else 'value without an exact bf16 form'}")
    return out
