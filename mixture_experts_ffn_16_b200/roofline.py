"""Algorithmic cost of the MoE block and of each of its kernels.

Counts only what the method must do, not what an implementation moves:
  FLOPs  2*M*N*K per GEMM: router (T x E x d), gate and up (T*k rows and S*T
         shared rows, each 2 x f x d), down (same rows, d x f).
  bytes  every weight matrix a kernel needs read once (routed experts only if
         some token picked them), activations read once and results written
         once, in their stored dtype (block-scaled FP8 expert weights: one
         byte per code plus one scale byte per 32 codes).
"""
from __future__ import annotations

import hashlib
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def measured_peaks():
    """Peaks measured on this machine's B200s (generated file), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def weight_bytes(cfg):
    """Bytes per expert-weight element: bf16, or FP8 code + 1/32 scale byte."""
    return 1.0 + 1.0 / 32.0 if getattr(cfg, "fp8", False) else 2.0


def kernel_costs(cfg, touched=None):
    """Per-step algorithmic (flops, bytes) of each step of the block.

    touched: number of routed experts with at least one token (default: all E).
    """
    T, d, E, k, f, S, fs = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.S, cfg.fs
    wb = weight_bytes(cfg)
    ne = E if touched is None else int(touched)
    R = T * k
    c = {}
    # a1+a2: router GEMM (x, W_router in; fp32 logits out) + top-k (logits in, idx/w out)
    c["route"] = (2.0 * T * E * d, 2.0 * (T * d + E * d) + 4.0 * T * E * 2 + 8.0 * T * k)
    # a3: permute: read idx/w twice, write perm/row_w/inv
    c["permute"] = (0.0, 8.0 * R * 2 + 12.0 * R)
    # a4 + a6 gate/up: weights of touched experts and shared, x, H out
    c["gate_up"] = (2.0 * (R * 2 * f * d + S * T * 2 * fs * d),
                    wb * (ne * 2 * f * d + S * 2 * fs * d) + 2.0 * (T * d + R * f + S * T * fs))
    # a5 + a6 down: W_down, H in, Y out
    c["down"] = (2.0 * (R * d * f + S * T * d * fs),
                 wb * (ne * d * f + S * d * fs) + 2.0 * (R * f + S * T * fs + R * d + S * T * d))
    # a7 combine: Y rows in, out written
    c["combine"] = (float((R + S * T) * d), 2.0 * ((R + S * T) * d + T * d) + 4.0 * R)
    return c


def block_cost(cfg, touched=None):
    """Whole-block algorithmic (flops, bytes): the minimum any implementation
    needs (weights of touched experts once, x in, out and routing out)."""
    T, d, E, k, f, S, fs = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.S, cfg.fs
    ne = E if touched is None else int(touched)
    flops = 2.0 * T * E * d + 2.0 * T * k * 3 * f * d + 2.0 * T * S * 3 * fs * d
    bytes_ = (weight_bytes(cfg) * (ne * 3 * f * d + S * 3 * fs * d) + 2.0 * (E * d + 2 * T * d)
              + 8.0 * T * k)
    return flops, bytes_


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch, from
# the committed ncu captures (profiles/): the three GEMMs of one
# prefill_softmax step, captured at full size.  Each figure holds for the
# moe_gemm.cu revision listed with it (sha256 prefix of the source without
# comments, see _gemm_source_sha).  The other workloads are too large for a
# full-counter capture; their reduced-size captures (profiles/) do not scale
# to a full launch in proportion (token-row reuse depends on k and E), so
# their traffic is reported as unknown (None).
_CAPTURED = "a6521d2b2a109933"
NCU_TRAFFIC = {
    ("prefill_softmax", "route"): (17.9e6, {_CAPTURED}),
    ("prefill_softmax", "gate_up"): (1106.0e6, {_CAPTURED}),
    ("prefill_softmax", "down"): (710.0e6, {_CAPTURED}),
}


def _gemm_source_sha():
    """sha256 prefix of moe_gemm.cu with comments and blank lines removed: a
    comment edit does not change the kernels the counters were taken from."""
    p = os.path.join(ROOT, "mixture_experts_ffn_16_b200", "csrc", "moe_gemm.cu")
    try:
        with open(p, encoding="utf-8") as fh:
            lines = [ln.split("//", 1)[0].rstrip() for ln in fh]
    except OSError:
        return None
    code = "\n".join(ln for ln in lines if ln.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def measured_traffic(workload, kernel):
    """Bytes per launch from the committed capture, or None when there is none
    or the kernel source has changed since it was taken."""
    rec = NCU_TRAFFIC.get((workload, kernel))
    if rec is None or _gemm_source_sha() not in rec[1]:
        return None
    return rec[0]
