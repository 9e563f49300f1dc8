"""Seeded synthetic inputs for the MoE FFN block.

This module only draws numbers: it holds none of the block's arithmetic, and
both the CUDA path and the fp64 oracle take their inputs from it.

Recipe (same for every workload):
  * one ``torch.Generator`` on the target device, seeded with the workload's
    seed;
  * draw order: x, W_router, expert_bias, W_gate, W_up, W_down,
    W_shared_gate, W_shared_up, W_shared_down, then (gated shared expert only)
    W_shared_gate_vec [S,d], then (pre-norm only) the zero-centred RMSNorm
    gains norm_gain [d] ~ N(0, 0.1), then (skewed workload only) the shuffled
    expert ranks;
  * each tensor is drawn as fp32 N(0, std) in slabs of at most 2**27 elements
    along its first axis, then rounded to bf16 (expert_bias stays fp32);
  * x ~ N(0, 1); all weights ~ N(0, 0.02); expert_bias ~ N(0, 0.1) where the
    workload has one.

Skewed workload ("large_imbalanced"): each expert e gets a rank r_e from a
seeded shuffle of 1..E, and its logit is offset by 0.5*ln(1/r_e).  The block
has no logit-bias input, so the offset is carried by the data: x[:, 0] = 1 and
W_router[e, 0] = bf16(0.5*ln(1/r_e)).  That shifts logit e by exactly that bf16
value in every implementation.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import numpy as np
import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    S: int
    fs: int
    score_fn: str = "softmax"          # softmax | sigmoid | sqrt_softplus
    norm_topk: bool = True
    route_scale: float = 1.0
    bias_std: float = 0.0              # 0 = no expert_bias tensor
    skew: str = ""                     # "" | "zipf_rank"
    shared_gate: bool = False          # per-token sigmoid gate on the shared experts (Qwen3.5)
    prenorm: bool = False              # pre-norm RMSNorm (zero-centred gains) in front of the block
    fp8: bool = False                  # expert weights also as block-scaled FP8 (quantised from the bf16 draw)
    norm_eps: float = 1e-6
    seed: int = 0
    x_std: float = 1.0
    w_std: float = 0.02

    def shape_dict(self):
        return dict(T=self.T, d_model=self.d, E=self.E, k=self.k, d_ff=self.f,
                    n_shared=self.S, d_ff_shared=self.fs)

    def as_dict(self):
        return asdict(self)


# The five workloads of the block, with the sizes the pages' models use.
CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, d=256, E=8, k=2, f=128, S=1, fs=128,
                      score_fn="softmax", seed=0),
    "prefill_softmax": MoEConfig("prefill_softmax", T=4096, d=2048, E=256, k=8, f=512, S=1, fs=512,
                                 score_fn="softmax", seed=1),
    "prefill_sigmoid": MoEConfig("prefill_sigmoid", T=8192, d=4096, E=384, k=8, f=1024, S=1, fs=2048,
                                 score_fn="sigmoid", bias_std=0.1, seed=2),
    "decode_sqrt_softplus": MoEConfig("decode_sqrt_softplus", T=64, d=4096, E=512, k=10, f=1024, S=1,
                                      fs=1024, score_fn="sqrt_softplus", bias_std=0.1, seed=3),
    "large_imbalanced": MoEConfig("large_imbalanced", T=16384, d=7168, E=896, k=22, f=512, S=2, fs=1024,
                                  score_fn="softmax", skew="zipf_rank", seed=4),
}

_SLAB = 1 << 27


def _randn_bf16(shape, std, gen, device):
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if out.numel() == 0:
        return out
    per_row = max(1, out[0].numel()) if len(shape) > 1 else 1
    rows = max(1, _SLAB // per_row)
    n0 = shape[0]
    for i in range(0, n0, rows):
        j = min(n0, i + rows)
        tmp = torch.randn((j - i,) + tuple(shape[1:]), generator=gen, device=device,
                          dtype=torch.float32)
        out[i:j] = (tmp * std).to(torch.bfloat16)
        del tmp
    return out


def make_inputs(cfg: MoEConfig, device="cpu", seed=None):
    """Draw the seeded inputs of ``cfg`` on ``device``.  Returns a dict of tensors."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(cfg.seed if seed is None else seed)
    T, d, E, f, S, fs = cfg.T, cfg.d, cfg.E, cfg.f, cfg.S, cfg.fs
    x = _randn_bf16((T, d), cfg.x_std, gen, device)
    W_router = _randn_bf16((E, d), cfg.w_std, gen, device)
    bias = None
    if cfg.bias_std > 0:
        bias = torch.randn((E,), generator=gen, device=device, dtype=torch.float32) * cfg.bias_std
    W_gate = _randn_bf16((E, f, d), cfg.w_std, gen, device)
    W_up = _randn_bf16((E, f, d), cfg.w_std, gen, device)
    W_down = _randn_bf16((E, d, f), cfg.w_std, gen, device)
    if S > 0:
        W_shared_gate = _randn_bf16((S, fs, d), cfg.w_std, gen, device)
        W_shared_up = _randn_bf16((S, fs, d), cfg.w_std, gen, device)
        W_shared_down = _randn_bf16((S, d, fs), cfg.w_std, gen, device)
    else:
        W_shared_gate = W_shared_up = W_shared_down = None
    W_shared_gate_vec = None
    if cfg.shared_gate and S > 0:
        W_shared_gate_vec = _randn_bf16((S, d), cfg.w_std, gen, device)
    fp8 = {}
    if cfg.fp8:
        for name, w in (("W_gate", W_gate), ("W_up", W_up), ("W_down", W_down), ("W_shared_gate", W_shared_gate),
                        ("W_shared_up", W_shared_up), ("W_shared_down", W_shared_down)):
            fp8[name + "_f8"] = quantize_mxfp8(w) if w is not None else None
    norm_gain = None
    if cfg.prenorm:
        norm_gain = _randn_bf16((d,), 0.1, gen, device)
    ranks = None
    if cfg.skew == "zipf_rank":
        ranks = torch.randperm(E, generator=gen, device=device) + 1
        offset = 0.5 * torch.log(1.0 / ranks.to(torch.float64))
        x[:, 0] = 1.0
        W_router[:, 0] = offset.to(torch.bfloat16)
    return dict(x=x, W_router=W_router, expert_bias=bias, W_gate=W_gate, W_up=W_up, W_down=W_down,
                W_shared_gate=W_shared_gate, W_shared_up=W_shared_up, W_shared_down=W_shared_down,
                W_shared_gate_vec=W_shared_gate_vec, norm_gain=norm_gain, ranks=ranks, **fp8)


def quantize_mxfp8(w, block=32):
    """bf16 weights [G, rows, K] -> (codes uint8 [G, rows, K], scales uint8 [G, K/32, rows]).

    Synthetic FP8 weights: per 32-element block along K the scale is the
    smallest power of two 2^(u-127) with max|w| / 2^(u-127) <= 448 (the largest
    E4M3 magnitude), and each code is w / 2^(u-127) rounded to the nearest
    E4M3 value (ties to even).  An all-zero block gets u = 127."""
    G, rows, K = w.shape
    if K % block:
        raise ValueError("K must be a multiple of the block size")
    nb = K // block
    codes = torch.empty((G, rows, K), dtype=torch.uint8, device=w.device)
    scales = torch.empty((G, nb, rows), dtype=torch.uint8, device=w.device)
    per = max(1, (1 << 26) // max(1, rows * K))
    for g0 in range(0, G, per):
        g1 = min(G, g0 + per)
        wf = w[g0:g1].float().view(g1 - g0, rows, nb, block)
        amax = wf.abs().amax(-1)                                      # [g, rows, nb]
        m, e = torch.frexp(amax / 448.0)                              # amax/448 = m 2^e, 0.5 <= m < 1
        ce = torch.where(m == 0.5, e - 1, e)                          # ceil(log2(amax / 448))
        u = torch.where(amax > 0, ce + 127, torch.full_like(ce, 127)).clamp(1, 254)
        scaled = wf / torch.exp2((u - 127).float()).unsqueeze(-1)
        q = scaled.to(torch.float8_e4m3fn).view(torch.uint8)
        codes[g0:g1] = q.view(g1 - g0, rows, K)
        scales[g0:g1] = u.to(torch.uint8).permute(0, 2, 1)
        del wf, amax, m, e, ce, u, scaled, q
    return codes, scales


def bf16_bits(t):
    """Raw bf16 bit patterns of a tensor as a host numpy uint16 array (None passes through)."""
    if t is None:
        return None
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def host_f32(t):
    return None if t is None else t.detach().contiguous().cpu().numpy().astype(np.float32)


def oracle_args(inp):
    """Host copies of a make_inputs() dict in the form the oracle takes."""
    return dict(x=bf16_bits(inp["x"]), W_router=bf16_bits(inp["W_router"]),
                W_gate=bf16_bits(inp["W_gate"]), W_up=bf16_bits(inp["W_up"]),
                W_down=bf16_bits(inp["W_down"]),
                W_shared_gate=bf16_bits(inp["W_shared_gate"]),
                W_shared_up=bf16_bits(inp["W_shared_up"]),
                W_shared_down=bf16_bits(inp["W_shared_down"]),
                expert_bias=host_f32(inp["expert_bias"]),
                shared_gate=bf16_bits(inp.get("W_shared_gate_vec")))


def from_bits(a, device="cpu"):
    """Inverse of bf16_bits: uint16 numpy array -> bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def bf16_round(a):
    """Round a float array to the nearest bf16 (ties to even) and return its bits."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def pad_to(n, m):
    return (n + m - 1) // m * m


__all__ = ["MoEConfig", "CONFIGS", "make_inputs", "bf16_bits", "host_f32", "oracle_args",
           "from_bits", "bf16_round", "pad_to"]
