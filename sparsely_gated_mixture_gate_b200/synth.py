"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws numbers: it holds none of the layer's arithmetic and
imports neither the CUDA library nor the oracle, so both sides of a parity
test can take their inputs from it.  The random numbers the layer itself draws
(the gate noise) are not made here: each side generates those from its own
counter-based stream.

Recipe (per workload, seed 0 unless stated):
  x        ~ N(0, 1); for the LM-shaped workloads each row is rescaled to
             Euclidean norm sqrt(d_model).
  W_g, W_noise, secondary gates ~ N(0, 1/d_model)   (variance = 1/fan_in)
  W1 ~ N(0, 1/d_model), W2 ~ N(0, 1/f)               (variance = 1/fan_in)
  biases   0, or N(0, bias_var) when a workload asks for biases
  b_g      0, or N(0, logit_bias_var) per expert to skew the load
  expert weights are cast to bf16 (round to nearest even) for bf16 experts.
Expert weights are stored K-major, i.e. as each linear map's
[out_features][in_features]: W1 is [n][f][d], W2 is [n][d][f].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    n: int
    k: int
    f: int
    hier_a: int = 0
    hier_b: int = 0
    hier_k1: int = 0
    hier_k2: int = 0
    router: int = 0             # 0 noisy top-k gate, 1 Switch top-1 router, 2 sigmoid router
    noise: int = 1
    expert_bf16: int = 1
    capacity_factor: float = 0.0
    passthrough: int = 0
    x_unit_rows: bool = False   # rescale each token to norm sqrt(d)
    logit_bias_var: float = 0.0
    bias_var: float = 0.0
    seed: int = 0
    w_importance: float = 0.1
    w_load: float = 0.1
    alpha: float = 0.01
    gate_precision: int = 0     # library option; the oracle is always fp64
    shared_expert: int = 0      # 1: one always-active expert added to every token
    sel_bias_std: float = 0.0   # sigmoid router: spread of the selection bias
    router_stats: int = 0       # 1: the router z-loss and entropy are reported too
    w_z: float = 0.0            # backward: weights of the z-loss and of the entropy
    w_entropy: float = 0.0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def gate_n(self) -> int:
        """Width of the flat (or primary) gate."""
        return self.hier_a if self.hier_a else self.n

    def cfg(self) -> dict:
        keys = ("T", "d", "n", "k", "f", "hier_a", "hier_b", "hier_k1", "hier_k2", "router",
                "noise", "expert_bf16", "capacity_factor", "passthrough", "seed",
                "w_importance", "w_load", "alpha", "shared_expert", "router_stats", "w_z",
                "w_entropy")
        return {k: getattr(self, k) for k in keys}


# The five workloads of the layer, smallest first.
WORKLOADS = {
    "tiny-flat": Workload("tiny-flat", T=64, d=32, n=8, k=2, f=64, expert_bf16=0),
    "lm-flat": Workload("lm-flat", T=8192, d=512, n=256, k=4, f=1024, x_unit_rows=True),
    "many-expert": Workload("many-expert", T=65536, d=512, n=4096, k=4, f=1024,
                            x_unit_rows=True, logit_bias_var=0.5),
    "hierarchical": Workload("hierarchical", T=65536, d=512, n=64 * 128, k=4, f=1024,
                             hier_a=64, hier_b=128, hier_k1=2, hier_k2=2, x_unit_rows=True),
    "switch-top1": Workload("switch-top1", T=32768, d=1024, n=128, k=1, f=4096, router=1,
                            noise=0, capacity_factor=1.25, passthrough=1),
}

# Parity-only variants (not benchmark workloads).
VARIANTS = {
    # biases drawn so that the bias adds are exercised
    "tiny-bias": WORKLOADS["tiny-flat"].with_(name="tiny-bias", bias_var=0.1, logit_bias_var=0.1),
    # a skewed Switch router so that the capacity limit actually drops tokens
    "switch-skew": WORKLOADS["switch-top1"].with_(name="switch-skew", logit_bias_var=0.5),
    # sigmoid router with a selection bias and a shared expert ("MoE 稀疏架构深度
    # 解析" §5.2, §6.2, §6.3), DeepSeek-V3's shape scaled to the lm-flat layer:
    # 256 routed experts, top 8 of them, experts half as wide, one shared expert
    "deepseek-tiny": Workload("deepseek-tiny", T=64, d=32, n=16, k=4, f=64, router=2, noise=0,
                              shared_expert=1, sel_bias_std=0.5, bias_var=0.1),
    "deepseek-tiny-f32": Workload("deepseek-tiny-f32", T=64, d=32, n=16, k=4, f=64, router=2,
                                  noise=0, shared_expert=1, sel_bias_std=0.5, expert_bf16=0),
    "deepseek-flat": Workload("deepseek-flat", T=8192, d=512, n=256, k=8, f=512, router=2,
                              noise=0, shared_expert=1, sel_bias_std=0.1, x_unit_rows=True),
    # the hierarchical layer with 8 of its 64 groups and the same ~32 rows per
    # expert: 2.1 GB of expert weights instead of 17.2 GB, for profiler captures
    "hierarchical-a8": WORKLOADS["hierarchical"].with_(name="hierarchical-a8", T=8192, n=8 * 128,
                                                       hier_a=8),
}


def _gen(device, seed: int, tag: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + tag)
    return g


def _randn(shape, std, device, seed, tag, dtype=torch.float32):
    t = torch.randn(*shape, generator=_gen(device, seed, tag), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t if dtype == torch.float32 else t.to(dtype)


def _randn_chunked(n, rows, cols, std, device, seed, tag, dtype, chunk=256):
    """[n][rows][cols], drawn expert by expert in chunks so that the fp32
    temporary stays small for bf16 outputs."""
    out = torch.empty(n, rows, cols, device=device, dtype=dtype)
    g = _gen(device, seed, tag)
    for e0 in range(0, n, chunk):
        e1 = min(n, e0 + chunk)
        t = torch.randn(e1 - e0, rows, cols, generator=g, device=device, dtype=torch.float32)
        t.mul_(std)
        out[e0:e1].copy_(t)
    return out


def make_inputs(w: Workload, device="cpu", T: Optional[int] = None, seed: Optional[int] = None,
                experts: bool = True) -> dict:
    """All tensors of one workload.  ``T`` overrides the token count (the
    first T rows of x are the same for any T); ``experts=False`` skips the
    expert weights."""
    s = w.seed if seed is None else seed
    T = w.T if T is None else T
    d, n, f = w.d, w.n, w.f
    gn = w.gate_n
    out = {}
    x = _randn((w.T, d), 1.0, device, s, 1)[:T].contiguous()
    if w.x_unit_rows:
        x.mul_(math.sqrt(d) / x.norm(dim=1, keepdim=True).clamp_min(1e-30))
    out["x"] = x
    gstd = 1.0 / math.sqrt(d)
    out["Wg"] = _randn((d, gn), gstd, device, s, 2)
    out["Wn"] = _randn((d, gn), gstd, device, s, 3) if w.noise else None
    if w.logit_bias_var > 0:
        out["bg"] = _randn((gn,), math.sqrt(w.logit_bias_var), device, s, 4)
    else:
        out["bg"] = None
    if w.hier_a:
        out["Wg2"] = _randn((w.hier_a, d, w.hier_b), gstd, device, s, 5)
        out["Wn2"] = _randn((w.hier_a, d, w.hier_b), gstd, device, s, 6) if w.noise else None
        out["bg2"] = None
    out["sel_bias"] = (_randn((gn,), w.sel_bias_std, device, s, 12)
                       if w.router == 2 and w.sel_bias_std > 0 else None)
    if experts:
        edt = torch.bfloat16 if w.expert_bf16 else torch.float32
        out["W1"] = _randn_chunked(n, f, d, 1.0 / math.sqrt(d), device, s, 7, edt)
        out["W2"] = _randn_chunked(n, d, f, 1.0 / math.sqrt(f), device, s, 8, edt)
        if w.bias_var > 0:
            out["b1"] = _randn((n, f), math.sqrt(w.bias_var), device, s, 9)
            out["b2"] = _randn((n, d), math.sqrt(w.bias_var), device, s, 10)
        else:
            out["b1"] = torch.zeros(n, f, device=device)
            out["b2"] = torch.zeros(n, d, device=device)
        if w.shared_expert:
            out["W1s"] = _randn_chunked(1, f, d, 1.0 / math.sqrt(d), device, s, 13, edt)[0]
            out["W2s"] = _randn_chunked(1, d, f, 1.0 / math.sqrt(f), device, s, 14, edt)[0]
            sv = math.sqrt(w.bias_var) if w.bias_var > 0 else 0.0
            out["b1s"] = _randn((f,), sv, device, s, 15) if sv else torch.zeros(f, device=device)
            out["b2s"] = _randn((d,), sv, device, s, 16) if sv else torch.zeros(d, device=device)
    return out


def make_dy(w: Workload, device="cpu", T: Optional[int] = None, seed: Optional[int] = None):
    """Upstream gradient of the layer output for the backward pass: [T][d]
    standard normal (the first T rows are the same for any T)."""
    s = w.seed if seed is None else seed
    T = w.T if T is None else T
    return _randn((w.T, w.d), 1.0, device, s, 17)[:T].contiguous()


def random_routing(T: int, k: int, n: int, device="cpu", seed: int = 0, skew: float = 0.0,
                   invalid_frac: float = 0.0) -> torch.Tensor:
    """Synthetic expert choices [T][k] for stand-alone dispatch tests: k
    distinct experts per token, drawn with optional Zipf-like skew; a fraction
    of entries can be replaced by out-of-range ids."""
    if T == 0:
        return torch.zeros(0, k, dtype=torch.int32, device=device)
    g = _gen(device, seed, 11)
    if skew > 0:
        w = torch.arange(1, n + 1, device=device, dtype=torch.float64).pow(-skew)
    else:
        w = torch.ones(n, device=device, dtype=torch.float64)
    idx = torch.multinomial(w.float().expand(T, n), k, replacement=False, generator=g).to(torch.int32)
    if invalid_frac > 0:
        m = torch.rand(T, k, generator=g, device=device) < invalid_frac
        bad = torch.where(torch.rand(T, k, generator=g, device=device) < 0.5,
                          torch.full_like(idx, -1), torch.full_like(idx, n + 3))
        idx = torch.where(m, bad, idx)
    return idx.contiguous()


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (for the oracle)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view("uint16")
