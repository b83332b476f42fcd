"""Seeded synthetic inputs for the KDA recurrence.

This module only draws random numbers and prepares them the way the host
model prepares real activations; it holds none of the recurrence's own
arithmetic.  The CUDA path and the float64 oracle both consume the exact
tensors produced here (the oracle after an exact upcast to float64).

Preparation follows "kimi_k3_host/kda.rs":

* ``l2norm_rows``: x * (sum(x^2) + 1e-6)^(-1/2) per head row (the epsilon is
  added to the sum of squares, inside the square root), in fp32, then the
  result is rounded to the workload's input dtype;
* ``bounded_gate``: with a lower bound lb, g = lb * sigmoid(x); without one,
  g = -exp(A_log[h]) * softplus(z + dt_bias[h, d]) (the "twin" geometry has
  no bound);
* beta = sigmoid(logit) -- the recurrence takes beta after the sigmoid.

All random draws use one CPU ``torch.Generator`` seeded with
20261202 + workload index, in this fixed order: q, k, v, gate noise z,
beta logit, (A_log, dt_bias for the unbounded gate), S0, dO.  Overriding a
size (``T=...``) keeps the recipe and the draw order, so smaller parity cases
have the same value distributions as the full workloads.
"""
from __future__ import annotations

import dataclasses
import math

import torch

L2_EPS = 1e-6
SEED_BASE = 20261202


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic KDA workload (sizes, dtype and value recipe)."""

    name: str
    index: int
    B: int
    T: int
    H: int
    HV: int
    K: int
    V: int
    dtype: str            # "fp32" or "bf16": q, k, v, o (and dq, dk, dv, dO)
    gate: str             # "bounded" (-5 * sigmoid(z)) or "softplus" (unbounded)
    s0_std: float         # 0.0 means S0 = 0
    path: str             # "fwd", "fwdbwd" or "decode"
    chunk: int            # chunk length the prefill kernels use at this K

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.K)

    def with_sizes(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = [
    Workload("tiny", 0, B=1, T=64, H=2, HV=2, K=32, V=32, dtype="fp32",
             gate="bounded", s0_std=0.0, path="fwd", chunk=32),
    Workload("twin", 1, B=4, T=1024, H=8, HV=8, K=32, V=32, dtype="fp32",
             gate="softplus", s0_std=0.01, path="fwd", chunk=32),
    Workload("prefill_gqa", 2, B=1, T=8192, H=16, HV=96, K=128, V=128, dtype="bf16",
             gate="bounded", s0_std=0.0, path="fwd", chunk=64),
    Workload("fwdbwd", 3, B=2, T=4096, H=96, HV=96, K=128, V=128, dtype="bf16",
             gate="bounded", s0_std=0.0, path="fwdbwd", chunk=64),
    Workload("decode", 4, B=256, T=1, H=96, HV=96, K=128, V=128, dtype="bf16",
             gate="bounded", s0_std=0.02, path="decode", chunk=64),
]
BY_NAME = {w.name: w for w in WORKLOADS}
# The asymmetric erase/write variant ("research_layers.py"): H counts query
# heads (32), HV state heads (8, groups of 4 query heads), K the feature
# dimension (the layer's default 64), V the head dimension.
ERASE = Workload("erase", 5, B=1, T=8192, H=32, HV=8, K=64, V=128, dtype="bf16",
                 gate="erase", s0_std=0.0, path="erase", chunk=32)
BY_NAME[ERASE.name] = ERASE


def _l2norm_rows(x):
    return x * torch.rsqrt((x * x).sum(-1, keepdim=True) + L2_EPS)


def make_inputs(w: Workload, seed: int | None = None, with_do: bool | None = None):
    """Draw the inputs of workload ``w`` on the CPU.

    Returns a dict of contiguous CPU tensors: q, k [B,T,H,K] and v [B,T,HV,V]
    in the workload dtype; g [B,T,HV,K], beta [B,T,HV], S0 [B,HV,K,V] (or None)
    in fp32; dO [B,T,HV,V] in the workload dtype when ``with_do`` (default:
    the fwd+bwd workload).  For the decode workload the T axis is dropped:
    q, k [B,H,K], v [B,HV,V], g [B,HV,K], beta [B,HV] and the state is "S".
    """
    if seed is None:
        seed = SEED_BASE + w.index
    if with_do is None:
        with_do = w.path == "fwdbwd"
    gen = torch.Generator().manual_seed(seed)
    B, T, H, HV, K, V = w.B, w.T, w.H, w.HV, w.K, w.V

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = randn(B, T, H, K)
    k = randn(B, T, H, K)
    v = randn(B, T, HV, V)
    z = randn(B, T, HV, K)
    beta_logit = randn(B, T, HV)
    if w.gate == "bounded":
        g = -5.0 * torch.sigmoid(z)
    elif w.gate == "softplus":
        a_log = torch.rand(HV, generator=gen, dtype=torch.float32) * 2.0 - 2.0
        dt_bias = randn(HV, K) * 0.1
        g = -torch.exp(a_log)[:, None] * torch.nn.functional.softplus(z + dt_bias)
    else:
        raise ValueError(w.gate)
    S0 = randn(B, HV, K, V) * w.s0_std if w.s0_std > 0 else None
    dO = randn(B, T, HV, V) if with_do else None

    dt = w.torch_dtype
    out = {
        "q": _l2norm_rows(q).to(dt).contiguous(),
        "k": _l2norm_rows(k).to(dt).contiguous(),
        "v": v.to(dt).contiguous(),
        "g": g.contiguous(),
        "beta": torch.sigmoid(beta_logit).contiguous(),
        "S0": S0,
        "dO": None if dO is None else dO.to(dt).contiguous(),
    }
    if w.path == "decode":
        if T != 1:
            raise ValueError("the decode workload has T = 1")
        out = {
            "q": out["q"][:, 0].contiguous(),
            "k": out["k"][:, 0].contiguous(),
            "v": out["v"][:, 0].contiguous(),
            "g": out["g"][:, 0].contiguous(),
            "beta": out["beta"][:, 0].contiguous(),
            "S": S0 if S0 is not None else torch.zeros(B, HV, K, V),
        }
    return out


def make_raw_inputs(w: Workload, seed: int | None = None, conv_width: int = 0, lower_bound: float = -5.0):
    """Draw the RAW projections of workload ``w`` for the fused-preparation
    entry points (nothing normalised, no gate or sigmoid applied).

    One CPU generator (default seed 20261202 + 100 + workload index), draws in
    this order: q, k [B,T,H,K] and v [B,T,HV,V] ~ N(0, 1); gate noise z
    [B,T,HV,K] ~ N(0, 1); beta logit [B,T,HV] ~ N(0, 1); A_log [HV] ~ U(-2, 0);
    dt_bias [HV,K] ~ N(0, 0.1^2); output-gate pre-activation [B,T,HV,V] ~
    N(0, 1); S0 as in ``make_inputs``; with ``conv_width`` W > 0 the
    convolution weights [2HK + HV V, W] ~ N(0, 0.5^2) and an initial window
    [B, 2HK + HV V, W] ~ N(0, 1).  q, k, v, z and the output gate are rounded
    to the workload dtype; the rest stays fp32.  ``lower_bound`` is the gate's
    (-5 for the production geometry, 0 = the unbounded softplus form).
    """
    if seed is None:
        seed = SEED_BASE + 100 + w.index
    gen = torch.Generator().manual_seed(seed)
    B, T, H, HV, K, V = w.B, w.T, w.H, w.HV, w.K, w.V

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    dt = w.torch_dtype
    out = {
        "q": randn(B, T, H, K).to(dt), "k": randn(B, T, H, K).to(dt), "v": randn(B, T, HV, V).to(dt),
        "z": randn(B, T, HV, K).to(dt), "beta_logit": randn(B, T, HV),
        "A_log": torch.rand(HV, generator=gen, dtype=torch.float32) * 2.0 - 2.0,
        "dt_bias": randn(HV, K) * 0.1, "og": randn(B, T, HV, V).to(dt),
        "S0": randn(B, HV, K, V) * w.s0_std if w.s0_std > 0 else None,
        "lower_bound": float(lower_bound),
    }
    if conv_width:
        Cn = 2 * H * K + HV * V
        out["conv_w"] = randn(Cn, conv_width) * 0.5
        out["conv_state"] = randn(B, Cn, conv_width)
    return out


def make_erase_inputs(w: Workload, seed: int | None = None):
    """Draw the inputs of the erase/write variant with the value ranges of the
    research layer's feature maps ("research_layers.py", features): q, k rows
    L2-normalised; erase = k * sigmoid(N(-1, 1)) (gate bias -1); z = v *
    sigmoid(N(-1, 1)) with v ~ N(0, 1); g = -0.25 sigmoid(N(log(0.04/0.96), 1))
    (the layer's bounded forget gate).  One CPU generator (default seed
    20261202 + 200 + workload index), draws in the order q, k, v, erase noise,
    write noise, forget noise, S0.  q, k, erase and z are rounded to the
    dtype; g and S0 stay fp32.  Shapes: q [B,T,H,K] (H query heads), k,
    erase, g [B,T,HV,K], z [B,T,HV,V], S0 [B,HV,K,V] or None.
    """
    if seed is None:
        seed = SEED_BASE + 200 + w.index
    gen = torch.Generator().manual_seed(seed)
    B, T, H, HV, K, V = w.B, w.T, w.H, w.HV, w.K, w.V

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    dt = w.torch_dtype
    q = _l2norm_rows(randn(B, T, H, K))
    k = _l2norm_rows(randn(B, T, HV, K))
    v = randn(B, T, HV, V)
    erase = k * torch.sigmoid(randn(B, T, HV, K) - 1.0)
    z = v * torch.sigmoid(randn(B, T, HV, V) - 1.0)
    g = -0.25 * torch.sigmoid(randn(B, T, HV, K) + math.log(0.04 / 0.96))
    S0 = randn(B, HV, K, V) * w.s0_std if w.s0_std > 0 else None
    return {"q": q.to(dt).contiguous(), "k": k.to(dt).contiguous(), "e": erase.to(dt).contiguous(),
            "z": z.to(dt).contiguous(), "g": g.contiguous(), "S0": S0}


def head_subset(inputs: dict, H: int, HV: int, groups):
    """Slice whole grouped-query blocks out of forward/backward inputs.

    ``groups`` lists query/key heads h; the result keeps q/k head h and value
    heads h*G .. h*G+G-1 for each, so the oracle can check a seeded subset of
    heads with complete dq/dk sums.
    """
    G = HV // H
    groups = list(groups)
    hv_idx = [h * G + j for h in groups for j in range(G)]
    sub = {}
    for name, x in inputs.items():
        if x is None:
            sub[name] = None
        elif name in ("q", "k"):
            sub[name] = x[:, :, groups].contiguous()
        elif name in ("v", "g", "beta", "dO"):
            sub[name] = x[:, :, hv_idx].contiguous()
        elif name in ("S0",):
            sub[name] = x[:, hv_idx].contiguous()
        else:
            raise KeyError(name)
    return sub, hv_idx
