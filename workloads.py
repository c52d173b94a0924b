"""Seeded synthetic inputs for the causal linear-attention forward.

This module is the only code shared by the oracle side (``oracle/``, the tests)
and the CUDA side (``bench.py``, the GPU tests).  It draws random numbers and
shapes them into the five workloads; it holds none of the method's arithmetic
(no feature map, no recurrence, no chunking).

Recipe (the same for every workload):

* one ``torch.Generator('cpu')`` seeded with ``seed`` (0 by default);
* draws are fp32 ``N(0,1)`` in the fixed order q, k, v, gate source,
  beta source, initial state;
* scaling and per-token L2 normalisation are applied in fp32, then q/k/v are
  rounded to bf16 (round-to-nearest-even) for the bf16 workloads;
* gate transforms (GLA ``g = exp(-softplus(x)/16)``, gated-delta
  ``alpha = sigmoid(x+3)``, ``beta = sigmoid(x)``) are evaluated in fp64 and
  rounded once to fp32.

Layouts: q, k ``[B,T,H,dk]``; v ``[B,T,H,dv]``; GLA gate ``[B,T,H,dk]``;
alpha, beta ``[B,T,H]``; state ``[B,H,dk,dv]``; ELU normaliser ``[B,H,dk]``.
Both the GPU path and the oracle read exactly these tensors (the oracle after
an exact upcast to fp64).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

RULES = ("elu", "gla", "gdn", "kda")


@dataclass
class Problem:
    """One prefill problem: inputs for ``la_fwd``."""

    rule: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: Optional[torch.Tensor] = None       # GLA gate [B,T,H,dk] / GDN alpha [B,T,H]
    beta: Optional[torch.Tensor] = None    # GDN [B,T,H]
    S0: Optional[torch.Tensor] = None      # [B,H,dk,dv] fp32
    z0: Optional[torch.Tensor] = None      # ELU [B,H,dk] fp32
    eps: float = 1e-6
    name: str = ""
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, T, H, dk = self.q.shape
        return B, T, H, dk, self.v.shape[-1]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _randn(gen, *shape):
    return torch.randn(*shape, generator=gen, dtype=torch.float32)


def _l2norm_last(x: torch.Tensor) -> torch.Tensor:
    # Input preparation (the workload says "q and k L2-normalised per head"),
    # done in fp32 before the bf16 rounding.
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def gla_gate_from(x: torch.Tensor) -> torch.Tensor:
    """g = exp(-softplus(x)/16) in fp64, rounded once to fp32; g is in (0,1)."""
    x64 = x.double()
    return torch.exp(-torch.nn.functional.softplus(x64) / 16.0).float()


def gdn_alpha_from(x: torch.Tensor) -> torch.Tensor:
    return torch.sigmoid(x.double() + 3.0).float()


def gdn_beta_from(x: torch.Tensor) -> torch.Tensor:
    return torch.sigmoid(x.double()).float()


def kda_alpha_from(x: torch.Tensor, g_min: float = -5.0) -> torch.Tensor:
    """Per-channel KDA retention with the bounded log-decay of page "状态空间与线性注意力"
    (有界 log-decay): alpha = exp(g_min * sigmoid(x)) in (e^g_min, 1), the scale
    e^A taken as 1; evaluated in fp64 and rounded once to fp32."""
    return torch.exp(g_min * torch.sigmoid(x.double())).float()


def retention_decay(H: int) -> torch.Tensor:
    """One constant decay per head for the retention workloads: 1 - 2^-(5 + h mod 4)
    (fp32, exact).  A synthetic choice spanning fast and slow heads."""
    return torch.tensor([1.0 - 2.0 ** -(5 + h % 4) for h in range(H)], dtype=torch.float32)


def make_problem(rule: str, B: int, T: int, H: int, dk: int, dv: int, *,
                 dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                 init_state: str = "zero", eps: float = 1e-6,
                 gla_gate: str = "softplus16", gdn_alpha: str = "sigmoid3",
                 name: str = "") -> Problem:
    """Generic generator used by all prefill workloads and by the tests.

    ``init_state``: ``"zero"`` (S0=None, z0=None), ``"abs"`` (S0=|N(0,1)|,
    z0=1 for ELU), ``"normal"`` (S0=N(0,1)*0.1, z0=1+|N(0,1)| for ELU).
    ``gla_gate``: ``"softplus16"`` (the workload recipe), ``"ones"`` (g=1: the
    Lightning accumulation S_t = S_{t-1} + k_t v_t^T) or ``"retnet"`` (one
    constant decay per head, 1 - 2^-(5 + h mod 4), on every key dim and token:
    retention S_t = gamma S_{t-1} + k_t v_t^T).
    ``gdn_alpha``: ``"sigmoid3"`` (the workload recipe) or ``"ones"`` (alpha=1:
    the plain delta rule).
    """
    assert rule in RULES
    gen = _gen(seed)
    q = _randn(gen, B, T, H, dk)
    k = _randn(gen, B, T, H, dk)
    v = _randn(gen, B, T, H, dv)
    g = beta = None
    if rule == "gla":
        k = k / math.sqrt(dk)
        src = _randn(gen, B, T, H, dk)
        if gla_gate == "softplus16":
            g = gla_gate_from(src)
        elif gla_gate == "ones":
            g = torch.ones(B, T, H, dk)
        elif gla_gate == "retnet":
            g = retention_decay(H).view(1, 1, H, 1).expand(B, T, H, dk).contiguous()
        else:
            raise ValueError(gla_gate)
    elif rule == "kda":
        q = _l2norm_last(q)
        k = _l2norm_last(k)
        g = kda_alpha_from(_randn(gen, B, T, H, dk))
        beta = gdn_beta_from(_randn(gen, B, T, H))
    elif rule == "gdn":
        q = _l2norm_last(q)
        k = _l2norm_last(k)
        a_src = _randn(gen, B, T, H)
        if gdn_alpha == "sigmoid3":
            g = gdn_alpha_from(a_src)
        elif gdn_alpha == "ones":
            g = torch.ones(B, T, H)
        else:
            raise ValueError(gdn_alpha)
        beta = gdn_beta_from(_randn(gen, B, T, H))
    S0 = z0 = None
    if init_state == "abs":
        S0 = _randn(gen, B, H, dk, dv).abs()
        if rule == "elu":
            z0 = torch.ones(B, H, dk)
    elif init_state == "normal":
        S0 = _randn(gen, B, H, dk, dv) * 0.1
        if rule == "elu":
            z0 = 1.0 + _randn(gen, B, H, dk).abs()
    elif init_state != "zero":
        raise ValueError(init_state)
    q, k, v = (x.to(dtype).contiguous() for x in (q, k, v))
    return Problem(rule, q, k, v, g, beta, S0, z0, eps, name or f"{rule}_B{B}T{T}H{H}_{dk}x{dv}")


# ---------------------------------------------------------------------------
# The five named workloads.
# ---------------------------------------------------------------------------

def elu_fp32_small(seed: int = 0) -> Problem:
    """Normalized ELU+1, fp32: B=1,H=1,T=256,dk=dv=32, zero S and z."""
    return make_problem("elu", 1, 256, 1, 32, 32, dtype=torch.float32, seed=seed,
                        name="elu_fp32_B1H1T256_d32")


def gla_prefill(B: int = 4, H: int = 8, T: int = 2048, seed: int = 0) -> Problem:
    """GLA prefill, bf16 q/k/v, d=128, zero state (B=4,H=8,T=2048 by default)."""
    return make_problem("gla", B, T, H, 128, 128, seed=seed, name=f"gla_B{B}H{H}T{T}_d128")


def elu_long(seed: int = 0, T: int = 32768) -> Problem:
    """Normalized ELU+1 at the pages' worked shape: B=1,H=16,N=32768,dk=128,dv=64."""
    return make_problem("elu", 1, T, 16, 128, 64, seed=seed, init_state="abs",
                        name=f"elu_B1H16T{T}_dk128_dv64")


def gdn_prefill(B: int = 2, H: int = 16, T: int = 8192, seed: int = 0) -> Problem:
    """Gated delta rule prefill, d=128, L2-normalised q/k, zero state."""
    return make_problem("gdn", B, T, H, 128, 128, seed=seed, name=f"gdn_B{B}H{H}T{T}_d128")


@dataclass
class DecodeWorkload:
    """Decode: one fp32 state and ``steps`` single-token inputs per rule."""

    S0: torch.Tensor                       # [N,H,dk,dv] fp32
    gla: list                              # per step: (q,k,v,g)
    gdn: list                              # per step: (q,k,v,alpha,beta)


def decode_state(N: int = 256, H: int = 16, dk: int = 128, dv: int = 128,
                 seed: int = 0) -> torch.Tensor:
    gen = _gen(seed)
    return _randn(gen, N, H, dk, dv) * 0.02


def decode_steps(rule: str, steps: int, N: int = 256, H: int = 16, dk: int = 128,
                 dv: int = 128, seed: int = 0) -> list:
    """Per-step decode inputs; q,k,v are [N,H,d] bf16 (one token per sequence).

    Each rule uses its own generator stream (seed+1 for GLA, seed+2 for the
    gated delta rule) so that the state draw (seed) is shared by both.
    """
    gen = _gen(seed + (1 if rule == "gla" else 2))
    out = []
    for _ in range(steps):
        q = _randn(gen, N, H, dk)
        k = _randn(gen, N, H, dk)
        v = _randn(gen, N, H, dv)
        if rule == "gla":
            k = k / math.sqrt(dk)
            g = gla_gate_from(_randn(gen, N, H, dk))
            out.append((q.bfloat16(), k.bfloat16(), v.bfloat16(), g))
        elif rule == "gdn":
            q = _l2norm_last(q)
            k = _l2norm_last(k)
            a = gdn_alpha_from(_randn(gen, N, H))
            b = gdn_beta_from(_randn(gen, N, H))
            out.append((q.bfloat16(), k.bfloat16(), v.bfloat16(), a, b))
        else:
            k_ = k
            out.append((q.bfloat16(), k_.bfloat16(), v.bfloat16()))
    return out


def decode_workload(steps: int = 64, N: int = 256, H: int = 16, seed: int = 0) -> DecodeWorkload:
    """Decode: state [256,16,128,128] fp32 ~ N(0,0.02); 64 GLA and 64 GDN steps."""
    return DecodeWorkload(decode_state(N, H, seed=seed),
                          decode_steps("gla", steps, N, H, seed=seed),
                          decode_steps("gdn", steps, N, H, seed=seed))
