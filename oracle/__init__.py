"""Oracle: plain fp64 CPU per-token recurrence for the causal linear-attention
forward (normalized ELU+1, GLA, gated delta rule).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``gated_delta_rule_attn_b200``) and neither imports the
other.

The arithmetic lives in ``la_oracle.c`` (see its header for the passages each
rule follows).  This wrapper only converts arrays to contiguous fp64 (an exact
upcast of the bf16/fp32 inputs) and calls the C functions.

Pins: every function here is checked in ``tests/test_oracle.py`` against
brute-force quadratic / transition-product forms, closed forms, the pages'
worked delta-rule example and split invariance; ``head_rmsnorm`` against fixed
points, scale invariance, a constant-row closed form and per-row independence.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        # LA_ORACLE_LIB lets the mutation test load a deliberately broken copy.
        path = os.environ.get("LA_ORACLE_LIB") or _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        lib.oracle_elu.argtypes = [I, I, I, I, I, P, P, P, P, P, ctypes.c_double, P, P, P]
        lib.oracle_gla.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P]
        lib.oracle_gdn.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_kda.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.oracle_head_rmsnorm.argtypes = [I, I, P, P, ctypes.c_double, P]
        lib.oracle_head_rmsnorm.restype = None
        for f in (lib.oracle_elu, lib.oracle_gla, lib.oracle_gdn):
            f.restype = None
        _lib = lib
    return _lib


def _f64(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    try:  # torch tensor (bf16 has no numpy dtype: upcast in torch, exactly)
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().cpu().double().numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _shape(q, v):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    assert v.shape[:3] == (B, T, H)
    return B, T, H, dk, dv


def elu_fwd(q, k, v, S0=None, z0=None, eps: float = 1e-6):
    """Normalized ELU+1 linear attention. Returns (o, S, z) as fp64 arrays."""
    q, k, v, S0, z0 = map(_f64, (q, k, v, S0, z0))
    B, T, H, dk, dv = _shape(q, v)
    o = np.empty((B, T, H, dv))
    S = np.empty((B, H, dk, dv))
    z = np.empty((B, H, dk))
    _load().oracle_elu(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(S0), _ptr(z0),
                       float(eps), _ptr(o), _ptr(S), _ptr(z))
    return o, S, z


def gla_fwd(q, k, v, g, S0=None):
    """GLA: S_t = diag(g_t) S_{t-1} + k_t v_t^T, o_t = S_t^T q_t. Returns (o, S)."""
    q, k, v, g, S0 = map(_f64, (q, k, v, g, S0))
    B, T, H, dk, dv = _shape(q, v)
    assert g.shape == (B, T, H, dk)
    o = np.empty((B, T, H, dv))
    S = np.empty((B, H, dk, dv))
    _load().oracle_gla(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(S0),
                       _ptr(o), _ptr(S))
    return o, S


def gdn_fwd(q, k, v, alpha, beta, S0=None):
    """Gated delta rule, dk x dv state. Returns (o, S)."""
    q, k, v, alpha, beta, S0 = map(_f64, (q, k, v, alpha, beta, S0))
    B, T, H, dk, dv = _shape(q, v)
    assert alpha.shape == (B, T, H) and beta.shape == (B, T, H)
    o = np.empty((B, T, H, dv))
    S = np.empty((B, H, dk, dv))
    _load().oracle_gdn(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                       _ptr(S0), _ptr(o), _ptr(S))
    return o, S


def kda_fwd(q, k, v, alpha, beta, S0=None):
    """KDA (per-key-channel retention alpha [B,T,H,dk] with the delta rule), dk x dv
    state. Returns (o, S)."""
    q, k, v, alpha, beta, S0 = map(_f64, (q, k, v, alpha, beta, S0))
    B, T, H, dk, dv = _shape(q, v)
    assert alpha.shape == (B, T, H, dk) and beta.shape == (B, T, H)
    o = np.empty((B, T, H, dv))
    S = np.empty((B, H, dk, dv))
    _load().oracle_kda(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                       _ptr(S0), _ptr(o), _ptr(S))
    return o, S


def fwd(problem):
    """Run the oracle on a ``workloads.Problem``; returns (o, S, z-or-None)."""
    p = problem
    if p.rule == "elu":
        return elu_fwd(p.q, p.k, p.v, p.S0, p.z0, p.eps)
    if p.rule == "gla":
        o, S = gla_fwd(p.q, p.k, p.v, p.g, p.S0)
        return o, S, None
    if p.rule == "gdn":
        o, S = gdn_fwd(p.q, p.k, p.v, p.g, p.beta, p.S0)
        return o, S, None
    if p.rule == "kda":
        o, S = kda_fwd(p.q, p.k, p.v, p.g, p.beta, p.S0)
        return o, S, None
    raise ValueError(p.rule)


def head_rmsnorm(o, w=None, eps: float = 1e-6) -> np.ndarray:
    """Head-wise RMS normalisation of an output array [..., dv] over its last
    axis (Lightning's o_t = Norm(q_t^T S_t), "Linear / RNN 路线" §2.4; K3's
    head-wise RMSNorm, "状态空间与线性注意力" KDA section): each row x becomes
    w * x / sqrt(mean(x^2) + eps), w None = ones.  Returns a new fp64 array."""
    x = _f64(o)
    dv = x.shape[-1]
    rows = int(np.prod(x.shape[:-1])) if x.ndim > 1 else 1
    y = np.empty_like(x)
    wd = _f64(w)
    if wd is not None and wd.shape != (dv,):
        raise ValueError("w must have shape [dv]")
    _load().oracle_head_rmsnorm(rows, dv, _ptr(x), _ptr(wd), float(eps), _ptr(y))
    return y


def step(rule: str, q, k, v, S, z=None, g=None, beta=None, eps: float = 1e-6):
    """One decode step = the recurrence at T=1. q,k,v are [N,H,d]; S is [N,H,dk,dv].

    Returns (o [N,H,dv], S', z' or None).
    """
    q1, k1, v1 = (_f64(x)[:, None] for x in (q, k, v))
    if rule == "elu":
        o, S2, z2 = elu_fwd(q1, k1, v1, S, z, eps)
        return o[:, 0], S2, z2
    if rule == "gla":
        o, S2 = gla_fwd(q1, k1, v1, _f64(g)[:, None], S)
        return o[:, 0], S2, None
    if rule == "gdn":
        o, S2 = gdn_fwd(q1, k1, v1, _f64(g)[:, None], _f64(beta)[:, None], S)
        return o[:, 0], S2, None
    if rule == "kda":
        o, S2 = kda_fwd(q1, k1, v1, _f64(g)[:, None], _f64(beta)[:, None], S)
        return o[:, 0], S2, None
    raise ValueError(rule)


def num_threads() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    if n:
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
