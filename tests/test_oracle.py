"""Pins for the fp64 oracle: each check uses a formula or fact other than the
oracle's own recurrence, so that a dropped term, a wrong sign, a transposed
operand or a wrong gate index in ``oracle/la_oracle.c`` fails at least one.

Sources (page title, section):
  [LR]  "Linear / RNN 路线：砍 softmax，固定 state 替代 KV": §2.1 (ELU+1, the
        causal sum form), §2.2 (GLA), §2.4 (g = 1 is plain linear attention).
  [LS]  "线性注意力与 SSM：把整张关系表变成一条状态流": §02 (normalized form;
        hand count N*dphi*dv), GDN box (gated delta rule, residual reading).
  [SS]  "状态空间与线性注意力": 线性注意力 (epsilon in the denominator), State
        Space Duality (semiseparable products), Retention/Delta Rule, Delta-rule
        语义核 (worked example), KDA recurrent reference (decay before delta,
        current-token read, split test), 验证矩阵 (chunk boundaries, reset).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _feature(x):
    # ELU(x)+1 written as max(x,0) + exp(min(x,0)): equal to x+1 for x>0 and e^x
    # for x<=0 ([LR] §2.1), but not the same expression as the oracle's.
    return np.maximum(x, 0.0) + np.exp(np.minimum(x, 0.0))


def _rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


# ---------------------------------------------------------------------------
# ELU+1
# ---------------------------------------------------------------------------

def test_elu_matches_quadratic_causal_form():
    """[LR] §2.1 / [SS] 线性注意力: o_t = phi(q_t)^T(S0 + sum_{i<=t} phi(k_i) v_i^T)
    / (phi(q_t)^T(z0 + sum_{i<=t} phi(k_i)) + eps), evaluated as a masked
    T x T score matrix (no recurrence)."""
    B, T, H, dk, dv = 2, 23, 3, 5, 4
    q, k, v = _rand(B, T, H, dk), _rand(B, T, H, dk), _rand(B, T, H, dv)
    S0 = np.abs(_rand(B, H, dk, dv))
    z0 = 1.0 + np.abs(_rand(B, H, dk))
    eps = 0.3
    o, S, z = oracle.elu_fwd(q, k, v, S0, z0, eps)
    mask = np.tril(np.ones((T, T)))
    for b in range(B):
        for h in range(H):
            pq, pk = _feature(q[b, :, h]), _feature(k[b, :, h])
            A = (pq @ pk.T) * mask                       # [T,T] causal scores
            num = A @ v[b, :, h] + pq @ S0[b, h]
            den = A.sum(1) + pq @ z0[b, h] + eps
            np.testing.assert_allclose(o[b, :, h], num / den[:, None], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(S[b, h], S0[b, h] + pk.T @ v[b, :, h], rtol=1e-12)
            np.testing.assert_allclose(z[b, h], z0[b, h] + pk.sum(0), rtol=1e-12)


def test_elu_constant_values_closed_form():
    """All v_t = c, zero initial state: o_t = c * D_t / (D_t + eps) with
    D_t = sum_{i<=t} phi(q_t).phi(k_i); eps sits outside the dot product."""
    T, dk, dv = 17, 6, 3
    q, k = _rand(1, T, 1, dk), _rand(1, T, 1, dk)
    c = np.array([1.5, -2.0, 0.25])
    v = np.broadcast_to(c, (1, T, 1, dv)).copy()
    eps = 2.0
    o, _, _ = oracle.elu_fwd(q, k, v, None, None, eps)
    pq, pk = _feature(q[0, :, 0]), _feature(k[0, :, 0])
    D = np.array([(pq[t] * pk[: t + 1]).sum() for t in range(T)])
    np.testing.assert_allclose(o[0, :, 0], (D / (D + eps))[:, None] * c, rtol=1e-13)


def test_elu_feature_branches():
    """phi = ELU+1: exercises x>0, x=0 and x<0 through a single key dim."""
    x = np.array([-3.0, -0.5, 0.0, 0.5, 2.0])
    T = len(x)
    q = np.ones((1, T, 1, 1)) * 1e-9  # phi(q)=1+1e-9 ~ 1
    k = x.reshape(1, T, 1, 1)
    v = np.ones((1, T, 1, 1))
    _, _, z = oracle.elu_fwd(q, k, v, None, None, 0.0)
    expect = np.exp(-3.0) + np.exp(-0.5) + 1.0 + 1.5 + 3.0
    assert abs(z[0, 0, 0] - expect) < 1e-13


def test_elu_equals_gla_with_unit_gate_on_features():
    """Cross-rule: normalized ELU(q,k,v) = num/(den+eps) where [num | den] is
    GLA(g=1) run on (phi(q), phi(k), [v | 1]) with state [S0 | z0] ([LR] §2.1,
    §2.4: with no gate the state is a plain sum)."""
    B, T, H, dk, dv = 1, 19, 2, 4, 3
    q, k, v = _rand(B, T, H, dk), _rand(B, T, H, dk), _rand(B, T, H, dv)
    S0 = np.abs(_rand(B, H, dk, dv))
    z0 = 1.0 + np.abs(_rand(B, H, dk))
    eps = 0.1
    o_e, S_e, z_e = oracle.elu_fwd(q, k, v, S0, z0, eps)
    v1 = np.concatenate([v, np.ones((B, T, H, 1))], -1)
    Sz0 = np.concatenate([S0, z0[..., None]], -1)
    o_g, S_g = oracle.gla_fwd(_feature(q), _feature(k), v1, np.ones((B, T, H, dk)), Sz0)
    np.testing.assert_allclose(o_e, o_g[..., :dv] / (o_g[..., dv:] + eps), rtol=1e-12)
    np.testing.assert_allclose(S_e, S_g[..., :dv], rtol=1e-12)
    np.testing.assert_allclose(z_e, S_g[..., dv], rtol=1e-12)


# ---------------------------------------------------------------------------
# GLA
# ---------------------------------------------------------------------------

def test_gla_matches_explicit_gate_products():
    """[LR] §2.2 + [SS] State Space Duality: o_t = sum_{i<=t} sum_d q_td k_id
    (prod_{s=i+1..t} g_sd) v_i + sum_d q_td (prod_{s<=t} g_sd) S0[d,:]."""
    B, T, H, dk, dv = 1, 13, 2, 4, 3
    q, k, v = _rand(B, T, H, dk), _rand(B, T, H, dk), _rand(B, T, H, dv)
    g = rng.uniform(0.3, 1.0, (B, T, H, dk))
    S0 = _rand(B, H, dk, dv)
    o, S = oracle.gla_fwd(q, k, v, g, S0)
    for h in range(H):
        for t in range(T):
            acc = np.zeros(dv)
            for i in range(t + 1):
                decay = np.prod(g[0, i + 1: t + 1, h], axis=0)  # empty product = 1
                acc += (q[0, t, h] * k[0, i, h] * decay).sum() * v[0, i, h]
            acc += (q[0, t, h] * np.prod(g[0, : t + 1, h], axis=0)) @ S0[0, h]
            np.testing.assert_allclose(o[0, t, h], acc, rtol=1e-11, atol=1e-12)
        Sx = np.prod(g[0, :, h], axis=0)[:, None] * S0[0, h]
        for i in range(T):
            Sx += np.outer(k[0, i, h] * np.prod(g[0, i + 1:, h], axis=0), v[0, i, h])
        np.testing.assert_allclose(S[0, h], Sx, rtol=1e-11, atol=1e-12)


def test_gla_unit_gate_is_unnormalised_linear_attention():
    """g = 1 ([LR] §2.4, [LS] complexity table): o = (Q K^T * M) V + Q S0."""
    T, dk, dv = 31, 8, 5
    q, k, v = _rand(1, T, 1, dk), _rand(1, T, 1, dk), _rand(1, T, 1, dv)
    S0 = _rand(1, 1, dk, dv)
    o, S = oracle.gla_fwd(q, k, v, np.ones((1, T, 1, dk)), S0)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    expect = np.tril(Q @ K.T) @ V + Q @ S0[0, 0]
    np.testing.assert_allclose(o[0, :, 0], expect, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], S0[0, 0] + K.T @ V, rtol=1e-12)


def test_gla_constant_decay_is_retention_closed_form():
    """[SS] Retention: S_t = gamma S_{t-1} + k_t v_t^T with one constant gamma,
    so S_t = gamma^(t+1) S0 + sum_{i<=t} gamma^(t-i) k_i v_i^T and the outputs are
    the decayed causal score matrix (gamma^(t-i) (q_t . k_i)) applied to V plus
    gamma^(t+1) S0^T q_t; the GLA recurrence with that gamma on every key dim."""
    T, dk, dv, gam = 19, 4, 3, 0.8125
    q, k, v = _rand(1, T, 1, dk), _rand(1, T, 1, dk), _rand(1, T, 1, dv)
    S0 = _rand(1, 1, dk, dv)
    o, S = oracle.gla_fwd(q, k, v, np.full((1, T, 1, dk), gam), S0)
    t_idx = np.arange(T)
    D = np.where(t_idx[:, None] >= t_idx[None, :], gam ** (t_idx[:, None] - t_idx[None, :]), 0.0)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    ref = ((Q @ K.T) * D) @ V + (gam ** (t_idx + 1))[:, None] * (Q @ S0[0, 0])
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=1e-11, atol=1e-12)
    S_ref = gam ** T * S0[0, 0] + (K * (gam ** (T - 1 - t_idx))[:, None]).T @ V
    np.testing.assert_allclose(S[0, 0], S_ref, rtol=1e-11, atol=1e-12)


def test_gla_gate_scales_rows_of_state():
    """[LR] §2.2: g_t[i] multiplies row i (a key dim) of S; v = 0 isolates it."""
    dk, dv = 3, 2
    S0 = _rand(1, 1, dk, dv)
    g = np.array([0.5, 0.25, 0.9]).reshape(1, 1, 1, dk)
    _, S = oracle.gla_fwd(np.zeros((1, 1, 1, dk)), np.zeros((1, 1, 1, dk)),
                          np.zeros((1, 1, 1, dv)), g, S0)
    np.testing.assert_allclose(S[0, 0], S0[0, 0] * g[0, 0, 0][:, None], rtol=0, atol=0)


# ---------------------------------------------------------------------------
# Gated delta rule
# ---------------------------------------------------------------------------

def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_gdn_matches_transition_matrix_products():
    """[LS] GDN box in dk x dv orientation: S_t = (prod_s A_s) S0 +
    sum_i (prod_{s>i} A_s) beta_i k_i v_i^T with dense A_s = alpha_s (I - beta_s
    k_s k_s^T); o_t = S_t^T q_t."""
    T, dk, dv = 9, 4, 3
    q, k, v = _rand(1, T, 1, dk), _unit(_rand(1, T, 1, dk)), _rand(1, T, 1, dv)
    a = rng.uniform(0.5, 1.0, (1, T, 1))
    be = rng.uniform(0.1, 1.0, (1, T, 1))
    S0 = _rand(1, 1, dk, dv)
    o, S = oracle.gdn_fwd(q, k, v, a, be, S0)
    A = [a[0, s, 0] * (np.eye(dk) - be[0, s, 0] * np.outer(k[0, s, 0], k[0, s, 0]))
         for s in range(T)]

    def prod(lo, hi):  # A_hi ... A_lo (later tokens on the left)
        M = np.eye(dk)
        for s in range(lo, hi + 1):
            M = A[s] @ M
        return M

    for t in range(T):
        St = prod(0, t) @ S0[0, 0]
        for i in range(t + 1):
            St = St + prod(i + 1, t) @ np.outer(be[0, i, 0] * k[0, i, 0], v[0, i, 0])
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-11, atol=1e-12)


def test_gdn_unit_alpha_is_delta_rule_products():
    """[SS] Retention/Delta Rule: with alpha = 1 the gated rule is the delta rule
    S_t = S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T, i.e. a product of the
    rank-one corrections (I - beta_s k_s k_s^T) applied to S0 plus the written
    values, evaluated here as dense products (no recurrence)."""
    T, dk, dv = 10, 5, 3
    q, k, v = _rand(1, T, 1, dk), _unit(_rand(1, T, 1, dk)), _rand(1, T, 1, dv)
    be = rng.uniform(0.1, 1.0, (1, T, 1))
    S0 = _rand(1, 1, dk, dv)
    o, S = oracle.gdn_fwd(q, k, v, np.ones((1, T, 1)), be, S0)
    E = [np.eye(dk) - be[0, s, 0] * np.outer(k[0, s, 0], k[0, s, 0]) for s in range(T)]
    for t in range(T):
        St = S0[0, 0].copy()
        for s in range(t + 1):
            St = E[s] @ St
        for i in range(t + 1):
            M = np.eye(dk)
            for s in range(i + 1, t + 1):
                M = E[s] @ M
            St = St + M @ np.outer(be[0, i, 0] * k[0, i, 0], v[0, i, 0])
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-11, atol=1e-12)


def test_kda_matches_transition_matrix_products():
    """[SS] KDA: decay, then the delta write on the decayed state, i.e.
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T, evaluated
    as dense transition products (an oracle that wrote before decaying, or
    decayed the written term, fails this)."""
    T, dk, dv = 9, 4, 3
    q, k, v = _rand(1, T, 1, dk), _unit(_rand(1, T, 1, dk)), _rand(1, T, 1, dv)
    a = rng.uniform(0.2, 1.0, (1, T, 1, dk))
    be = rng.uniform(0.1, 1.0, (1, T, 1))
    S0 = _rand(1, 1, dk, dv)
    o, S = oracle.kda_fwd(q, k, v, a, be, S0)
    A = [(np.eye(dk) - be[0, s, 0] * np.outer(k[0, s, 0], k[0, s, 0])) @ np.diag(a[0, s, 0])
         for s in range(T)]

    def prod(lo, hi):  # A_hi ... A_lo
        M = np.eye(dk)
        for s in range(lo, hi + 1):
            M = A[s] @ M
        return M

    for t in range(T):
        St = prod(0, t) @ S0[0, 0]
        for i in range(t + 1):
            St = St + prod(i + 1, t) @ np.outer(be[0, i, 0] * k[0, i, 0], v[0, i, 0])
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-11, atol=1e-12)


def test_kda_with_one_retention_per_token_is_gated_delta_rule():
    """alpha_t equal on every key channel: Diag(alpha_t) = alpha_t I commutes with
    I - beta k k^T, so KDA is the gated delta rule ([SS] KDA vs [LS] GDN box)."""
    B, T, H, dk, dv = 2, 17, 2, 5, 3
    q, k, v = _rand(B, T, H, dk), _unit(_rand(B, T, H, dk)), _rand(B, T, H, dv)
    a = rng.uniform(0.3, 1.0, (B, T, H))
    be = rng.uniform(0.0, 1.0, (B, T, H))
    S0 = _rand(B, H, dk, dv)
    o1, S1 = oracle.kda_fwd(q, k, v, np.repeat(a[..., None], dk, axis=-1), be, S0)
    o2, S2 = oracle.gdn_fwd(q, k, v, a, be, S0)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S1, S2, rtol=1e-12, atol=1e-13)


def test_kda_zero_beta_is_channelwise_decay():
    """beta = 0: S_t = Diag(prod_{s<=t} alpha_s) S0 and o_t = S_t^T q_t."""
    T, dk, dv = 10, 4, 3
    q, k, v = _rand(1, T, 1, dk), _rand(1, T, 1, dk), _rand(1, T, 1, dv)
    a = rng.uniform(0.5, 1.0, (1, T, 1, dk))
    S0 = _rand(1, 1, dk, dv)
    o, S = oracle.kda_fwd(q, k, v, a, np.zeros((1, T, 1)), S0)
    cum = np.cumprod(a[0, :, 0], axis=0)                     # [T, dk]
    ref = np.einsum("td,dj,td->tj", q[0, :, 0], S0[0, 0], cum)
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=1e-12)
    np.testing.assert_allclose(S[0, 0], cum[-1][:, None] * S0[0, 0], rtol=1e-12)


def test_kda_workload_decay_is_bounded():
    """The bounded log-decay keeps every retention in (e^-5, 1) ([SS] 有界 log-decay)."""
    p = workloads.make_problem("kda", 2, 300, 3, 16, 8, seed=1)
    assert float(p.g.min()) > math.exp(-5.0) and float(p.g.max()) < 1.0


def test_gdn_zero_beta_is_pure_decay():
    """beta = 0: S_t = (prod alpha) S0 and o_t = (prod_{s<=t} alpha_s) S0^T q_t."""
    T, dk, dv = 12, 5, 4
    q, k, v = _rand(1, T, 1, dk), _rand(1, T, 1, dk), _rand(1, T, 1, dv)
    a = rng.uniform(0.6, 1.0, (1, T, 1))
    S0 = _rand(1, 1, dk, dv)
    o, S = oracle.gdn_fwd(q, k, v, a, np.zeros((1, T, 1)), S0)
    cum = np.cumprod(a[0, :, 0])
    np.testing.assert_allclose(o[0, :, 0], cum[:, None] * (q[0, :, 0] @ S0[0, 0]), rtol=1e-12)
    np.testing.assert_allclose(S[0, 0], cum[-1] * S0[0, 0], rtol=1e-12)


def test_gdn_worked_delta_example_from_pages():
    """[SS] Delta-rule 语义核: keys = I2, values [[2,-1],[.5,3]], rate 1, zero
    state: reads before each write are 0 and keys @ state = values.  With
    alpha = 1 the gated rule is this delta rule.  Read-after-write with q_t = k_t
    returns v_t (orthonormal keys)."""
    with open(os.path.join(GOLDEN, "delta_worked_example.json")) as f:
        ex = json.load(f)
    K = np.array(ex["keys"])
    V = np.array(ex["values"])
    T = K.shape[0]
    k = K.reshape(1, T, 1, 2)
    v = V.reshape(1, T, 1, 2)
    a = np.array(ex["alpha"]).reshape(1, T, 1)
    be = np.array(ex["beta"]).reshape(1, T, 1)
    o, S = oracle.gdn_fwd(k, k, v, a, be)
    assert list(S[0, 0].shape) == ex["state_shape"]
    np.testing.assert_allclose(K @ S[0, 0], np.array(ex["keys_at_final_state"]), atol=1e-15)
    np.testing.assert_allclose(o[0, :, 0], V, atol=1e-15)
    # reads before write: S_{t-1}^T k_t from the prefix run (S_{-1} = 0)
    reads = [np.zeros(2)]
    for t in range(1, T):
        _, St = oracle.gdn_fwd(k[:, :t], k[:, :t], v[:, :t], a[:, :t], be[:, :t])
        reads.append(St[0, 0].T @ K[t])
    np.testing.assert_allclose(np.array(reads), np.array(ex["reads_before_write"]), atol=1e-15)


def test_gdn_unit_beta_writes_value_exactly():
    """beta = 1 and |k| = 1: S_t^T k_t = alpha (S^T k - S^T k) + v_t = v_t for any
    alpha and prior state ([LS] GDN box, residual reading)."""
    T, dk, dv = 15, 6, 4
    k = _unit(_rand(1, T, 1, dk))
    v = _rand(1, T, 1, dv)
    a = rng.uniform(0.3, 1.0, (1, T, 1))
    S0 = _rand(1, 1, dk, dv)
    o, _ = oracle.gdn_fwd(k, k, v, a, np.ones((1, T, 1)), S0)  # q_t = k_t
    np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=1e-12, atol=1e-12)


def test_gdn_equals_decay_then_delta_form():
    """[SS] KDA: decay the state, then write the residual of the *decayed*
    state's prediction, then read with the current query.  With the per-channel
    retention set to the scalar alpha_t on every channel this is the gated
    delta rule (scalar alpha commutes with I - beta k k^T)."""
    T, dk, dv = 11, 4, 3
    q, k, v = _rand(1, T, 1, dk), _unit(_rand(1, T, 1, dk)), _rand(1, T, 1, dv)
    a = rng.uniform(0.4, 1.0, (1, T, 1))
    be = rng.uniform(0.0, 1.0, (1, T, 1))
    o, S = oracle.gdn_fwd(q, k, v, a, be)
    St = np.zeros((dk, dv))
    outs = []
    for t in range(T):
        decayed = np.full(dk, a[0, t, 0])[:, None] * St
        pred = k[0, t, 0] @ decayed
        St = decayed + be[0, t, 0] * np.outer(k[0, t, 0], v[0, t, 0] - pred)
        outs.append(St.T @ q[0, t, 0])
    np.testing.assert_allclose(o[0, :, 0], np.array(outs), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Properties shared by all rules
# ---------------------------------------------------------------------------

def _run(rule, q, k, v, g, be, S0, z0):
    if rule == "elu":
        return oracle.elu_fwd(q, k, v, S0, z0, 1e-6)
    if rule == "gla":
        o, S = oracle.gla_fwd(q, k, v, g, S0)
        return o, S, None
    if rule == "kda":
        o, S = oracle.kda_fwd(q, k, v, g, be, S0)
        return o, S, None
    o, S = oracle.gdn_fwd(q, k, v, g, be, S0)
    return o, S, None


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn", "kda"])
@pytest.mark.parametrize("tau", [0, 1, 7, 20, 29])
def test_split_invariance_bitwise(rule, tau):
    """[SS] selective scan / KDA recurrent reference / 验证矩阵 (chunk boundary):
    scanning [0,tau), carrying the state and scanning [tau,T) equals the whole
    scan; the oracle does the same operations in the same order, so exactly."""
    p = workloads.make_problem(rule, 2, 29, 2, 8, 6, dtype=torch.bfloat16, seed=3,
                               init_state="normal")
    q, k, v = p.q.double().numpy(), p.k.double().numpy(), p.v.double().numpy()
    g = None if p.g is None else p.g.double().numpy()
    be = None if p.beta is None else p.beta.double().numpy()
    S0 = p.S0.double().numpy()
    z0 = None if p.z0 is None else p.z0.double().numpy()
    sl = lambda x, a, b: None if x is None else x[:, a:b]
    o, S, z = _run(rule, q, k, v, g, be, S0, z0)
    o1, S1, z1 = _run(rule, q[:, :tau], k[:, :tau], v[:, :tau], sl(g, 0, tau), sl(be, 0, tau), S0, z0)
    o2, S2, z2 = _run(rule, q[:, tau:], k[:, tau:], v[:, tau:], sl(g, tau, None), sl(be, tau, None), S1, z1)
    assert np.array_equal(np.concatenate([o1, o2], 1), o)
    assert np.array_equal(S2, S)
    if z is not None:
        assert np.array_equal(z2, z)


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn", "kda"])
def test_sequences_are_independent(rule):
    """[SS] 验证矩阵 (reset: a batched run equals per-sample runs)."""
    p = workloads.make_problem(rule, 2, 10, 3, 4, 4, seed=5, init_state="normal")
    o, S, z = oracle.fwd(p)
    for b in range(2):
        for h in range(3):
            sub = workloads.Problem(
                rule, p.q[b:b + 1, :, h:h + 1], p.k[b:b + 1, :, h:h + 1], p.v[b:b + 1, :, h:h + 1],
                None if p.g is None else p.g[b:b + 1, :, h:h + 1],
                None if p.beta is None else p.beta[b:b + 1, :, h:h + 1],
                p.S0[b:b + 1, h:h + 1], None if p.z0 is None else p.z0[b:b + 1, h:h + 1])
            o1, S1, z1 = oracle.fwd(sub)
            assert np.array_equal(o1[0, :, 0], o[b, :, h])
            assert np.array_equal(S1[0, 0], S[b, h])


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn", "kda"])
def test_step_is_recurrence_at_T1(rule):
    """A decode step is one token of the recurrence: T steps of ``step`` equal
    one ``fwd`` over T tokens."""
    p = workloads.make_problem(rule, 1, 6, 2, 4, 3, seed=9, init_state="normal")
    o, S, z = oracle.fwd(p)
    St = p.S0.double().numpy()
    zt = None if p.z0 is None else p.z0.double().numpy()
    for t in range(6):
        g = None if p.g is None else p.g[:, t]
        be = None if p.beta is None else p.beta[:, t]
        ot, St, zt = oracle.step(rule, p.q[:, t], p.k[:, t], p.v[:, t], St, zt, g, be, p.eps)
        assert np.array_equal(ot, o[:, t])
    assert np.array_equal(St, S)


def test_zero_length_returns_initial_state():
    p = workloads.make_problem("gdn", 1, 0, 2, 4, 4, seed=1, init_state="normal")
    o, S, _ = oracle.fwd(p)
    assert o.shape == (1, 0, 2, 4)
    assert np.array_equal(S, p.S0.double().numpy())


# ---------------------------------------------------------------------------
# Output RMS normalisation (Lightning's o_t = Norm(q_t^T S_t), page "Linear / RNN
# 路线" §2.4; K3's head-wise RMSNorm of the recurrent output, page "状态空间与线性
# 注意力", KDA section).  The pages name the norm; these pins fix what it does.
# ---------------------------------------------------------------------------

def test_rmsnorm_worked_row_by_hand():
    """x = (3, 4, 0, 0): mean square 25/4, root 2.5, so y = (1.2, 1.6, 0, 0)."""
    y = oracle.head_rmsnorm(np.array([3.0, 4.0, 0.0, 0.0]), eps=0.0)
    np.testing.assert_allclose(y, [1.2, 1.6, 0.0, 0.0], rtol=0, atol=1e-15)


def test_rmsnorm_unit_rows_are_fixed_points_and_weight_scales_channels():
    """Rows of +-1 already have mean square 1: unchanged without a weight, and
    multiplied channel by channel by the weight."""
    rng = np.random.default_rng(0)
    x = np.where(rng.random((5, 3, 64)) < 0.5, -1.0, 1.0)
    np.testing.assert_array_equal(oracle.head_rmsnorm(x, eps=0.0), x)
    w = rng.normal(size=64)
    np.testing.assert_allclose(oracle.head_rmsnorm(x, w, eps=0.0), x * w, rtol=1e-15, atol=0)


def test_rmsnorm_constant_row_closed_form():
    """x = c * 1: every entry becomes c / sqrt(c^2 + eps)."""
    for c, eps in ((-3.0, 0.5), (1e-3, 1e-6), (250.0, 1e-6)):
        y = oracle.head_rmsnorm(np.full((2, 32), c), eps=eps)
        np.testing.assert_allclose(y, c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rmsnorm_is_scale_invariant_without_eps():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(4, 2, 128))
    y = oracle.head_rmsnorm(x, eps=0.0)
    for lam in (1e-3, 7.5, 1e4):
        np.testing.assert_allclose(oracle.head_rmsnorm(lam * x, eps=0.0), y, rtol=1e-13, atol=1e-15)
    # and every output row has mean square one
    np.testing.assert_allclose((y * y).mean(axis=-1), 1.0, rtol=1e-13)


def test_rmsnorm_normalises_each_row_on_its_own():
    """Rows that are multiples of one row (per head and per token, at very
    different scales) all normalise to the same row: the mean is taken over the
    dv values of each row, not over heads or tokens."""
    rng = np.random.default_rng(2)
    base = rng.normal(size=64)
    scales = np.array([[1.0, 10.0, 0.01], [3.0, 1e3, 0.5]])   # [tokens, heads]
    x = scales[:, :, None] * base
    y = oracle.head_rmsnorm(x, eps=0.0)
    want = oracle.head_rmsnorm(base[None], eps=0.0)[0]
    for t in range(2):
        for h in range(3):
            np.testing.assert_allclose(y[t, h], want, rtol=1e-13)


def test_rmsnorm_zero_row_with_eps_stays_zero():
    y = oracle.head_rmsnorm(np.zeros((3, 32)), w=np.arange(32.0), eps=1e-6)
    np.testing.assert_array_equal(y, 0.0)
