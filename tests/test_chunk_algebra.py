"""The chunk algebra the tensor-core kernels evaluate, checked in fp64 against
the oracle's per-token recurrence before any rounding enters.

These are test-only NumPy restatements of the chunked forms (64-token chunks,
the state carried across chunks), written from the derivations in the kernel
headers, not from the kernels:

* gated delta rule (WY / UT form, page "线性注意力与 SSM", GDN box): with
  gamma the cumulative alpha inside a chunk, A = diag(beta)(K K^T o Gamma o
  strict-lower), T = (I + A)^-1, W = T diag(beta)(V - diag(gamma) K S0),
  O = diag(gamma) Q S0 + ((Q K^T) o Gamma o M) W,
  S <- gamma_C S0 + K^T diag(gamma_C / gamma) W;
* KDA (page "状态空间与线性注意力", KDA：逐通道遗忘与误差写入) with per-channel
  cumulative retention Gamma, and the pairwise factors Gamma_t / Gamma_i formed
  as the KDA prep kernel forms them: per 16-token sub-chunk, relative to its
  middle token, from products of alpha and one reciprocal, with the
  cross-sub-chunk factors as products of sub-chunk products.

A dropped term, a wrong reference token or a transposed operand in these
derivations makes the chunked result differ from the recurrence by far more
than fp64 rounding.
"""
import numpy as np
import pytest

import oracle
import workloads

C, SUB = 64, 16


def _f64(x):
    return None if x is None else x.double().numpy()


def _chunk(x, b, h, c0, n, fill, width):
    out = np.full((C, width), fill, dtype=np.float64)
    out[:n] = x[b, c0:c0 + n, h]
    return out


def gdn_chunked(q, k, v, alpha, beta, S0):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_out = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, C):
                n = min(C, T - c0)
                Q, K, V = (_chunk(x, b, h, c0, n, 0.0, x.shape[-1]) for x in (q, k, v))
                al = _chunk(alpha[..., None], b, h, c0, n, 1.0, 1)[:, 0]
                be = _chunk(beta[..., None], b, h, c0, n, 0.0, 1)[:, 0]
                gam = np.cumprod(al)
                Gam = np.tril(gam[:, None] / gam[None, :])
                A = be[:, None] * np.tril(K @ K.T * Gam, -1)
                Tm = np.linalg.inv(np.eye(C) + A)
                W = Tm @ (be[:, None] * (V - gam[:, None] * (K @ S)))
                O = gam[:, None] * (Q @ S) + (Q @ K.T * Gam) @ W
                S = gam[-1] * S + K.T @ ((gam[-1] / gam)[:, None] * W)
                o[b, c0:c0 + n, h] = O[:n]
            S_out[b, h] = S
    return o, S_out


def kda_subchunk_factors(al):
    """For one chunk of alphas [C, dk] (1 past the end): G_t = Gamma_t /
    Gamma_{m(t)} with m(t) the middle (8th) token of t's 16-token sub-chunk,
    H_t = 1 / G_t, and per sub-chunk the alpha products up to and including its
    middle token (D) and after it (U).  Products and one reciprocal only."""
    ns, dk = C // SUB, al.shape[1]
    G = np.zeros((C, dk))
    Hh = np.zeros((C, dk))
    D = np.zeros((ns, dk))
    U = np.zeros((ns, dk))
    for s in range(ns):
        a = al[s * SUB:(s + 1) * SUB]
        suf = np.ones(dk)
        for j in range(7, -1, -1):          # G = 1 / prod_{j+1..7} alpha
            Hh[s * SUB + j] = suf
            G[s * SUB + j] = 1.0 / suf
            suf = suf * a[j]
        D[s] = suf
        run = np.ones(dk)
        for j in range(8, SUB):             # G = prod_{8..j} alpha
            run = run * a[j]
            G[s * SUB + j] = run
            Hh[s * SUB + j] = 1.0 / run
        U[s] = run
    return G, Hh, D, U


def kda_chunked(q, k, v, alpha, beta, S0):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    ns = C // SUB
    sub = np.arange(C) // SUB
    o = np.zeros((B, T, H, dv))
    S_out = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, C):
                n = min(C, T - c0)
                Q, K, V = (_chunk(x, b, h, c0, n, 0.0, x.shape[-1]) for x in (q, k, v))
                al = _chunk(alpha, b, h, c0, n, 1.0, dk)
                be = _chunk(beta[..., None], b, h, c0, n, 0.0, 1)[:, 0]
                G, Hh, D, U = kda_subchunk_factors(al)
                L = D * U
                gmid = np.array([np.prod(L[:s], axis=0) * D[s] for s in range(ns)])    # Gamma at m_s
                cmid = np.array([U[s] * np.prod(L[s + 1:], axis=0) for s in range(ns)])  # Gamma_C / that
                Qp, Kp = Q * G * gmid[sub], K * G * gmid[sub]
                Kc = K * Hh * cmid[sub]
                P = np.zeros((C, C))
                A = np.zeros((C, C))
                for a in range(ns):
                    Kr = np.zeros((C, dk))
                    for i in range(C):
                        s = sub[i]
                        if s < a:
                            Kr[i] = K[i] * Hh[i] * U[s] * np.prod(L[s + 1:a], axis=0) * D[a]
                        elif s == a:
                            Kr[i] = K[i] * Hh[i]
                    SP, SA = (Q * G) @ Kr.T, (K * G) @ Kr.T
                    for t in np.where(sub == a)[0]:
                        P[t, :t + 1] = SP[t, :t + 1]
                        A[t, :t] = be[t] * SA[t, :t]
                Tm = np.linalg.inv(np.eye(C) + A)
                W = Tm @ (be[:, None] * (V - Kp @ S))
                O = Qp @ S + P @ W
                S = np.prod(L, axis=0)[:, None] * S + Kc.T @ W
                o[b, c0:c0 + n, h] = O[:n]
            S_out[b, h] = S
    return o, S_out


def _rel(x, ref):
    return float(np.abs(x - ref).max() / np.abs(ref).max())


@pytest.mark.parametrize("T", [1, 37, 64, 130, 200])
def test_gdn_chunk_form_equals_recurrence(T):
    p = workloads.make_problem("gdn", 2, T, 2, 16, 8, seed=T, init_state="normal")
    ro, rS, _ = oracle.fwd(p)
    o, S = gdn_chunked(*(_f64(x) for x in (p.q, p.k, p.v, p.g, p.beta, p.S0)))
    assert _rel(o, ro) < 1e-12 and _rel(S, rS) < 1e-12


@pytest.mark.parametrize("T", [1, 16, 37, 64, 130, 200])
def test_kda_chunk_form_with_subchunk_factors_equals_recurrence(T):
    p = workloads.make_problem("kda", 2, T, 2, 16, 8, seed=T + 1, init_state="normal")
    ro, rS, _ = oracle.fwd(p)
    o, S = kda_chunked(*(_f64(x) for x in (p.q, p.k, p.v, p.g, p.beta, p.S0)))
    assert _rel(o, ro) < 1e-12 and _rel(S, rS) < 1e-12


def test_kda_subchunk_factors_stay_in_range_on_the_pages_bound():
    """With log alpha > -5 (the page's bounded log-decay) every G and H is within
    2^(+-58): 7 tokens on one side of the middle, 8 on the other, each at most
    e^5 = 2^7.2."""
    rng = np.random.default_rng(0)
    al = np.exp(-5.0 * rng.uniform(0.999, 1.0, size=(C, 128)))   # near the bound
    G, Hh, D, U = kda_subchunk_factors(al)
    assert np.log2(G).max() <= 7 * 5 / np.log(2) + 1e-9
    assert np.log2(Hh).max() <= 8 * 5 / np.log(2) + 1e-9
    assert min(D.min(), U.min()) >= 2.0 ** -60   # inside the kernel's domain


def test_kda_subchunk_factors_recover_pairwise_decay():
    """G_t H_i times the products between the two middles is Gamma_t / Gamma_i."""
    rng = np.random.default_rng(1)
    al = rng.uniform(0.2, 1.0, size=(C, 4))
    G, Hh, D, U = kda_subchunk_factors(al)
    L = D * U
    gam = np.cumprod(al, axis=0)
    for t in range(C):
        for i in range(t + 1):
            a, s = t // SUB, i // SUB
            mid = np.ones(4) if s == a else U[s] * np.prod(L[s + 1:a], axis=0) * D[a]
            np.testing.assert_allclose(G[t] * Hh[i] * mid, gam[t] / gam[i], rtol=1e-12)
