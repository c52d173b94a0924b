"""GPU parity of the output normalisation (``out_norm``): Lightning attention's
o_t = Norm(q_t^T S_t) (page "Linear / RNN 路线", §2.4: GLA with g = 1 and an
RMSNorm at the output) and the head-wise RMSNorm of the recurrent output that K3
applies (page "状态空间与线性注意力", KDA section).

Reference: the fp64 oracle's recurrence followed by ``oracle.head_rmsnorm`` on
its exact output.  The library normalises its stored (bf16-rounded for bf16
problems) output in a second pass and rounds once more.  The state is not
touched by the normalisation: it must equal, bit for bit, the state of the same
call without it.

Bounds.  Every rule but KDA: the normalised output is held to the fixed bf16
(2e-2) or fp32 (1e-4) bound against the oracle's normalised output, like any
other output.  KDA: its per-channel retention leaves rows whose RMS is a small
fraction of the largest, and dividing a row by its RMS sigma multiplies the
row's absolute error by about (1 + max|o_row| / sigma) / sigma to first order,
whatever the method.  So a KDA row may differ from the reference by one rounding
of the normalised scale (the tolerance times max|y_ref|) plus that propagation
of the un-normalised error budget, the tolerance times max|o_ref| (which the
un-normalised output is held to first), with the row's conditioning taken from
the oracle's output (times 1.5 for second-order terms).  No part of the bound
comes from the GPU's own measured error.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_parity import TOL_BF16, TOL_F32, la, rel_err, sub_heads, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu

EPS_N = 1e-6


def weight(dv, seed):
    g = torch.Generator().manual_seed(seed)
    return (1.0 + 0.5 * torch.randn(dv, generator=g)).float()


def run(la, p, w, out_norm=True, norm_eps=EPS_N):
    t = to_dev(p)
    o, S, z = la.fwd(p.rule, t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["z0"], p.eps,
                     out_norm=out_norm, norm_w=None if w is None else w.cuda(), norm_eps=norm_eps)
    torch.cuda.synchronize()
    la.check_device()
    return o, S, z


def check_norm(la, p, w, tol, norm_eps=EPS_N):
    o, S, z = run(la, p, w, norm_eps=norm_eps)
    o_plain, S_plain, z_plain = run(la, p, None, out_norm=False)
    ro, rS, _ = oracle.fwd(p)
    want = oracle.head_rmsnorm(ro, None if w is None else w.double().numpy(), norm_eps)
    # the output bound, before normalisation
    op = o_plain.float().cpu().numpy().astype(np.float64)
    assert rel_err(op, ro) <= tol, f"{p.name}: un-normalised o rel err {rel_err(op, ro):.3e}"
    y = o.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(y))
    e = rel_err(y, want)
    if p.rule != "kda":
        assert e <= tol, f"{p.name}: normalised o rel err {e:.3e} > {tol}"
    else:
        # each row: one rounding of the normalised scale plus the first-order
        # propagation of the un-normalised error budget through w o / sigma
        wmax = 1.0 if w is None else float(w.abs().max())
        sigma = np.sqrt((ro ** 2).mean(axis=-1) + norm_eps)
        cond = (1.0 + np.abs(ro).max(axis=-1) / sigma) / sigma
        bound = tol * np.abs(want).max() + 1.5 * wmax * (tol * np.abs(ro).max()) * cond
        dy = np.abs(y - want).max(axis=-1)
        worst = np.unravel_index(np.argmax(dy / bound), dy.shape)
        assert np.all(dy <= bound), (f"{p.name}: normalised row {worst} off by {dy[worst]:.3e} "
                                     f"> bound {bound[worst]:.3e}")
    assert torch.equal(S, S_plain)
    if z is not None:
        assert torch.equal(z, z_plain)
    assert rel_err(S.cpu().numpy(), rS) <= tol
    return e


@pytest.mark.parametrize("with_w", [False, True])
@pytest.mark.parametrize("T,dv", [(65, 128), (517, 64), (1100, 32), (3000, 128)])
def test_lightning_prefill_chunked(la, T, dv, with_w):
    """Lightning = GLA at g = 1 with the output norm, on the tensor-core path
    (bf16, dk = 128), several chunks and a ragged tail; T = 3000 over 2 heads
    also runs segment-parallel."""
    p = workloads.make_problem("gla", 1, T, 2, 128, dv, gla_gate="ones", seed=T + dv, init_state="normal")
    check_norm(la, p, weight(dv, T) if with_w else None, TOL_BF16)


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn", "kda"])
@pytest.mark.parametrize("dk,dv,dtype", [(128, 64, torch.bfloat16), (32, 32, torch.float32),
                                         (64, 128, torch.bfloat16)])
def test_norm_every_rule_and_path(la, rule, dk, dv, dtype):
    p = workloads.make_problem(rule, 2, 150, 3, dk, dv, dtype=dtype, seed=dk + dv, init_state="normal")
    check_norm(la, p, weight(dv, 3), TOL_F32 if dtype == torch.float32 else TOL_BF16)


@pytest.mark.parametrize("rule,T", [("elu", 300), ("elu", 3000), ("gla", 777)])
def test_norm_over_two_value_slabs(la, rule, T):
    """dv = 128: each row spans two 64-column value slabs of the chunked kernel
    (T = 3000 over 3 heads also runs segment-parallel)."""
    kw = {"gla_gate": "ones"} if rule == "gla" else {}
    p = workloads.make_problem(rule, 1, T, 3, 128, 128, seed=T + 1, init_state="normal", **kw)
    check_norm(la, p, weight(128, T), TOL_BF16)


@pytest.mark.parametrize("dv", [64, 128])
def test_norm_on_recomputed_gla_sequences(la, dv):
    """GLA gates of 0.02 take every chunk out of the chunked form's range: the
    sequences are recomputed by the per-token kernel before the normalisation
    pass."""
    p = workloads.make_problem("gla", 2, 300, 2, 128, dv, seed=dv, init_state="normal")
    p = workloads.Problem("gla", p.q, p.k, p.v, torch.full((2, 300, 2, 128), 0.02), None, p.S0, None, p.eps,
                          f"gla_0.02_norm_dv{dv}")
    check_norm(la, p, weight(dv, 4), TOL_BF16)


def test_norm_eps_matters_for_small_rows(la):
    """A large eps against an output of small RMS scales the rows down rather than
    up to unit RMS; the library follows the oracle there too."""
    p = workloads.make_problem("gla", 1, 200, 2, 128, 64, gla_gate="ones", seed=9)
    check_norm(la, p, None, TOL_BF16, norm_eps=4.0)


@pytest.mark.parametrize("rule,variant", [("gla", "ones"), ("gdn", None), ("kda", None)])
def test_decode_step_with_norm(la, rule, variant):
    kw = {"gla_gate": variant} if variant else {}
    p = workloads.make_problem(rule, 4, 5, 3, 128, 64, seed=17, init_state="normal", **kw)
    w = weight(64, 5)
    S = p.S0.cuda()
    S_ref = p.S0.double().numpy()
    for t in range(5):
        q, k, v, g = (x[:, t].contiguous() for x in (p.q, p.k, p.v, p.g))
        be = None if p.beta is None else p.beta[:, t].contiguous()
        o = la.step(rule, q.cuda(), k.cuda(), v.cuda(), S, g=g.cuda(), beta=None if be is None else be.cuda(),
                    out_norm=True, norm_w=w.cuda(), norm_eps=EPS_N)
        o_ref, S_ref, _ = oracle.step(rule, q, k, v, S_ref, g=g, beta=be)
        want = oracle.head_rmsnorm(o_ref, w.double().numpy(), EPS_N)
        assert rel_err(o.float().cpu().numpy(), want) <= TOL_BF16, f"step {t}"
    la.check_device()
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL_BF16


@pytest.mark.parametrize("dv", [64, 128])
def test_packed_sequences_with_norm(la, dv):
    lengths = [70, 0, 3, 200]
    parts = [workloads.make_problem("gla", 1, L, 2, 128, dv, gla_gate="ones", seed=80 + i, init_state="normal")
             for i, L in enumerate(lengths)]
    cat = lambda n: torch.cat([getattr(p, n) for p in parts], dim=1).contiguous().cuda()
    S0 = torch.cat([p.S0 for p in parts], dim=0).contiguous().cuda()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int64).cuda()
    w = weight(dv, 8)
    o, S, _ = la.fwd("gla", cat("q"), cat("k"), cat("v"), cat("g"), S0=S0, cu_seqlens=cu,
                     max_seqlen=max(lengths), out_norm=True, norm_w=w.cuda(), norm_eps=EPS_N)
    torch.cuda.synchronize()
    la.check_device()
    o = o.float().cpu().numpy()
    for i, p in enumerate(parts):
        ro, rS, _ = oracle.fwd(p)
        s0, s1 = int(cu[i]), int(cu[i + 1])
        if s1 > s0:
            assert rel_err(o[:, s0:s1], oracle.head_rmsnorm(ro, w.double().numpy(), EPS_N)) <= TOL_BF16
        assert rel_err(S[i:i + 1].cpu().numpy(), rS) <= TOL_BF16


def test_lightning_full_size(la):
    """B=2, H=16, T=8192, d=128 (the prefill benchmark shape) with g = 1 and the
    norm, every head against the oracle at the fixed bound."""
    p = workloads.make_problem("gla", 2, 8192, 16, 128, 128, gla_gate="ones", seed=3)
    w = weight(128, 1)
    o, S, _ = run(la, p, w)
    ro, rS, _ = oracle.fwd(p)
    want = oracle.head_rmsnorm(ro, w.double().numpy(), EPS_N)
    assert rel_err(o.float().cpu().numpy(), want) <= TOL_BF16
    assert rel_err(S.cpu().numpy(), rS) <= TOL_BF16


def test_host_buffers_with_norm_match_device(la):
    p = workloads.make_problem("gla", 2, 300, 2, 128, 64, gla_gate="ones", seed=12, init_state="normal")
    w = weight(64, 2)
    o_d, S_d, _ = run(la, p, w)
    pin = lambda x: None if x is None else x.pin_memory()
    hq, hk, hv, hg, hS = (pin(x) for x in (p.q, p.k, p.v, p.g, p.S0))
    o_h = torch.empty(2, 300, 2, 64, dtype=torch.bfloat16).pin_memory()
    S_h = torch.empty(2, 2, 128, 64).pin_memory()
    n = la.host_staging_size("gla", hq, hk, hv, g=hg, S0=hS, out_norm=True, norm_w=w)
    staging = torch.empty(n, dtype=torch.uint8, device="cuda")
    la.fwd_host("gla", hq, hk, hv, g=hg, S0=hS, o=o_h, S_out=S_h, staging=staging,
                out_norm=True, norm_w=w.pin_memory(), norm_eps=EPS_N)
    assert torch.equal(o_h, o_d.cpu())
    assert torch.equal(S_h, S_d.cpu())
