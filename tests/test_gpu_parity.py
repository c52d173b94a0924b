"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Metric (per tensor): max|x - ref| / max|ref|.  Bounds: 1e-4 for fp32 inputs,
2e-2 for bf16 inputs with fp32 accumulation (outputs and final state each).
The full-size workloads are checked on every (batch, head) sequence.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2
TOL_F32 = 1e-4


@pytest.fixture(scope="module")
def la():
    from gated_delta_rule_attn_b200 import build
    build.build()
    import gated_delta_rule_attn_b200 as m
    assert torch.cuda.is_available()
    return m


def rel_err(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert x.shape == ref.shape
    assert np.all(np.isfinite(x))
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


def to_dev(p: workloads.Problem):
    d = lambda t: None if t is None else t.cuda()
    return dict(q=d(p.q), k=d(p.k), v=d(p.v), g=d(p.g), beta=d(p.beta), S0=d(p.S0), z0=d(p.z0))


def run_gpu(la, p: workloads.Problem):
    t = to_dev(p)
    o, S, z = la.fwd(p.rule, t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["z0"], p.eps)
    torch.cuda.synchronize()
    la.check_device()
    return o.float().cpu().numpy(), S.cpu().numpy(), None if z is None else z.cpu().numpy()


def sub_heads(p: workloads.Problem, bs, hs):
    """The same problem restricted to batches bs and heads hs (independent sequences)."""
    sl = lambda t: None if t is None else t[bs][:, :, hs].contiguous()
    st = lambda t: None if t is None else t[bs][:, hs].contiguous()
    return workloads.Problem(p.rule, sl(p.q), sl(p.k), sl(p.v), sl(p.g), sl(p.beta),
                             st(p.S0), st(p.z0), p.eps, p.name)


def check(p, o, S, z, tol, heads=None):
    ref = p if heads is None else sub_heads(p, *heads)
    if heads is not None:
        bs, hs = heads
        o = o[bs][:, :, hs]
        S = S[bs][:, hs]
        z = None if z is None else z[bs][:, hs]
    ro, rS, rz = oracle.fwd(ref)
    errs = {"o": rel_err(o, ro), "S": rel_err(S, rS)}
    if rz is not None:
        errs["z"] = rel_err(z, rz)
    for k, e in errs.items():
        assert e <= tol, f"{p.name}: {k} rel err {e:.3e} > {tol}"
    return errs


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def test_elu_fp32_small(la):
    p = workloads.elu_fp32_small()
    check(p, *run_gpu(la, p), TOL_F32)


def test_gla_prefill_full(la):
    p = workloads.gla_prefill()
    check(p, *run_gpu(la, p), TOL_BF16)


def test_gla_prefill_long_full(la):
    """GLA at the prefill benchmark shape, B=2 H=16 T=8192 d=128, every head."""
    p = workloads.gla_prefill(B=2, H=16, T=8192)
    check(p, *run_gpu(la, p), TOL_BF16)


def test_elu_long_full(la):
    """Normalized ELU+1 at the pages' worked shape, B=1 H=16 N=32768 dphi=128 dv=64,
    with S0 >= 0 and z0 = 1 carried in, every head."""
    p = workloads.elu_long()
    check(p, *run_gpu(la, p), TOL_BF16)


def test_gdn_prefill_full(la):
    """The gated delta rule at B=2 H=16 T=8192 d=128, every head."""
    p = workloads.gdn_prefill()
    check(p, *run_gpu(la, p), TOL_BF16)


def test_gdn_split_invariance_at_3000(la):
    """Scan [0,3000), carry the state, scan [3000,8192): matches the oracle's whole
    scan and the GPU's whole scan (page "状态空间与线性注意力", chunk boundaries),
    every head."""
    p = workloads.gdn_prefill()
    hs = None
    t = to_dev(p)
    o_w, S_w, _ = la.fwd("gdn", t["q"], t["k"], t["v"], t["g"], t["beta"])
    tau = 3000
    cut = lambda x, a, b: x[:, a:b].contiguous()
    o1, S1, _ = la.fwd("gdn", *(cut(t[n], 0, tau) for n in ("q", "k", "v", "g", "beta")))
    o2, S2, _ = la.fwd("gdn", *(cut(t[n], tau, None) for n in ("q", "k", "v", "g", "beta")), S0=S1)
    torch.cuda.synchronize()
    o_s = torch.cat([o1, o2], 1).float().cpu().numpy()
    check(p, o_s, S2.cpu().numpy(), None, TOL_BF16, heads=hs)
    assert rel_err(o_s, o_w.float().cpu().numpy()) <= TOL_BF16
    assert rel_err(S2.cpu().numpy(), S_w.cpu().numpy()) <= TOL_BF16


# ---------------------------------------------------------------------------
# Small shapes: several chunks, ragged tails, every supported dk/dv, both dtypes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("rule", ["elu", "gla", "gdn"])
@pytest.mark.parametrize("T", [1, 17, 64, 65, 200])
@pytest.mark.parametrize("dv", [32, 64, 128])
def test_small_bf16_d128(la, rule, T, dv):
    p = workloads.make_problem(rule, 2, T, 3, 128, dv, seed=11 + T, init_state="normal")
    check(p, *run_gpu(la, p), TOL_BF16)


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn"])
@pytest.mark.parametrize("dk,dv", [(32, 32), (64, 128), (32, 64), (128, 32)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_small_other_dims(la, rule, dk, dv, dtype):
    p = workloads.make_problem(rule, 2, 77, 2, dk, dv, dtype=dtype, seed=dk + dv,
                               init_state="normal")
    check(p, *run_gpu(la, p), TOL_F32 if dtype == torch.float32 else TOL_BF16)


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn"])
def test_single_sequence_long_chain(la, rule):
    """B*H = 1: one CTA slab carries the state through 40 chunks."""
    p = workloads.make_problem(rule, 1, 2560 + 13, 1, 128, 128, seed=4, init_state="abs")
    check(p, *run_gpu(la, p), TOL_BF16)


@pytest.mark.parametrize("B,H,T,dv", [(1, 2, 1500, 64), (1, 1, 4096 + 33, 32), (2, 1, 3000, 128)])
def test_elu_sequence_parallel(la, B, H, T, dv):
    """Few heads and long sequences: the ELU+1 path cuts every sequence into
    segments that run side by side, each starting from S0 plus the state
    contributions of the earlier segments (summed by a first pass)."""
    p = workloads.make_problem("elu", B, T, H, 128, dv, seed=T + dv, init_state="abs")
    check(p, *run_gpu(la, p), TOL_BF16)


@pytest.mark.parametrize("gate", ["softplus16", "retnet", "ones"])
@pytest.mark.parametrize("B,H,T,dv", [(1, 2, 1500, 64), (1, 1, 4096 + 33, 32), (2, 1, 3000, 128)])
def test_gla_sequence_parallel(la, B, H, T, dv, gate):
    """GLA over few heads and long sequences runs segment-parallel: each segment
    starts from S0 folded through the earlier segments' ranges, S <- D o S + dS
    (D the range's gate product per key dim, from a first pass that walks each
    range backwards).  With the retention gate and with g = 1 the initial state
    and the early tokens still weigh on the last segment."""
    p = workloads.make_problem("gla", B, T, H, 128, dv, seed=T + dv, init_state="normal", gla_gate=gate)
    check(p, *run_gpu(la, p), TOL_BF16)


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_zero_length(la, rule, dtype):
    p = workloads.make_problem(rule, 2, 0, 2, 128, 64, dtype=dtype, seed=1, init_state="normal")
    o, S, z = run_gpu(la, p)
    assert o.shape == (2, 0, 2, 64)
    assert np.array_equal(S, p.S0.numpy())
    if rule == "elu":
        assert np.array_equal(z, p.z0.numpy())


def test_state_in_place(la):
    """S_out may alias S0."""
    p = workloads.make_problem("gla", 1, 130, 2, 128, 64, seed=2, init_state="normal")
    t = to_dev(p)
    S = t["S0"].clone()
    o, _, _ = la.fwd("gla", t["q"], t["k"], t["v"], t["g"], S0=S, S_out=S)
    torch.cuda.synchronize()
    check(p, o.float().cpu().numpy(), S.cpu().numpy(), None, TOL_BF16)


def _gla_gates(kind, B, T, H, seed):
    """Strongly decaying GLA gates, fp32 [B,T,H,128] in (0, 1]."""
    if kind == "0.3":       # 64-token product 2^-111: still the chunked form
        return torch.full((B, T, H, 128), 0.3)
    if kind == "0.02":      # 64-token product 2^-361: recomputed per token
        return torch.full((B, T, H, 128), 0.02)
    # half the key dims keep almost everything, half forget almost everything
    g = torch.full((B, T, H, 128), 0.999)
    g[..., 1::2] = 0.01
    return g


@pytest.mark.parametrize("kind", ["0.3", "0.02", "mix"])
@pytest.mark.parametrize("T,dv", [(517, 32), (1100, 64), (200, 128)])
def test_gla_any_gate_in_range(la, kind, T, dv):
    """GLA is defined for every g in (0, 1] ("Linear / RNN 路线" §2.2).  Chunks
    whose 64-token gate product stays >= 2^-120 per key dim run in the chunked
    tensor-core form; a sequence with any other chunk is recomputed exactly by the
    per-token recurrent kernel.  Every case matches the oracle and raises no
    device error."""
    p = workloads.make_problem("gla", 2, T, 2, 128, dv, seed=T + dv, init_state="normal")
    p = workloads.Problem("gla", p.q, p.k, p.v, _gla_gates(kind, 2, T, 2, 0), None, p.S0, None, p.eps,
                          f"gla_{kind}_T{T}_dv{dv}")
    check(p, *run_gpu(la, p), TOL_BF16)


@pytest.mark.parametrize("kind", ["0.02", "mix"])
def test_gla_any_gate_segment_parallel_and_in_place(la, kind):
    """Few heads and a long sequence (the segment-parallel path, whose first pass
    flags the earlier segments), with S_out aliasing S0, and a batch in which only
    one sequence leaves the range: each sequence matches the oracle."""
    B, T, H = 2, 3000, 2
    p = workloads.make_problem("gla", B, T, H, 128, 128, seed=44, init_state="normal")
    g = p.g.clone()
    # (5 segments of 10 chunks here: the first pass summarises segments 0-3)
    g[1] = _gla_gates(kind, 1, T, H, 1)[0]               # batch 1: every token, every segment
    g[0, 2600:2664] = _gla_gates(kind, 1, 64, H, 2)[0]   # batch 0: chunks 40-41, the last segment
    p = workloads.Problem("gla", p.q, p.k, p.v, g, None, p.S0, None, p.eps, f"gla_seg_{kind}")
    t = to_dev(p)
    assert la.fwd_workspace_size("gla", t["q"], t["k"], t["v"], t["g"]) > 1024   # segments
    S = t["S0"].clone()
    o, _, _ = la.fwd("gla", t["q"], t["k"], t["v"], t["g"], S0=S, S_out=S)
    torch.cuda.synchronize()
    la.check_device()
    check(p, o.float().cpu().numpy(), S.cpu().numpy(), None, TOL_BF16)


def test_gla_any_gate_packed(la):
    """Packed sequences: the flagged ones are recomputed on the packed layout."""
    lengths = [70, 0, 300, 129]
    parts = []
    for i, L in enumerate(lengths):
        q = workloads.make_problem("gla", 1, L, 2, 128, 64, seed=60 + i, init_state="normal")
        if i % 2 == 0:
            q = workloads.Problem("gla", q.q, q.k, q.v, _gla_gates("mix", 1, L, 2, i), None, q.S0, None, q.eps, "p")
        parts.append(q)
    cat = lambda n: torch.cat([getattr(q, n) for q in parts], dim=1).contiguous().cuda()
    S0 = torch.cat([q.S0 for q in parts], dim=0).contiguous().cuda()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int64).cuda()
    o, S, _ = la.fwd("gla", cat("q"), cat("k"), cat("v"), cat("g"), S0=S0, cu_seqlens=cu, max_seqlen=max(lengths))
    torch.cuda.synchronize()
    la.check_device()
    o = o.float().cpu().numpy()
    off = np.concatenate([[0], np.cumsum(lengths)])
    for i, q in enumerate(parts):
        ro, rS, _ = oracle.fwd(q)
        if lengths[i]:
            assert rel_err(o[:, off[i]:off[i + 1]], ro) <= TOL_BF16
        assert rel_err(S[i:i + 1].cpu().numpy(), rS) <= TOL_BF16


def test_host_buffer_entry_point_matches_device(la):
    p = workloads.make_problem("gdn", 2, 300, 3, 128, 64, seed=8, init_state="normal")
    t = to_dev(p)
    o_d, S_d, _ = la.fwd("gdn", t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"])
    pin = lambda x: None if x is None else x.pin_memory()
    hq, hk, hv, hg, hb, hS = (pin(x) for x in (p.q, p.k, p.v, p.g, p.beta, p.S0))
    o = torch.empty(2, 300, 3, 64, dtype=torch.bfloat16).pin_memory()
    S = torch.empty(2, 3, 128, 64).pin_memory()
    n = la.host_staging_size("gdn", hq, hk, hv, hg, hb, hS)
    staging = torch.empty(n, dtype=torch.uint8, device="cuda")
    la.fwd_host("gdn", hq, hk, hv, hg, hb, hS, o=o, S_out=S, staging=staging)
    torch.cuda.synchronize()
    assert torch.equal(o, o_d.cpu())
    assert torch.equal(S, S_d.cpu())
