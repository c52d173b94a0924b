"""la_fwd_noalloc: prefill for callers that cannot allocate device memory.

Such callers (a host framework that owns every device allocation, a plugin with
a fixed memory budget, a latency-critical path that must not touch the
allocator) cannot hand la_fwd the workspace that the gated delta rule's
tensor-core path, chunked KDA and segment-parallel ELU+1 / GLA need.
la_fwd_noalloc uses the library's own fixed 16 MiB device array instead.

These tests call it through the C ABI.  It runs the same kernels as la_fwd on
the same inputs, so where la_fwd runs the same path the results must be equal
bit for bit; this holds on two calls in a row with different inputs (the array
keeps the previous call's contents).  KDA problems whose chunked scratch does
not fit run on the scratch-free recurrent kernel and are checked against the
fp64 oracle.  A problem needing more scratch than the array holds is refused
before anything runs, and a call changes neither the device's free memory nor
PyTorch's allocations.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

TOL = 2e-2   # the bf16 parity bound of the other GPU tests (oracle comparisons only)


def _lib():
    from gated_delta_rule_attn_b200 import build
    build.build()
    import gated_delta_rule_attn_b200 as la
    return la


def _rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(x))
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def _dev(p):
    return {n: (None if getattr(p, n) is None else getattr(p, n).cuda())
            for n in ("q", "k", "v", "g", "beta", "S0", "z0")}


def _noalloc(la, rule, d, eps=1e-6, cu=None, max_seqlen=None, out_norm=False, norm_w=None):
    """la_fwd_noalloc through the C ABI; returns (o, S_out, z_out)."""
    L = la.lib()
    ns = d["q"].shape[0] if cu is None else cu.numel() - 1
    H, dk, dv = d["q"].shape[2], d["q"].shape[3], d["v"].shape[3]
    o = torch.empty(*d["q"].shape[:3], dv, dtype=d["q"].dtype, device="cuda")
    S = torch.empty(ns, H, dk, dv, device="cuda")
    z = torch.empty(ns, H, dk, device="cuda") if rule == "elu" else None
    a = la.make_fwd_args(rule, d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["z0"], eps, o, S, z,
                         cu, max_seqlen, out_norm, norm_w, 1e-6)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.la_fwd_noalloc(ctypes.byref(a), stream)
    assert rc == 0, L.la_last_error_message()
    torch.cuda.synchronize()
    la.check_device()
    return o, S, z


def _same(a, b):
    for x, y in zip(a, b):
        if x is None:
            assert y is None
        else:
            assert torch.equal(x, y)


def test_oversized_problem_refused_on_host():
    """Needs no GPU: the size check runs before any CUDA call."""
    la = _lib()
    L = la.lib()
    a = la.FwdArgs()
    a.struct_size = ctypes.sizeof(a)
    a.rule, a.dtype = 2, 1
    a.B, a.T, a.H, a.dk, a.dv = 1, 64 * 65, 32, 128, 128      # 2080 chunk units > 512
    a.q = a.k = a.v = a.o = a.g = a.beta = 0x10000
    assert L.la_fwd_noalloc(ctypes.byref(a), None) == 8
    assert b"la_fwd_noalloc" in L.la_last_error_message()


@pytest.mark.gpu
def test_noalloc_equals_la_fwd_bitwise_on_two_calls():
    """The gated delta rule's tensor-core path (prep kernel items in the array),
    two different problems in a row."""
    la = _lib()
    for seed, (B, T, H, dv) in ((17, (2, 300, 3, 64)), (23, (1, 517, 4, 128))):
        p = workloads.make_problem("gdn", B, T, H, 128, dv, seed=seed, init_state="normal")
        d = _dev(p)
        ref = la.fwd("gdn", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
        got = _noalloc(la, "gdn", d)
        _same(got, ref)


@pytest.mark.gpu
@pytest.mark.parametrize("rule", ["gla", "elu"])
def test_noalloc_segment_parallel_in_the_array(rule):
    """Few heads and a long sequence: ELU+1 / GLA run as parallel segments whose
    summaries live in the array; with and without the output normalisation."""
    la = _lib()
    p = workloads.make_problem(rule, 1, 3000, 2, 128, 128, seed=31, init_state="normal")
    d = _dev(p)
    assert la.fwd_workspace_size(rule, d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["z0"]) > 0
    for out_norm in (False, True):
        ref = la.fwd(rule, d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["z0"], 1e-6,
                     out_norm=out_norm)
        got = _noalloc(la, rule, d, out_norm=out_norm)
        _same(got, ref)
        if not out_norm:
            ro, rS, rz = oracle.fwd(p)
            assert _rel(got[0].float().cpu().numpy(), ro) <= TOL
            assert _rel(got[1].cpu().numpy(), rS) <= TOL


def _packed(rule, lengths, H, seed):
    parts = [workloads.make_problem(rule, 1, L, H, 128, 128, seed=seed + i, init_state="normal")
             for i, L in enumerate(lengths)]
    cat = lambda n: torch.cat([getattr(q, n) for q in parts], dim=1).contiguous().cuda()
    d = dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"),
             S0=torch.cat([q.S0 for q in parts], dim=0).contiguous().cuda(), z0=None)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int64).cuda()
    return parts, d, cu


@pytest.mark.gpu
def test_noalloc_packed_gated_delta_bitwise():
    la = _lib()
    lengths = [65, 0, 300, 1, 128]
    _, d, cu = _packed("gdn", lengths, 3, seed=70)
    ref = la.fwd("gdn", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], cu_seqlens=cu,
                 max_seqlen=max(lengths))
    got = _noalloc(la, "gdn", d, cu=cu, max_seqlen=max(lengths))
    _same(got, ref)


@pytest.mark.gpu
def test_noalloc_packed_kda_falls_back_to_the_recurrent_kernel():
    """Packed KDA whose chunked scratch (about 50 MB) does not fit the array runs
    on the recurrent kernel; each sequence against the oracle run alone."""
    la = _lib()
    lengths = [2048, 700, 1500, 33]
    parts, d, cu = _packed("kda", lengths, 8, seed=90)
    assert la.fwd_workspace_size("kda", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"]) > (16 << 20)
    o, S, _ = _noalloc(la, "kda", d, cu=cu, max_seqlen=max(lengths))
    o = o.float().cpu().numpy()
    off = np.concatenate([[0], np.cumsum(lengths)])
    for i, p in enumerate(parts):
        ro, rS, _ = oracle.fwd(p)
        assert _rel(o[:, off[i]:off[i + 1]], ro) <= TOL
        assert _rel(S[i:i + 1].cpu().numpy(), rS) <= TOL


@pytest.mark.gpu
@pytest.mark.parametrize("T", [300, 2048])
def test_noalloc_kda_fits_or_runs_without_scratch(T):
    """T=300 (B*H = 4) fits the array and runs chunked (bitwise equal to la_fwd);
    T=2048 at H=16 needs about 25 MB of chunked scratch and runs on the
    recurrent kernel (checked against the oracle on two of its heads)."""
    la = _lib()
    H = 4 if T == 300 else 16
    p = workloads.make_problem("kda", 1, T, H, 128, 128, seed=T, init_state="normal")
    d = _dev(p)
    need = la.fwd_workspace_size("kda", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert (need > (16 << 20)) == (T == 2048)
    ref = la.fwd("kda", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    for _ in range(2):
        got = _noalloc(la, "kda", d)
        if T == 300:
            _same(got, ref)
        else:
            hs = [0, H - 1]
            sub = workloads.Problem("kda", p.q[:, :, hs].contiguous(), p.k[:, :, hs].contiguous(),
                                    p.v[:, :, hs].contiguous(), p.g[:, :, hs].contiguous(),
                                    p.beta[:, :, hs].contiguous(), p.S0[:, hs].contiguous(), None, p.eps, "kda2")
            ro, rS, _ = oracle.fwd(sub)
            assert _rel(got[0][:, :, hs].float().cpu().numpy(), ro) <= TOL
            assert _rel(got[1][:, hs].cpu().numpy(), rS) <= TOL


@pytest.mark.gpu
def test_noalloc_allocates_nothing():
    """After a first call (which may look up the array's address), a call leaves
    the device's free memory and PyTorch's allocations exactly as they were."""
    la = _lib()
    p = workloads.make_problem("gdn", 2, 700, 4, 128, 128, seed=5, init_state="normal")
    d = _dev(p)
    L = la.lib()
    o = torch.empty(2, 700, 4, 128, dtype=torch.bfloat16, device="cuda")
    S = torch.empty(2, 4, 128, 128, device="cuda")
    a = la.make_fwd_args("gdn", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], None, 1e-6, o, S, None)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.la_fwd_noalloc(ctypes.byref(a), stream) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        assert L.la_fwd_noalloc(ctypes.byref(a), stream) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0
    la.check_device()
