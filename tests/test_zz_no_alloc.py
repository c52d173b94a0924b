"""la_fwd_noalloc: prefill for callers that cannot allocate device memory.

Such callers (a host framework that owns every device allocation, a plugin with
a fixed memory budget, a latency-critical path that must not touch the
allocator) cannot hand la_fwd the workspace the gated delta rule's tensor-core
path needs.  la_fwd_noalloc uses the library's own fixed 16 MiB device array
instead.  These tests call it through the C ABI and check that it gives what
la_fwd gives, on two calls in a row with different inputs (the array keeps the
previous call's contents), and that a problem needing more scratch than the
array holds is refused before anything runs.  KDA, whose chunked path keeps
scaled q/k tensors in the scratch, runs chunked when they fit and on the
scratch-free recurrent kernel when they do not; both must match la_fwd.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

TOL = 2e-2   # the bf16 parity bound used by the other GPU tests


def _lib():
    from gated_delta_rule_attn_b200 import build
    build.build()
    import gated_delta_rule_attn_b200 as la
    return la


def _rel(x, ref):
    x = x.float().cpu().numpy().astype(np.float64)
    ref = ref.float().cpu().numpy().astype(np.float64)
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def test_oversized_problem_refused_on_host():
    """Needs no GPU: the size check runs before any CUDA call."""
    la = _lib()
    L = la.lib()
    a = la.FwdArgs()
    a.struct_size = ctypes.sizeof(a)
    a.rule, a.dtype = 2, 1
    a.B, a.T, a.H, a.dk, a.dv = 1, 64 * 65, 32, 128, 128      # 2080 chunk units > 1024
    a.q = a.k = a.v = a.o = a.g = a.beta = 0x10000
    assert L.la_fwd_noalloc(ctypes.byref(a), None) == 8
    assert b"la_fwd_noalloc" in L.la_last_error_message()


@pytest.mark.gpu
def test_noalloc_matches_la_fwd_on_two_calls():
    la = _lib()
    L = la.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed, (B, T, H, dv) in ((17, (2, 300, 3, 64)), (23, (1, 517, 4, 128))):
        p = workloads.make_problem("gdn", B, T, H, 128, dv, seed=seed, init_state="normal")
        d = {n: getattr(p, n).cuda() for n in ("q", "k", "v", "g", "beta", "S0")}
        o_ref, S_ref, _ = la.fwd("gdn", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
        o = torch.empty_like(o_ref)
        S = torch.empty_like(S_ref)
        a = la.make_fwd_args("gdn", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], None, 1e-6,
                             o, S, None)
        rc = L.la_fwd_noalloc(ctypes.byref(a), stream)
        assert rc == 0, L.la_last_error_message()
        torch.cuda.synchronize()
        la.check_device()
        assert _rel(o, o_ref) <= TOL
        assert _rel(S, S_ref) <= TOL


@pytest.mark.gpu
@pytest.mark.parametrize("T", [300, 2048])
def test_noalloc_kda_fits_or_runs_without_scratch(T):
    """T=300 (B*H = 4) fits the array and runs chunked; T=2048 at H=16 needs
    about 25 MB of chunked scratch and runs on the recurrent kernel."""
    la = _lib()
    L = la.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    H = 4 if T == 300 else 16
    p = workloads.make_problem("kda", 1, T, H, 128, 128, seed=T, init_state="normal")
    d = {n: getattr(p, n).cuda() for n in ("q", "k", "v", "g", "beta", "S0")}
    o_ref, S_ref, _ = la.fwd("kda", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    assert (la.fwd_workspace_size("kda", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
            > (16 << 20)) == (T == 2048)
    for _ in range(2):
        o = torch.empty_like(o_ref)
        S = torch.empty_like(S_ref)
        a = la.make_fwd_args("kda", d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], None, 1e-6,
                             o, S, None)
        rc = L.la_fwd_noalloc(ctypes.byref(a), stream)
        assert rc == 0, L.la_last_error_message()
        torch.cuda.synchronize()
        la.check_device()
        assert _rel(o, o_ref) <= TOL
        assert _rel(S, S_ref) <= TOL
