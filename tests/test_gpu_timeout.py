"""Failure detection on the GPU, without a fault: waits that run out.

Every wait in the chunked kernels is bounded.  A wait that runs out raises the
timeout bit of the device error word; the CTA stops issuing, lets its copies and
MMAs in flight finish, frees its tensor memory and exits.  With the default
limit (about one second) no correct call reaches that path, so these tests
shorten the limit through the testing hook (include/la_testing.h), check that a
call then ends with LA_ERR_TIMEOUT and no fault, restore the limit, and check
that the next call on the same context still matches the oracle.  Nothing here
traps, faults or waits without a bound.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

LA_ERR_TIMEOUT = 5
DEFAULT_LIMIT = 2_000_000_000
TOL_BF16 = 2e-2


@pytest.fixture(scope="module")
def la():
    from gated_delta_rule_attn_b200 import build
    build.build()
    import gated_delta_rule_attn_b200 as m
    assert torch.cuda.is_available()
    return m


def _rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(x))
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def _run(la, p):
    d = {n: getattr(p, n).cuda() for n in ("q", "k", "v", "g", "beta")}
    return la.fwd(p.rule, d["q"], d["k"], d["v"], d["g"], d["beta"])


@pytest.mark.parametrize("T", [64 * 9 + 17, 4096])
def test_short_wait_limit_reports_timeout_and_context_recovers(la, T):
    """The gated delta rule on the tensor-core path (a prep kernel and the main
    pass, both with bounded waits and drains before TMEM is released)."""
    L = la.lib()
    p = workloads.make_problem("gdn", 1, T, 2, 128, 128, seed=T)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    prev = ctypes.c_int64(0)
    flags = ctypes.c_uint32(0)
    torch.cuda.synchronize()
    assert L.la_check_device(stream, ctypes.byref(flags)) == 0   # nothing pending
    assert L.la_testing_set_wait_limit(1000, ctypes.byref(prev)) == 0, L.la_last_error_message()
    try:
        _run(la, p)
        torch.cuda.synchronize()
        status = L.la_check_device(stream, ctypes.byref(flags))
    finally:
        assert L.la_testing_set_wait_limit(0, None) == 0
    assert prev.value == DEFAULT_LIMIT
    assert status == LA_ERR_TIMEOUT, (status, L.la_last_error_message())
    assert flags.value & 1
    # the same context, the default limit: the next call is whole and correct
    o, S, _ = _run(la, p)
    torch.cuda.synchronize()
    la.check_device()
    ro, rS, _ = oracle.fwd(p)
    assert _rel(o.float().cpu().numpy(), ro) <= TOL_BF16
    assert _rel(S.cpu().numpy(), rS) <= TOL_BF16


def test_limit_round_trip(la):
    """Setting and restoring the limit reads back what was set."""
    L = la.lib()
    prev = ctypes.c_int64(0)
    assert L.la_testing_set_wait_limit(12345, ctypes.byref(prev)) == 0
    try:
        assert prev.value == DEFAULT_LIMIT
        assert L.la_testing_set_wait_limit(0, ctypes.byref(prev)) == 0
        assert prev.value == 12345
    finally:
        L.la_testing_set_wait_limit(0, None)
    assert L.la_testing_set_wait_limit(0, ctypes.byref(prev)) == 0
    assert prev.value == DEFAULT_LIMIT
