"""Stream order around la_fwd: inputs written by kernels queued just before the
call on the same stream, outputs read by kernels queued just after it.

Inside a call, the second kernel of a two-kernel prefill (the gated delta rule's
and KDA's main pass after their prep kernels, the ELU+1 / GLA main pass after the
segment summaries) is a programmatic dependent of the first: it may start before
the first finishes and waits for it before reading its results.  That must not
loosen the order towards the caller's own work.  Each input here is scaled by 4
on the device and halved twice by kernels queued right before the call, with no
synchronisation in between (powers of two: the values return exactly), so a
kernel of the call that read an input early would see 2x or 4x the data.  The
outputs are copied by kernels queued right after the call.  Results are checked
against the fp64 oracle on the unscaled inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL = 2e-2


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
    assert x.shape == ref.shape and np.all(np.isfinite(x))
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


# (rule, B, T, H, dv): the gated delta rule and KDA (prep + main pass), GLA and
# ELU+1 with few heads over 64 chunks (segment summaries + main pass)
CASES = [("gdn", 2, 700, 3, 128), ("kda", 1, 700, 2, 128), ("gla", 1, 4096, 2, 128), ("elu", 1, 4096, 2, 64)]


@pytest.mark.parametrize("rule,B,T,H,dv", CASES)
def test_inputs_from_preceding_kernels_outputs_to_following_ones(la, rule, B, T, H, dv):
    p = workloads.make_problem(rule, B, T, H, 128, dv, seed=31, init_state="normal")
    ro, rS, rz = oracle.fwd(p)
    names = ("q", "k", "v", "g", "beta", "S0", "z0")
    dev = {n: None if getattr(p, n) is None else getattr(p, n).cuda() * 4 for n in names}
    torch.cuda.synchronize()
    for t in dev.values():          # the writes the call must see, queued just before it
        if t is not None:
            t.mul_(0.5)
            t.mul_(0.5)
    o, S, z = la.fwd(rule, dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev["S0"], dev["z0"], p.eps)
    o2 = o.float() * 1.0            # the reads that must see the call's results, queued just after it
    S2 = S.clone()
    z2 = None if z is None else z.clone()
    torch.cuda.synchronize()
    la.check_device()
    assert rel_err(o2.cpu().numpy(), ro) <= TOL
    assert rel_err(S2.cpu().numpy(), rS) <= TOL
    if rz is not None:
        assert rel_err(z2.cpu().numpy(), rz) <= TOL
