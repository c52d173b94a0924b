"""GPU parity of the decode step (la_step) against the oracle's recurrence at T=1.

Full-size decode workload: state [256,16,128,128] fp32 ~ N(0,0.02), 64 GLA steps
and 64 gated-delta steps, each checked on all 256 sequences x 16 heads (every
step's output and the state after the last step).  Also: la_step equals la_fwd
at T=1, and 64 steps equal one 64-token prefill.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_parity import TOL_BF16, TOL_F32, la, rel_err, to_dev  # noqa: F401

pytestmark = pytest.mark.gpu

SAMPLE_N = slice(None)   # every sequence


@pytest.mark.parametrize("rule", ["gla", "gdn"])
def test_decode_full_workload(la, rule):
    steps = 64
    S0 = workloads.decode_state()
    inputs = workloads.decode_steps(rule, steps)
    S = S0.cuda()
    S_ref = S0[SAMPLE_N].double().numpy()
    worst = 0.0
    for i, inp in enumerate(inputs):
        q, k, v = (x.cuda() for x in inp[:3])
        if rule == "gla":
            o = la.step("gla", q, k, v, S, g=inp[3].cuda())
            o_ref, S_ref, _ = oracle.step("gla", inp[0][SAMPLE_N], inp[1][SAMPLE_N], inp[2][SAMPLE_N],
                                          S_ref, g=inp[3][SAMPLE_N])
        else:
            o = la.step("gdn", q, k, v, S, g=inp[3].cuda(), beta=inp[4].cuda())
            o_ref, S_ref, _ = oracle.step("gdn", inp[0][SAMPLE_N], inp[1][SAMPLE_N], inp[2][SAMPLE_N],
                                          S_ref, g=inp[3][SAMPLE_N], beta=inp[4][SAMPLE_N])
        e = rel_err(o[SAMPLE_N].float().cpu().numpy(), o_ref)
        worst = max(worst, e)
        assert e <= TOL_BF16, f"step {i}: o rel err {e:.3e}"
    la.check_device()
    assert rel_err(S[SAMPLE_N].cpu().numpy(), S_ref) <= TOL_BF16


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 32), (32, 128)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_step_small(la, rule, dk, dv, dtype):
    p = workloads.make_problem(rule, 5, 3, 3, dk, dv, dtype=dtype, seed=dk * 7 + dv,
                               init_state="normal")
    S = p.S0.cuda()
    z = None if p.z0 is None else p.z0.cuda()
    S_ref = p.S0.double().numpy()
    z_ref = None if p.z0 is None else p.z0.double().numpy()
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    for t in range(3):
        g = None if p.g is None else p.g[:, t]
        be = None if p.beta is None else p.beta[:, t]
        o = la.step(rule, p.q[:, t].contiguous().cuda(), p.k[:, t].contiguous().cuda(),
                    p.v[:, t].contiguous().cuda(), S, z,
                    None if g is None else g.contiguous().cuda(),
                    None if be is None else be.contiguous().cuda(), p.eps)
        o_ref, S_ref, z_ref = oracle.step(rule, p.q[:, t], p.k[:, t], p.v[:, t], S_ref, z_ref, g, be,
                                          p.eps)
        assert rel_err(o.float().cpu().numpy(), o_ref) <= tol
    assert rel_err(S.cpu().numpy(), S_ref) <= tol
    if z is not None:
        assert rel_err(z.cpu().numpy(), z_ref) <= tol


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn"])
def test_prefill_T1_equals_step(la, rule):
    p = workloads.make_problem(rule, 3, 1, 4, 128, 128, seed=21, init_state="normal")
    t = to_dev(p)
    o_f, S_f, z_f = la.fwd(rule, t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["z0"], p.eps)
    S = t["S0"].clone()
    z = None if t["z0"] is None else t["z0"].clone()
    o_s = la.step(rule, t["q"][:, 0].contiguous(), t["k"][:, 0].contiguous(), t["v"][:, 0].contiguous(),
                  S, z, None if t["g"] is None else t["g"][:, 0].contiguous(),
                  None if t["beta"] is None else t["beta"][:, 0].contiguous(), p.eps)
    torch.cuda.synchronize()
    assert rel_err(o_f[:, 0].float().cpu().numpy(), o_s.float().cpu().numpy()) <= TOL_BF16
    assert rel_err(S_f.cpu().numpy(), S.cpu().numpy()) <= TOL_BF16


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn"])
def test_64_steps_equal_prefill(la, rule):
    p = workloads.make_problem(rule, 2, 64, 2, 128, 64, seed=33, init_state="normal")
    t = to_dev(p)
    o_f, S_f, _ = la.fwd(rule, t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"], t["z0"], p.eps)
    S = t["S0"].clone()
    z = None if t["z0"] is None else t["z0"].clone()
    outs = []
    for i in range(64):
        sl = lambda x: None if x is None else x[:, i].contiguous()
        outs.append(la.step(rule, sl(t["q"]), sl(t["k"]), sl(t["v"]), S, z, sl(t["g"]), sl(t["beta"]),
                            p.eps))
    torch.cuda.synchronize()
    o_s = torch.stack(outs, 1)
    assert rel_err(o_s.float().cpu().numpy(), o_f.float().cpu().numpy()) <= TOL_BF16
    assert rel_err(S.cpu().numpy(), S_f.cpu().numpy()) <= TOL_BF16
