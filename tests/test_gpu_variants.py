"""GPU parity of the rule variants that run on the same kernels, against the
fp64 oracle:

  DeltaNet   the delta rule S_t = S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T,
             i.e. the gated delta rule with alpha = 1;
  RetNet     retention S_t = gamma S_{t-1} + k_t v_t^T with one constant gamma
             per head, i.e. GLA with that gamma on every key dim;
  Lightning  plain accumulation S_t = S_{t-1} + k_t v_t^T, i.e. GLA with g = 1
             (the output normalisation of that design is left to the caller).

(page "状态空间与线性注意力", Retention/Delta Rule; page "Linear / RNN 路线",
§2.4.)  Each is checked through the chunked tensor-core path (bf16, dk = 128),
the fp32 recurrent path and the decode step, at shapes with several chunks and a
ragged tail, and at the full d=128, T=8192 shape on a sample of heads.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_parity import TOL_BF16, TOL_F32, check, la, rel_err, run_gpu, sub_heads  # noqa: F401

pytestmark = pytest.mark.gpu

VARIANTS = {
    "deltanet": dict(rule="gdn", gdn_alpha="ones"),
    "retnet": dict(rule="gla", gla_gate="retnet"),
    "lightning": dict(rule="gla", gla_gate="ones"),
}


def problem(variant, B, T, H, dk, dv, **kw):
    v = dict(VARIANTS[variant])
    rule = v.pop("rule")
    return workloads.make_problem(rule, B, T, H, dk, dv, **v, **kw)


@pytest.mark.parametrize("variant", sorted(VARIANTS))
@pytest.mark.parametrize("T,dv", [(65, 128), (517, 64), (1100, 32)])
def test_variant_prefill_bf16(la, variant, T, dv):
    p = problem(variant, 2, T, 3, 128, dv, seed=T + dv, init_state="normal")
    check(p, *run_gpu(la, p), TOL_BF16)


@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_variant_prefill_fp32(la, variant):
    p = problem(variant, 2, 150, 2, 32, 32, dtype=torch.float32, seed=5, init_state="normal")
    check(p, *run_gpu(la, p), TOL_F32)


@pytest.mark.parametrize("variant", ["deltanet", "retnet"])
def test_variant_full_size_sampled(la, variant):
    """B=2, H=16, T=8192, d=128 (the prefill benchmark shape), heads (0,0) and (1,13)."""
    p = problem(variant, 2, 8192, 16, 128, 128, seed=3)
    o, S, _ = run_gpu(la, p)
    for b, h in ((0, 0), (1, 13)):
        check(p, o, S, None, TOL_BF16, heads=([b], [h]))


@pytest.mark.parametrize("variant", sorted(VARIANTS))
def test_variant_decode_steps(la, variant):
    """Six la_step calls on a carried state against the oracle's recurrence."""
    p = problem(variant, 4, 6, 3, 128, 64, seed=9, init_state="normal")
    S = p.S0.cuda()
    S_ref = p.S0.double().numpy()
    for t in range(6):
        g = p.g[:, t].contiguous()
        be = None if p.beta is None else p.beta[:, t].contiguous()
        q, k, v = (x[:, t].contiguous() for x in (p.q, p.k, p.v))
        o = la.step(p.rule, q.cuda(), k.cuda(), v.cuda(), S, g=g.cuda(),
                    beta=None if be is None else be.cuda())
        o_ref, S_ref, _ = oracle.step(p.rule, q, k, v, S_ref, g=g, beta=be)
        assert rel_err(o.float().cpu().numpy(), o_ref) <= TOL_BF16, f"step {t}"
    la.check_device()
    assert rel_err(S.cpu().numpy(), S_ref) <= TOL_BF16
