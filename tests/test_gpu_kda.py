"""GPU parity of KDA (per-key-channel retention with the delta rule, page
"状态空间与线性注意力", KDA：逐通道遗忘与误差写入) against the fp64 oracle.

KDA runs on the per-token recurrent kernel for every dtype and size (there is
no chunked tensor-core kernel for it yet): prefill at several shapes with
ragged lengths, the decode step on a carried state, the full decode shape on a
sample of sequences, and packed variable-length sequences.  Inputs follow the
page's recipe: L2-normalised q and k, beta = sigmoid(N(0,1)) and the bounded
retention alpha = exp(-5 sigmoid(N(0,1))) per key channel.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_parity import TOL_BF16, TOL_F32, check, la, rel_err, run_gpu  # noqa: F401

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 77, 300])
@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, torch.bfloat16), (64, 32, torch.bfloat16),
                                         (32, 64, torch.float32), (128, 32, torch.float32)])
def test_kda_prefill(la, T, dk, dv, dtype):
    p = workloads.make_problem("kda", 2, T, 3, dk, dv, dtype=dtype, seed=T + dk, init_state="normal")
    check(p, *run_gpu(la, p), TOL_F32 if dtype == torch.float32 else TOL_BF16)


def test_kda_long_sequence(la):
    """2 x 4 heads x 2049 tokens at d = 128: the state carried through a long walk."""
    p = workloads.make_problem("kda", 2, 2049, 4, 128, 128, seed=12, init_state="normal")
    check(p, *run_gpu(la, p), TOL_BF16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_kda_decode_steps(la, dtype):
    p = workloads.make_problem("kda", 6, 8, 4, 128, 64, dtype=dtype, seed=21, init_state="normal")
    S = p.S0.cuda()
    S_ref = p.S0.double().numpy()
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    for t in range(8):
        q, k, v, g = (x[:, t].contiguous() for x in (p.q, p.k, p.v, p.g))
        be = p.beta[:, t].contiguous()
        o = la.step("kda", q.cuda(), k.cuda(), v.cuda(), S, g=g.cuda(), beta=be.cuda())
        o_ref, S_ref, _ = oracle.step("kda", q, k, v, S_ref, g=g, beta=be)
        assert rel_err(o.float().cpu().numpy(), o_ref) <= tol, f"step {t}"
    la.check_device()
    assert rel_err(S.cpu().numpy(), S_ref) <= tol


def test_kda_decode_full_shape_sampled(la):
    """One step on the decode workload's state [256,16,128,128] fp32, checked on
    sequences 0, 100 and 255."""
    S0 = workloads.decode_state()
    p = workloads.make_problem("kda", 256, 1, 16, 128, 128, seed=31)
    q, k, v, g = (x[:, 0].contiguous() for x in (p.q, p.k, p.v, p.g))
    be = p.beta[:, 0].contiguous()
    S = S0.cuda()
    o = la.step("kda", q.cuda(), k.cuda(), v.cuda(), S, g=g.cuda(), beta=be.cuda())
    la.check_device()
    n = [0, 100, 255]
    o_ref, S_ref, _ = oracle.step("kda", q[n], k[n], v[n], S0[n].double().numpy(), g=g[n], beta=be[n])
    assert rel_err(o[n].float().cpu().numpy(), o_ref) <= TOL_BF16
    assert rel_err(S[n].cpu().numpy(), S_ref) <= TOL_BF16


def test_kda_packed_sequences(la):
    lengths = [5, 0, 130, 64, 1]
    parts = [workloads.make_problem("kda", 1, L, 2, 128, 64, seed=60 + i, init_state="normal")
             for i, L in enumerate(lengths)]
    cat = lambda n: torch.cat([getattr(p, n) for p in parts], dim=1).contiguous().cuda()
    S0 = torch.cat([p.S0 for p in parts], dim=0).contiguous().cuda()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int64).cuda()
    o, S, _ = la.fwd("kda", cat("q"), cat("k"), cat("v"), cat("g"), cat("beta"), S0,
                     cu_seqlens=cu, max_seqlen=max(lengths))
    torch.cuda.synchronize()
    la.check_device()
    o = o.float().cpu().numpy()
    for i, p in enumerate(parts):
        ro, rS, _ = oracle.fwd(p)
        s0, s1 = int(cu[i]), int(cu[i + 1])
        if s1 > s0:
            assert rel_err(o[:, s0:s1], ro) <= TOL_BF16
        assert rel_err(S[i:i + 1].cpu().numpy(), rS) <= TOL_BF16
