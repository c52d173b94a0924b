"""GPU parity of KDA (per-key-channel retention with the delta rule, page
"状态空间与线性注意力", KDA：逐通道遗忘与误差写入) against the fp64 oracle.

bf16 prefill with dk = 128 runs chunked on the tensor cores (kda_prep_kernel,
then gdn_main_kernel<true>): ragged lengths that span several 64-token chunks
and 16-token sub-chunks, every value width, zero and nonzero initial states, a
split with the state carried across it, the benchmark shape on a sample of
heads, the host-buffer entry point and the retention-range report.  fp32,
dk < 128, decode and packed sequences run on the per-token recurrent kernel.
Inputs follow the page's recipe: L2-normalised q and k, beta = sigmoid(N(0,1))
and the bounded retention alpha = exp(-5 sigmoid(N(0,1))) per key channel.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_parity import TOL_BF16, TOL_F32, check, la, rel_err, run_gpu, to_dev  # noqa: F401

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


@pytest.mark.parametrize("T", [1, 16, 64, 65, 517, 1100])
@pytest.mark.parametrize("dv", [32, 64, 128])
@pytest.mark.parametrize("init", ["zero", "normal"])
def test_kda_chunked_prefill(la, T, dv, init):
    """Chunked KDA against the oracle: tails inside a 16-token sub-chunk and
    inside a chunk, several chunks, every value width."""
    p = workloads.make_problem("kda", 2, T, 3, 128, dv, seed=T + 7 * dv, init_state=init)
    check(p, *run_gpu(la, p), TOL_BF16)


def test_kda_chunked_split_carries_state(la):
    """Prefill [0, 3000) then [3000, T) from the carried state equals the whole
    sequence (and the oracle); the split falls inside a chunk and a sub-chunk."""
    p = workloads.make_problem("kda", 2, 4100, 4, 128, 128, seed=44, init_state="normal")
    t = to_dev(p)
    cut = 3000
    part = lambda x, a, b: x[:, a:b].contiguous()
    args = lambda a, b: [part(t[n], a, b) for n in ("q", "k", "v", "g", "beta")]
    o1, S1, _ = la.fwd("kda", *args(0, cut), S0=t["S0"])
    o2, S2, _ = la.fwd("kda", *args(cut, 4100), S0=S1)
    torch.cuda.synchronize()
    la.check_device()
    o = torch.cat([o1, o2], dim=1).float().cpu().numpy()
    check(p, o, S2.cpu().numpy(), None, TOL_BF16)


def test_kda_chunked_bench_shape_sampled(la):
    """B=2, H=16, T=8192, d=128 (the benchmark's KDA prefill) in one call, checked
    on batch 0 head 0, batch 1 head 15 and batch 1 head 7."""
    from test_gpu_parity import sub_heads
    p = workloads.make_problem("kda", 2, 8192, 16, 128, 128, seed=0)
    o, S, _ = run_gpu(la, p)
    for b, h in ((0, 0), (1, 15), (1, 7)):
        check(p, o, S, None, TOL_BF16, heads=([b], [h]))


def test_kda_chunked_host_buffers(la):
    p = workloads.make_problem("kda", 2, 300, 3, 128, 64, seed=9, init_state="normal")
    t = to_dev(p)
    o_d, S_d, _ = la.fwd("kda", t["q"], t["k"], t["v"], t["g"], t["beta"], t["S0"])
    pin = lambda x: x.pin_memory()
    hq, hk, hv, hg, hb, hS = (pin(x) for x in (p.q, p.k, p.v, p.g, p.beta, p.S0))
    o = torch.empty(2, 300, 3, 64, dtype=torch.bfloat16).pin_memory()
    S = torch.empty(2, 3, 128, 64).pin_memory()
    n = la.host_staging_size("kda", hq, hk, hv, hg, hb, hS)
    staging = torch.empty(n, dtype=torch.uint8, device="cuda")
    la.fwd_host("kda", hq, hk, hv, hg, hb, hS, o=o, S_out=S, staging=staging)
    torch.cuda.synchronize()
    assert torch.equal(o, o_d.cpu())
    assert torch.equal(S, S_d.cpu())


def test_kda_range_error_reported(la):
    """Retention whose 8-token product falls below 2^-60 (alpha = 1e-4 on every
    channel) is outside the chunked kernel's domain: la_check_device reports
    LA_ERR_RANGE instead of returning silently wrong results."""
    p = workloads.make_problem("kda", 1, 64, 1, 128, 32, seed=3)
    t = to_dev(p)
    g = torch.full_like(t["g"], 1e-4)
    la.fwd("kda", t["q"], t["k"], t["v"], g, t["beta"])
    with pytest.raises(la.LAError) as ei:
        la.check_device()
    assert ei.value.status == 6
    la.check_device()  # the word was cleared
