"""Packed variable-length sequences (cu_seqlens): several sequences of different
lengths on one token axis, each starting from its own initial state (the state
reset at sequence boundaries of page "状态空间与线性注意力", 验证矩阵 / Shape 与
实现契约).

Checked against the fp64 oracle run on every sequence alone, and against the
library's own dense call on every sequence alone: the chunked kernels start
chunks at each sequence's first token, so a packed run does exactly the dense
run's arithmetic and the results must agree bit for bit.  Offsets that are out
of order, out of range or longer than max_seqlen are clamped on the device (no
access leaves the tensors) and reported by la_check_device.  KDA's chunked path
keeps its scaled q/k in one row block per sequence (the tail chunk's padding
rows zero), so it too matches its dense calls bit for bit.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from test_gpu_parity import TOL_BF16, TOL_F32, la, rel_err  # noqa: F401

pytestmark = pytest.mark.gpu

LENGTHS = [1, 64, 0, 65, 200, 517, 3, 128]


def packed_problem(rule, lengths, H, dk, dv, dtype, seed):
    """One dense problem per sequence (B=1 each, own S0), and their packing."""
    parts = [workloads.make_problem(rule, 1, L, H, dk, dv, dtype=dtype, seed=seed + i, init_state="normal")
             for i, L in enumerate(lengths)]
    cat = lambda name: (None if getattr(parts[0], name) is None
                        else torch.cat([getattr(p, name) for p in parts], dim=1).contiguous())
    S0 = torch.cat([p.S0 for p in parts], dim=0).contiguous()
    z0 = None if parts[0].z0 is None else torch.cat([p.z0 for p in parts], dim=0).contiguous()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int64)
    packed = dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"), S0=S0, z0=z0)
    return parts, packed, cu


def run_packed(la, rule, packed, cu, max_seqlen):
    d = {n: (None if t is None else t.cuda()) for n, t in packed.items()}
    o, S, z = la.fwd(rule, d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["z0"], 1e-6,
                     cu_seqlens=cu.cuda(), max_seqlen=max_seqlen)
    torch.cuda.synchronize()
    la.check_device()
    return o, S, z


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn", "kda"])
@pytest.mark.parametrize("dk,dv,dtype", [(128, 64, torch.bfloat16), (128, 128, torch.bfloat16),
                                         (32, 32, torch.float32), (64, 32, torch.bfloat16)])
def test_packed_matches_oracle_per_sequence(la, rule, dk, dv, dtype):
    parts, packed, cu = packed_problem(rule, LENGTHS, 3, dk, dv, dtype, seed=40 + dk + dv)
    o, S, z = run_packed(la, rule, packed, cu, max(LENGTHS))
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    o = o.float().cpu().numpy()
    for i, p in enumerate(parts):
        ro, rS, rz = oracle.fwd(p)
        s0, s1 = int(cu[i]), int(cu[i + 1])
        if s1 > s0:
            assert rel_err(o[:, s0:s1], ro) <= tol, f"sequence {i} (length {s1 - s0}): o"
        assert rel_err(S[i:i + 1].cpu().numpy(), rS) <= tol, f"sequence {i}: S"
        if rz is not None:
            assert rel_err(z[i:i + 1].cpu().numpy(), rz) <= tol, f"sequence {i}: z"


@pytest.mark.parametrize("rule", ["elu", "gla", "gdn", "kda"])
def test_packed_equals_dense_calls_bitwise(la, rule):
    """Chunked tensor-core path (bf16, dk = 128): every sequence's outputs and
    final state are bit-identical to a dense call on that sequence alone."""
    parts, packed, cu = packed_problem(rule, LENGTHS, 2, 128, 128, torch.bfloat16, seed=77)
    o, S, z = run_packed(la, rule, packed, cu, max(LENGTHS))
    for i, p in enumerate(parts):
        d = {n: (None if getattr(p, n) is None else getattr(p, n).cuda())
             for n in ("q", "k", "v", "g", "beta", "S0", "z0")}
        od, Sd, zd = la.fwd(rule, d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], d["z0"], 1e-6)
        s0, s1 = int(cu[i]), int(cu[i + 1])
        assert torch.equal(o[:, s0:s1], od), f"sequence {i}: o differs from the dense call"
        assert torch.equal(S[i:i + 1], Sd), f"sequence {i}: S differs from the dense call"
        if zd is not None:
            assert torch.equal(z[i:i + 1], zd), f"sequence {i}: z differs from the dense call"


@pytest.mark.parametrize("rule", ["gla", "gdn", "kda"])
def test_packed_many_sequences_full_width(la, rule):
    """Sixteen heads and 24 sequences of mixed lengths (the decode-batch shape
    of a serving prefill), checked on a few sequences."""
    rng = np.random.default_rng(5)
    lengths = [int(x) for x in rng.integers(0, 700, size=24)]
    parts, packed, cu = packed_problem(rule, lengths, 16, 128, 128, torch.bfloat16, seed=500)
    o, S, _ = run_packed(la, rule, packed, cu, max(lengths))
    o = o.float().cpu().numpy()
    for i in (0, 7, 23):
        ro, rS, _ = oracle.fwd(parts[i])
        s0, s1 = int(cu[i]), int(cu[i + 1])
        if s1 > s0:
            assert rel_err(o[:, s0:s1], ro) <= TOL_BF16
        assert rel_err(S[i:i + 1].cpu().numpy(), rS) <= TOL_BF16


@pytest.mark.parametrize("rule", ["gla", "gdn", "kda"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_bad_offsets_are_clamped_and_reported(la, rule, dtype):
    """Offsets out of order and beyond T, and a sequence longer than max_seqlen:
    every access stays inside the tensors (offsets clamped into [0, T], lengths
    to max_seqlen) and la_check_device reports LA_ERR_INVALID_ARG."""
    T, H = 300, 2
    p = workloads.make_problem(rule, 1, T, H, 128, 64, dtype=dtype, seed=3, init_state="normal")
    cu = torch.tensor([0, 120, 90, 400], dtype=torch.int64, device="cuda")   # 3 sequences
    S0 = torch.zeros(3, H, 128, 64, device="cuda")
    d = {n: (None if getattr(p, n) is None else getattr(p, n).cuda()) for n in ("q", "k", "v", "g", "beta")}
    la.fwd(rule, d["q"], d["k"], d["v"], d["g"], d["beta"], S0, cu_seqlens=cu, max_seqlen=100)
    torch.cuda.synchronize()
    with pytest.raises(la.LAError) as e:
        la.check_device()
    assert "cu_seqlens" in str(e.value)
    la.check_device()   # the error word was cleared
