"""Host-side checks of the C ABI (no GPU needed, no kernel launched).

* the library loads and exports every function ``include/*.h`` declares;
* invalid arguments are rejected on the host with the documented status codes
  before anything is launched (the pointers below are never dereferenced).
"""
import ctypes
import glob
import os
import re

import pytest

import gated_delta_rule_attn_b200 as la
from gated_delta_rule_attn_b200 import build as la_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    la_build.build()
    return la.lib()


def declared_functions():
    text = "".join(open(p).read() for p in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))))
    return sorted(set(re.findall(r"^\s*(?:la_status|const char \*|int)\s*(la_\w+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(L, n), n
    assert sorted(la.EXPORTS) == names


def test_abi_version_and_status_strings(L):
    assert L.la_abi_version() == 3
    assert L.la_status_string(0) == b"LA_OK"
    assert L.la_status_string(5) == b"LA_ERR_TIMEOUT"
    assert L.la_status_string(99) == b"LA_ERR_UNKNOWN"


FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced


def args(rule="gdn", dtype=1, B=1, T=8, H=2, dk=128, dv=128, **kw):
    a = la.FwdArgs()
    a.struct_size = ctypes.sizeof(a)
    a.rule, a.dtype = la.RULES[rule], dtype
    a.B, a.T, a.H, a.dk, a.dv = B, T, H, dk, dv
    a.q = a.k = a.v = a.o = FAKE
    if rule == "gla":
        a.g = FAKE
    if rule == "gdn":
        a.g = a.beta = FAKE
    a.eps = 1e-6
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def call(L, a):
    return L.la_fwd(ctypes.byref(a), None), L.la_last_error_message().decode()


@pytest.mark.parametrize("kw,status", [
    (dict(dk=48), 2), (dict(dv=256), 2), (dict(dk=16), 2),
    (dict(B=0), 1), (dict(H=0), 1), (dict(T=-1), 1),
    (dict(rule_raw=7), 1), (dict(dtype=5), 1),
    (dict(q=None), 1), (dict(o=None), 1),
    (dict(q=FAKE + 8), 3), (dict(S0=FAKE + 4), 3), (dict(S_out=FAKE + 2), 3),
    (dict(beta=None), 1), (dict(struct_size=8), 1), (dict(eps=-1.0), 1),
])
def test_invalid_fwd_arguments_rejected(L, kw, status):
    rule_raw = kw.pop("rule_raw", None)
    a = args(**kw)
    if rule_raw is not None:
        a.rule = rule_raw
    r, msg = call(L, a)
    assert r == status, msg
    assert msg


def test_rule_specific_gate_checks(L):
    assert call(L, args("elu", g=FAKE))[0] == 1          # ELU takes no gate
    assert call(L, args("gla", g=None))[0] == 1          # GLA needs g
    assert call(L, args("gla", beta=FAKE))[0] == 1       # GLA takes no beta
    assert call(L, args("gdn", z0=FAKE))[0] == 1         # z is ELU-only


def test_null_args_and_workspace_query(L):
    assert L.la_fwd(None, None) == 1
    n = ctypes.c_size_t(123)
    # gated delta rule, bf16, dk=128: the 8 KB T diag(beta), 8 KB P and 16 KB -U
    # operand images per (batch, head, 64-token chunk)
    assert L.la_fwd_workspace_size(ctypes.byref(args(T=130)), ctypes.byref(n)) == 0
    assert n.value == 1 * 2 * 3 * 32768
    for a in (args("elu"), args(dtype=0), args(dk=64), args(T=0), args("gla", dtype=0)):
        assert L.la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
        assert n.value == 0
    # chunked GLA: one uint32 range flag per (batch, head), in 256-byte units
    assert L.la_fwd_workspace_size(ctypes.byref(args("gla")), ctypes.byref(n)) == 0
    assert n.value == 256
    assert L.la_fwd_workspace_size(ctypes.byref(args("gla", B=9, H=16)), ctypes.byref(n)) == 0
    assert n.value == 768
    assert L.la_fwd_workspace_size(ctypes.byref(args(dk=3)), ctypes.byref(n)) == 2
    # long ELU+1 and GLA sequences over few heads run segment-parallel: the first
    # pass keeps a summary per piece of every segment but the last (dk*dv + dk
    # floats each).  Without a device the library plans for 148 SMs: 4 CTAs of
    # 64 value columns -> 8 segments of 8 chunks, 2 pieces each.
    for rule, flags in (("elu", 0), ("gla", 256)):
        assert L.la_fwd_workspace_size(ctypes.byref(args(rule, T=4096, H=2)), ctypes.byref(n)) == 0
        assert n.value == 1 * 2 * 7 * 2 * (128 * 128 + 128) * 4 + flags


def test_kda_workspace_query():
    """Chunked KDA (bf16, dk = 128, dense): 32.5 KB per (batch, head, 64-token
    chunk) for the images of T diag(beta), P and -U and the chunk's retention
    product, then two bf16 [B,T,H,128] tensors (q times the cumulative
    retention, k times the retention to the chunk's end), each at a 256-byte
    aligned offset.
    fp32 KDA runs on the recurrent kernel and needs none.  Queried through the
    binding, which reads shapes only (CPU tensors)."""
    import torch
    B, T, H = 2, 130, 3
    q = torch.zeros(B, T, H, 128, dtype=torch.bfloat16)
    v = torch.zeros(B, T, H, 64, dtype=torch.bfloat16)
    g = torch.ones(B, T, H, 128)
    beta = torch.zeros(B, T, H)
    up = lambda x: (x + 255) // 256 * 256
    items = up(B * H * 3 * (32768 + 512))
    tensor = up(B * T * H * 128 * 2)
    assert la.fwd_workspace_size("kda", q, q, v, g, beta) == items + 2 * tensor
    assert la.fwd_workspace_size("kda", q.float(), q.float(), v.float(), g, beta) == 0


def test_step_validation(L):
    s = la.StepArgs()
    s.struct_size = ctypes.sizeof(s)
    s.rule, s.dtype, s.N, s.H, s.dk, s.dv = 2, 1, 4, 2, 128, 128
    s.q = s.k = s.v = s.o = s.S = s.g = FAKE
    assert L.la_step(ctypes.byref(s), None) == 1           # GDN needs beta
    s.beta = FAKE + 1
    assert L.la_step(ctypes.byref(s), None) == 3           # misaligned
    s.rule, s.g, s.beta = 0, None, None
    assert L.la_step(ctypes.byref(s), None) == 1           # ELU decode needs z
    s.z, s.dk = FAKE, 100
    assert L.la_step(ctypes.byref(s), None) == 2


def test_missing_workspace_rejected_before_launch(L):
    # the workspace check happens on the host, before anything is launched
    assert call(L, args(T=64))[0] == 8
    assert call(L, args(T=64, workspace=FAKE, workspace_bytes=100))[0] == 8


def test_host_staging_layout(L):
    a = args("gla", B=2, T=100, H=3, dk=64, dv=32, S0=FAKE, S_out=FAKE)
    n = ctypes.c_size_t()
    assert L.la_fwd_host_staging_size(ctypes.byref(a), ctypes.byref(n)) == 0
    tok = 2 * 100 * 3
    parts = [tok * 64 * 2, tok * 64 * 2, tok * 32 * 2, tok * 64 * 4, 0, 2 * 3 * 64 * 32 * 4, 0,
             tok * 32 * 2, 2 * 3 * 64 * 32 * 4, 0]
    assert n.value == sum((p + 255) // 256 * 256 for p in parts)
    # a misaligned staging buffer is refused before any copy
    assert L.la_fwd_host(ctypes.byref(a), ctypes.c_void_p(FAKE + 16), n.value, None) == 3
    assert L.la_fwd_host(ctypes.byref(a), ctypes.c_void_p(FAKE), n.value - 1, None) == 8


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 1, 32, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        la.fwd("elu", q, q, q)


# ---------------------------------------------------------------------------
# Packed variable-length sequences (la_fwd_args fields of ABI version 2)
# ---------------------------------------------------------------------------

def test_version1_struct_size_still_accepted(L):
    """A caller built against the version-1 header passes the smaller struct
    (without cu_seqlens / max_seqlen) and gets the dense layout."""
    a = args(T=130)
    a.struct_size = la.FwdArgs.cu_seqlens.offset
    a.cu_seqlens = 0xDEAD   # past the caller's struct: must be ignored
    n = ctypes.c_size_t(0)
    assert L.la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 1 * 2 * 3 * 32768
    a.struct_size = la.FwdArgs.cu_seqlens.offset - 8
    assert L.la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 1


def test_packed_workspace_follows_max_seqlen(L):
    """Gated delta rule: the 32 KB of operand images per (sequence, head,
    64-token chunk of the longest sequence); packed ELU+1 runs without segments
    (no workspace)."""
    n = ctypes.c_size_t(0)
    a = args(B=5, T=1000, H=2, cu_seqlens=FAKE, max_seqlen=300)
    assert L.la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 5 * 2 * 5 * 32768
    a = args("elu", B=1, T=40000, H=2, cu_seqlens=FAKE, max_seqlen=40000)
    assert L.la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    assert n.value == 0


def test_packed_argument_checks(L):
    bad_len = args(B=3, T=100, cu_seqlens=FAKE, max_seqlen=101)
    assert L.la_fwd(ctypes.byref(bad_len), None) == 1
    assert b"max_seqlen" in L.la_last_error_message()
    neg = args(B=3, T=100, cu_seqlens=FAKE, max_seqlen=-1)
    assert L.la_fwd(ctypes.byref(neg), None) == 1
    mis = args(B=3, T=100, cu_seqlens=FAKE + 4, max_seqlen=50)
    assert L.la_fwd(ctypes.byref(mis), None) == 3
    # host buffers: packed sequences are not offered on la_fwd_host
    h = args(B=3, T=100, cu_seqlens=FAKE, max_seqlen=50)
    n = ctypes.c_size_t(0)
    assert L.la_fwd_host_staging_size(ctypes.byref(h), ctypes.byref(n)) == 2
    assert L.la_fwd_host(ctypes.byref(h), ctypes.c_void_p(FAKE), 1 << 30, None) == 2
    assert b"la_fwd" in L.la_last_error_message()


# ---------------------------------------------------------------------------
# Output normalisation (la_fwd_args / la_step_args fields of ABI version 3)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("kw,status,word", [
    (dict(out_norm=2), 1, "out_norm"),
    (dict(out_norm=1, norm_eps=0.0), 1, "norm_eps"),
    (dict(out_norm=1, norm_eps=-1e-6), 1, "norm_eps"),
    (dict(out_norm=1, norm_eps=float("inf")), 1, "norm_eps"),
    (dict(out_norm=1, norm_eps=float("nan")), 1, "norm_eps"),
    (dict(out_norm=1, norm_eps=1e-6, norm_w=FAKE + 4), 3, "aligned"),
])
def test_invalid_norm_arguments_rejected(L, kw, status, word):
    r, msg = call(L, args("gla", T=8, **kw))
    assert r == status and word in msg, msg


def test_norm_fields_ignored_when_off_or_past_an_older_struct(L):
    n = ctypes.c_size_t(7)
    # out_norm = 0: norm_eps and norm_w are not looked at
    a = args("gla", T=8, norm_eps=-5.0, norm_w=FAKE + 4)
    assert L.la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
    # a version-2 caller's struct ends before out_norm: garbage there is ignored
    a = args("gla", T=8, out_norm=9)
    a.struct_size = la.FwdArgs.out_norm.offset
    assert L.la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0


def step_args(**kw):
    s = la.StepArgs()
    s.struct_size = ctypes.sizeof(s)
    s.rule, s.dtype, s.N, s.H, s.dk, s.dv = 2, 1, 4, 2, 128, 128
    s.q = s.k = s.v = s.o = s.S = s.g = FAKE
    for k, v in kw.items():
        setattr(s, k, v)
    return s


def test_step_struct_versions_and_norm_checks(L):
    # version-2 struct (ends at o): accepted, validation goes on (GDN needs beta)
    s = step_args(out_norm=9)
    s.struct_size = la.StepArgs.out_norm.offset
    assert L.la_step(ctypes.byref(s), None) == 1
    assert b"beta" in L.la_last_error_message()
    s.struct_size = la.StepArgs.out_norm.offset - 8
    assert L.la_step(ctypes.byref(s), None) == 1
    assert b"struct_size" in L.la_last_error_message()
    # full struct: the norm fields are checked
    s = step_args(beta=FAKE, out_norm=1, norm_eps=0.0)
    assert L.la_step(ctypes.byref(s), None) == 1
    assert b"norm_eps" in L.la_last_error_message()
    s = step_args(beta=FAKE, out_norm=1, norm_eps=1e-6, norm_w=FAKE + 8)
    assert L.la_step(ctypes.byref(s), None) == 3


def test_host_staging_holds_the_norm_weight(L):
    a = args("gla", B=2, T=100, H=3, dk=64, dv=32, S0=FAKE, S_out=FAKE)
    n0, n1 = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.la_fwd_host_staging_size(ctypes.byref(a), ctypes.byref(n0)) == 0
    a.out_norm, a.norm_eps, a.norm_w = 1, 1e-6, FAKE + 4   # host pointer: no alignment rule
    assert L.la_fwd_host_staging_size(ctypes.byref(a), ctypes.byref(n1)) == 0
    assert n1.value == n0.value + 256   # 32 fp32 weights, padded to 256 bytes
    a.norm_w = None
    assert L.la_fwd_host_staging_size(ctypes.byref(a), ctypes.byref(n1)) == 0
    assert n1.value == n0.value
