"""Causal linear attention (ELU+1 / GLA / gated delta rule) for B200.

Thin Python binding over the C ABI in ``include/la.h``: it only checks tensor
properties, allocates outputs with PyTorch and passes pointers, sizes and the
current CUDA stream to ``libla_b200.so``.  Every step of the computation runs in
the library's CUDA kernels; there is no CPU path.  If the library is missing
the import of the binding raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libla_b200.so")
ABI_VERSION = 3   # LA_ABI_VERSION of include/la.h that these struct layouts follow

RULES = {"elu": 0, "gla": 1, "gdn": 2, "kda": 3}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}
STATUS = {0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED", 3: "LA_ERR_ALIGNMENT",
          4: "LA_ERR_CUDA", 5: "LA_ERR_TIMEOUT", 6: "LA_ERR_RANGE", 7: "LA_ERR_INTERNAL",
          8: "LA_ERR_WORKSPACE"}

# Symbols include/la.h and include/la_testing.h declare (checked by the CPU test suite).
EXPORTS = ("la_fwd", "la_fwd_workspace_size", "la_step", "la_fwd_host_staging_size",
           "la_fwd_host", "la_check_device", "la_status_string", "la_last_error_message",
           "la_abi_version", "la_fwd_noalloc", "la_testing_set_wait_limit")


class LAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class FwdArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("rule", ctypes.c_int), ("dtype", ctypes.c_int),
                ("B", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int64),
                ("dk", ctypes.c_int64), ("dv", ctypes.c_int64),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("S0", ctypes.c_void_p),
                ("z0", ctypes.c_void_p), ("eps", ctypes.c_float), ("o", ctypes.c_void_p),
                ("S_out", ctypes.c_void_p), ("z_out", ctypes.c_void_p),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
                ("cu_seqlens", ctypes.c_void_p), ("max_seqlen", ctypes.c_int64),
                ("out_norm", ctypes.c_int32), ("norm_eps", ctypes.c_float), ("norm_w", ctypes.c_void_p)]


class StepArgs(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("rule", ctypes.c_int), ("dtype", ctypes.c_int),
                ("N", ctypes.c_int64), ("H", ctypes.c_int64), ("dk", ctypes.c_int64),
                ("dv", ctypes.c_int64),
                ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("g", ctypes.c_void_p), ("beta", ctypes.c_void_p), ("S", ctypes.c_void_p),
                ("z", ctypes.c_void_p), ("eps", ctypes.c_float), ("o", ctypes.c_void_p),
                ("out_norm", ctypes.c_int32), ("norm_eps", ctypes.c_float), ("norm_w", ctypes.c_void_p)]


_lib = None


def lib():
    """Load ``libla_b200.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python gated_delta_rule_attn_b200/build.py` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        L.la_fwd.argtypes = [ctypes.POINTER(FwdArgs), P]
        L.la_fwd_workspace_size.argtypes = [ctypes.POINTER(FwdArgs), ctypes.POINTER(ctypes.c_size_t)]
        L.la_step.argtypes = [ctypes.POINTER(StepArgs), P]
        L.la_fwd_host_staging_size.argtypes = [ctypes.POINTER(FwdArgs), ctypes.POINTER(ctypes.c_size_t)]
        L.la_fwd_host.argtypes = [ctypes.POINTER(FwdArgs), P, ctypes.c_size_t, P]
        L.la_check_device.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
        L.la_fwd_noalloc.argtypes = [ctypes.POINTER(FwdArgs), P]
        L.la_testing_set_wait_limit.argtypes = [ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
        L.la_testing_set_wait_limit.restype = ctypes.c_int
        L.la_status_string.argtypes = [ctypes.c_int]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_last_error_message.restype = ctypes.c_char_p
        for f in (L.la_fwd, L.la_fwd_workspace_size, L.la_step, L.la_fwd_host_staging_size,
                  L.la_fwd_host, L.la_check_device, L.la_fwd_noalloc):
            f.restype = ctypes.c_int
        L.la_abi_version.restype = ctypes.c_int
        if L.la_abi_version() != ABI_VERSION:
            raise ImportError(f"{LIB_PATH} has ABI version {L.la_abi_version()}, the binding expects "
                              f"{ABI_VERSION}: rebuild it")
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise LAError(status, lib().la_last_error_message().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, device=True):
    if t is None:
        return
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _set_norm(a, out_norm, norm_w, norm_eps):
    """Output normalisation fields (la.h, ABI version 3)."""
    a.out_norm = 1 if out_norm else 0
    a.norm_eps = norm_eps
    a.norm_w = norm_w.data_ptr() if norm_w is not None else None


def make_fwd_args(rule, q, k, v, g=None, beta=None, S0=None, z0=None, eps=1e-6,
                  o=None, S_out=None, z_out=None, cu_seqlens=None, max_seqlen=None,
                  out_norm=False, norm_w=None, norm_eps=1e-6) -> FwdArgs:
    """Marshal tensors into la_fwd_args.  With ``cu_seqlens`` (int64 [B+1] on the
    device) the token tensors are one packed axis [1, T, H, d] and B is the
    number of sequences; ``max_seqlen`` bounds their lengths.  ``out_norm``:
    each (token, head) row of o is RMS-normalised over dv (weight ``norm_w``
    fp32 [dv] or None, ``norm_eps`` > 0)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("packed sequences take q, k, v as [1, T, H, d]")
        if cu_seqlens.dtype != torch.int64 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int64 tensor")
        B = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("packed sequences need max_seqlen")
    a = FwdArgs()
    a.struct_size = ctypes.sizeof(FwdArgs)
    a.rule = RULES[rule]
    a.dtype = DTYPES[q.dtype]
    a.B, a.T, a.H, a.dk, a.dv = B, T, H, dk, dv
    a.q, a.k, a.v, a.g, a.beta = (t.data_ptr() if t is not None else None for t in (q, k, v, g, beta))
    a.S0 = S0.data_ptr() if S0 is not None else None
    a.z0 = z0.data_ptr() if z0 is not None else None
    a.eps = eps
    a.o = o.data_ptr() if o is not None else None
    a.S_out = S_out.data_ptr() if S_out is not None else None
    a.z_out = z_out.data_ptr() if z_out is not None else None
    if cu_seqlens is not None:
        a.cu_seqlens = cu_seqlens.data_ptr()
        a.max_seqlen = int(max_seqlen)
    _set_norm(a, out_norm, norm_w, norm_eps)
    return a


_WORKSPACES = {}


def _workspace(device, stream, nbytes: int):
    """Scratch for la_fwd, cached per (device, stream): calls on one stream are
    ordered, so they can share it.  It is allocated with that stream current, so
    that when a larger one replaces it, the allocator reuses the old block only
    for work ordered after the kernels that used it."""
    key = (device.index, stream.cuda_stream)
    ws = _WORKSPACES.get(key)
    if ws is None or ws.numel() < nbytes:
        with torch.cuda.stream(stream):
            ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
        _WORKSPACES[key] = ws
    return ws


def fwd(rule: str, q, k, v, g=None, beta=None, S0=None, z0=None, eps: float = 1e-6,
        o=None, S_out=None, z_out=None, stream=None, want_state: bool = True, workspace=None,
        cu_seqlens=None, max_seqlen=None, out_norm: bool = False, norm_w=None, norm_eps: float = 1e-6):
    """Chunked prefill: returns (o, S_out, z_out-or-None). Enqueued on the current stream.

    ``workspace`` (a CUDA uint8 tensor of at least ``fwd_workspace_size`` bytes)
    is allocated and cached per stream when not given.  ``cu_seqlens`` /
    ``max_seqlen``: packed variable-length sequences (see ``make_fwd_args``);
    the states are then [number of sequences, H, dk, dv].  ``out_norm``,
    ``norm_w``, ``norm_eps``: head-wise RMS normalisation of o (see
    ``make_fwd_args``)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta"), (S0, "S0"), (z0, "z0"),
                 (cu_seqlens, "cu_seqlens"), (norm_w, "norm_w")):
        _need(t, n)
    NS = B if cu_seqlens is None else cu_seqlens.numel() - 1   # sequences (state rows)
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise ValueError("q, k, v must share a dtype")
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=q.dtype, device=q.device)
    if S_out is None and want_state:
        S_out = torch.empty(NS, H, dk, dv, dtype=torch.float32, device=q.device)
    if rule == "elu" and z_out is None and want_state:
        z_out = torch.empty(NS, H, dk, dtype=torch.float32, device=q.device)
    a = make_fwd_args(rule, q, k, v, g, beta, S0, z0, eps, o, S_out, z_out, cu_seqlens, max_seqlen,
                      out_norm, norm_w, norm_eps)
    st = stream if stream is not None else torch.cuda.current_stream(q.device)
    sh = _stream_handle(st)
    n = ctypes.c_size_t()
    _check(lib().la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    if n.value:
        ws = workspace if workspace is not None else _workspace(q.device, st, n.value)
        a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    _check(lib().la_fwd(ctypes.byref(a), sh))
    return o, S_out, z_out


def fwd_workspace_size(rule, q, k, v, g=None, beta=None, S0=None, z0=None) -> int:
    """Bytes of workspace ``fwd`` needs for these inputs (shapes only are read)."""
    a = make_fwd_args(rule, q, k, v, g, beta, S0, z0)
    # the query validates the arguments as la_fwd does, which needs a non-NULL o;
    # no data is touched, so q's address stands in for it
    a.o = a.q
    n = ctypes.c_size_t()
    _check(lib().la_fwd_workspace_size(ctypes.byref(a), ctypes.byref(n)))
    return n.value


def step(rule: str, q, k, v, S, z=None, g=None, beta=None, eps: float = 1e-6, o=None,
         stream=None, out_norm: bool = False, norm_w=None, norm_eps: float = 1e-6):
    """Decode step: updates S (and z) in place, returns o [N,H,dv] (RMS-normalised
    per (sequence, head) over dv with ``out_norm``)."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta"), (S, "S"), (z, "z"),
                 (norm_w, "norm_w")):
        _need(t, n)
    if o is None:
        o = torch.empty(N, H, dv, dtype=q.dtype, device=q.device)
    a = StepArgs()
    a.struct_size = ctypes.sizeof(StepArgs)
    a.rule = RULES[rule]
    a.dtype = DTYPES[q.dtype]
    a.N, a.H, a.dk, a.dv = N, H, dk, dv
    a.q, a.k, a.v, a.g, a.beta, a.S, a.z = (t.data_ptr() if t is not None else None
                                            for t in (q, k, v, g, beta, S, z))
    a.eps = eps
    a.o = o.data_ptr()
    _set_norm(a, out_norm, norm_w, norm_eps)
    _check(lib().la_step(ctypes.byref(a), _stream_handle(stream)))
    return o


def host_staging_size(rule, q, k, v, g=None, beta=None, S0=None, z0=None, want_state=True,
                      out_norm=False, norm_w=None, norm_eps=1e-6) -> int:
    """Bytes of device staging ``fwd_host`` needs for these host tensors."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    a = make_fwd_args(rule, q, k, v, g, beta, S0, z0, out_norm=out_norm, norm_w=norm_w, norm_eps=norm_eps)
    # output pointers only mark presence for the size computation
    a.o = 1
    a.S_out = 1 if want_state else None
    a.z_out = 1 if (want_state and rule == "elu") else None
    n = ctypes.c_size_t()
    _check(lib().la_fwd_host_staging_size(ctypes.byref(a), ctypes.byref(n)))
    return n.value


def fwd_host(rule: str, q, k, v, g=None, beta=None, S0=None, z0=None, eps: float = 1e-6,
             o=None, S_out=None, z_out=None, staging=None, stream=None,
             out_norm: bool = False, norm_w=None, norm_eps: float = 1e-6):
    """la_fwd on host (CPU, ideally pinned) tensors through the C ABI: the library
    copies inputs into ``staging`` (a CUDA uint8 tensor), runs, copies outputs back
    and synchronises the stream.  Returns (o, S_out, z_out)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (g, "g"), (beta, "beta"), (S0, "S0"), (z0, "z0"),
                 (o, "o"), (S_out, "S_out"), (z_out, "z_out"), (norm_w, "norm_w")):
        _need(t, n, device=False)
    a = make_fwd_args(rule, q, k, v, g, beta, S0, z0, eps, o, S_out, z_out,
                      out_norm=out_norm, norm_w=norm_w, norm_eps=norm_eps)
    _check(lib().la_fwd_host(ctypes.byref(a), ctypes.c_void_p(staging.data_ptr()),
                             staging.numel(), _stream_handle(stream)))
    return o, S_out, z_out


def check_device(stream=None) -> int:
    """Synchronise and read/clear the device error word; raises on a recorded error."""
    flags = ctypes.c_uint32()
    _check(lib().la_check_device(_stream_handle(stream), ctypes.byref(flags)))
    return flags.value


def abi_version() -> int:
    return lib().la_abi_version()
