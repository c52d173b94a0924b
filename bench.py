"""Benchmark of the causal linear-attention hot path on B200.

One step = one pass of every part of the path over one batch of synthetic
input, each part a separate library call on the current stream:
  * GLA prefill        B=2, H=16, T=8192, dk=dv=128  (gate per key dim)
  * gated-delta prefill B=2, H=16, T=8192, dk=dv=128
  * ELU+1 prefill      B=1, H=16, T=32768, dk=128, dv=64 (state carry-in)
  * one GLA and one gated-delta decode step on a [256,16,128,128] fp32 state
``value`` is the prefill throughput of the GLA + gated-delta pair at d=128,
T=8192 (tokens = B*T, both calls), from the device time of those two calls;
the other parts are reported per leg (decode as state GB/s).

Timing: W warm-up steps, then K steps between a barrier + synchronize on both
sides, CUDA events on the launching stream around every leg; multi-GPU runs are
weak-scaled (every rank runs the same step on its own GPU, no collective on the
data path) and the time is the max over ranks.  Every leg's inputs are larger
than the 126 MB L2, so nothing stays cached between reuses.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s + % roofline (GLA/GDN d=128 T=8192); decode state GB/s"
CHUNK = 64  # chunk length of the tensor-core kernels (for the algorithmic FLOP count)


# ---------------------------------------------------------------------------
# Algorithmic work (bytes each input read once / output written once; MACs of
# the chunkwise method counting only causally needed products)
# ---------------------------------------------------------------------------

def update_macs(N: int, dk: int, dv: int) -> int:
    """The state-update term alone: N * dk * dv multiply-adds per head (the hand
    count of page "线性注意力与 SSM", §02: N=32768, dphi=128, dv=64 -> ~2.684e8)."""
    return N * dk * dv


def macs_per_token_head(rule: str, dk: int, dv: int, C: int = CHUNK) -> float:
    P = C * (C + 1) / 2
    if rule == "elu":
        return (P * dk + P * (dv + 1)) / C + 2 * dk * (dv + 1)
    base = P * (dk + dv) / C + 2 * dk * dv
    if rule == "gla":
        return base
    return base + (C - 1) / 2 * dk + (C - 1) / 2 * (dk + dv) + dk * dv


def prefill_bytes(rule: str, B: int, T: int, H: int, dk: int, dv: int, esize: int = 2,
                  with_S0: bool = False, with_z: bool = False) -> int:
    tok = B * T * H
    b = tok * (2 * dk + 2 * dv) * esize              # q, k, v read; o written
    if rule == "gla":
        b += tok * dk * 4                            # gate
    elif rule == "gdn":
        b += tok * 2 * 4                             # alpha, beta
    b += B * H * dk * dv * 4 * (2 if with_S0 else 1)  # S0 read (if given), S_out written
    if with_z:
        b += B * H * dk * 4 * 2
    return b


def decode_bytes(rule: str, N: int, H: int, dk: int, dv: int) -> int:
    b = N * H * dk * dv * 4 * 2                     # state read + written
    b += N * H * (2 * dk + 2 * dv) * 2               # q, k, v, o bf16
    b += N * H * (dk * 4 if rule == "gla" else 8)    # gates
    return b


def prefill_flops(rule: str, B: int, T: int, H: int, dk: int, dv: int) -> float:
    return 2.0 * macs_per_token_head(rule, dk, dv) * B * T * H


# ---------------------------------------------------------------------------
# Peaks, clocks, traffic records
# ---------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# The csrc files behind each leg's kernels and their launches: a leg's DRAM
# traffic record stays valid while these files are unchanged.
LEG_SOURCES = {
    "gla_prefill": ["device.cuh", "chunk_tc.cuh", "chunk_ge.cuh", "chunk_agg.cuh", "recurrent.cuh", "la.cu"],
    "elu_prefill": ["device.cuh", "chunk_tc.cuh", "chunk_ge.cuh", "chunk_agg.cuh", "la.cu"],
    "gdn_prefill": ["device.cuh", "chunk_tc.cuh", "chunk_gdn.cuh", "la.cu"],
    "gla_decode": ["device.cuh", "recurrent.cuh", "la.cu"],
    "gdn_decode": ["device.cuh", "recurrent.cuh", "la.cu"],
    "kda_prefill": ["device.cuh", "chunk_tc.cuh", "chunk_gdn.cuh", "chunk_kda.cuh", "la.cu"],
}


def kernel_source_hash(files=None) -> str:
    """sha256 (first 16 hex digits) over the named csrc files, or all of them."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_attn_b200", "csrc")
    for name in sorted(files if files is not None else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch of each leg from a committed ncu capture; a leg's
    figure is valid only while the sources of its kernels are unchanged since
    the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return {}
    out = {}
    for leg, rec in d.get("legs", {}).items():
        files = LEG_SOURCES.get(leg)
        if files is not None and rec.get("source_hash") == kernel_source_hash(files):
            out[leg] = rec.get("bytes_per_launch")
    return out


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
               "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
               "display_clock_setting": 0x100}

    def __init__(self, index: int, period: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# Workload on the device
# ---------------------------------------------------------------------------

LEG_NAMES = ["gla_prefill", "gdn_prefill", "elu_prefill", "gla_decode", "gdn_decode"]
# kernels per call: gated delta rule 2 (operand images, then the main pass);
# ELU+1 at its shape 2 (summaries of the earlier sequence segments, then the
# segment-parallel main pass); GLA 3 (the same two, then the per-token kernel
# over the sequences the chunked form flagged, launched dependent on the main
# pass and exiting at once when none is flagged); each decode step 1
LEG_LAUNCHES = {"gla_prefill": 3, "gdn_prefill": 2, "elu_prefill": 2, "gla_decode": 1, "gdn_decode": 1,
                "kda_prefill": 2}
# legs that --profile-leg can run but the timed step does not: KDA prefill at the
# prefill benchmark shape (prep kernel, then the KDA main pass)
PROFILE_ONLY_LEGS = ["kda_prefill"]


class Legs:
    """Device inputs and preallocated outputs of the legs in `names` (all by default)."""

    def __init__(self, torch, la, workloads, seed: int, names=None):
        self.torch, self.la = torch, la
        self.names = list(names or LEG_NAMES)
        want = set(self.names)
        dev = lambda t: None if t is None else t.cuda()
        e = torch.empty
        self.host = {}
        if "gla_prefill" in want:
            gla = self.host["gla"] = workloads.gla_prefill(B=2, H=16, T=8192, seed=seed)
            self.gla = {k: dev(getattr(gla, k)) for k in ("q", "k", "v", "g")}
            self.o_gla = e(2, 8192, 16, 128, dtype=torch.bfloat16, device="cuda")
            self.S_gla = e(2, 16, 128, 128, device="cuda")
        if "gdn_prefill" in want:
            gdn = self.host["gdn"] = workloads.gdn_prefill(B=2, H=16, T=8192, seed=seed)
            self.gdn = {k: dev(getattr(gdn, k)) for k in ("q", "k", "v", "g", "beta")}
            self.o_gdn = e(2, 8192, 16, 128, dtype=torch.bfloat16, device="cuda")
            self.S_gdn = e(2, 16, 128, 128, device="cuda")
        if "elu_prefill" in want:
            elu = self.host["elu"] = workloads.elu_long(seed=seed)
            self.elu = {k: dev(getattr(elu, k)) for k in ("q", "k", "v", "S0", "z0")}
            self.o_elu = e(1, 32768, 16, 64, dtype=torch.bfloat16, device="cuda")
            self.S_elu = e(1, 16, 128, 64, device="cuda")
            self.z_elu = e(1, 16, 128, device="cuda")
        if "kda_prefill" in want:
            kda = self.host["kda"] = workloads.make_problem("kda", 2, 8192, 16, 128, 128, seed=seed)
            self.kda = {k: dev(getattr(kda, k)) for k in ("q", "k", "v", "g", "beta")}
            self.o_kda = e(2, 8192, 16, 128, dtype=torch.bfloat16, device="cuda")
            self.S_kda = e(2, 16, 128, 128, device="cuda")
        if want & {"gla_decode", "gdn_decode"}:
            self.S_dec = workloads.decode_state(seed=seed).cuda()
            self.dec_gla = [x.cuda() for x in workloads.decode_steps("gla", 1, seed=seed)[0]]
            self.dec_gdn = [x.cuda() for x in workloads.decode_steps("gdn", 1, seed=seed)[0]]
            self.o_dec = e(256, 16, 128, dtype=torch.bfloat16, device="cuda")
        self.launches_per_step = sum(LEG_LAUNCHES[n] for n in self.names)

    def run(self, name):
        la = self.la
        if name == "gla_prefill":
            a = self.gla
            la.fwd("gla", a["q"], a["k"], a["v"], a["g"], o=self.o_gla, S_out=self.S_gla)
        elif name == "gdn_prefill":
            a = self.gdn
            la.fwd("gdn", a["q"], a["k"], a["v"], a["g"], a["beta"], o=self.o_gdn, S_out=self.S_gdn)
        elif name == "kda_prefill":
            a = self.kda
            la.fwd("kda", a["q"], a["k"], a["v"], a["g"], a["beta"], o=self.o_kda, S_out=self.S_kda)
        elif name == "elu_prefill":
            a = self.elu
            la.fwd("elu", a["q"], a["k"], a["v"], S0=a["S0"], z0=a["z0"], eps=1e-6, o=self.o_elu,
                   S_out=self.S_elu, z_out=self.z_elu)
        elif name == "gla_decode":
            q, k, v, g = self.dec_gla
            la.step("gla", q, k, v, self.S_dec, g=g, o=self.o_dec)
        elif name == "gdn_decode":
            q, k, v, a_, b_ = self.dec_gdn
            la.step("gdn", q, k, v, self.S_dec, g=a_, beta=b_, o=self.o_dec)


def leg_work(name):
    if name == "gla_prefill":
        return dict(tokens=2 * 8192, bytes=prefill_bytes("gla", 2, 8192, 16, 128, 128),
                    flops=prefill_flops("gla", 2, 8192, 16, 128, 128))
    if name == "gdn_prefill":
        return dict(tokens=2 * 8192, bytes=prefill_bytes("gdn", 2, 8192, 16, 128, 128),
                    flops=prefill_flops("gdn", 2, 8192, 16, 128, 128))
    if name == "elu_prefill":
        return dict(tokens=32768, bytes=prefill_bytes("elu", 1, 32768, 16, 128, 64, with_S0=True,
                                                      with_z=True),
                    flops=prefill_flops("elu", 1, 32768, 16, 128, 64))
    rule = name.split("_")[0]
    return dict(tokens=256, bytes=decode_bytes(rule, 256, 16, 128, 128),
                flops=2.0 * 2 * 128 * 128 * 256 * 16)


# ---------------------------------------------------------------------------
# Multi-rank plumbing (one process per GPU; no collective on the data path)
# ---------------------------------------------------------------------------

def max_over_ranks(dist, values, device):
    """Element-wise maximum over all ranks of this rank's device times (ms): the
    job takes as long as its slowest rank.  Identity without a process group."""
    import torch
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_tokens_per_s(world: int, tokens_per_rank: int, ms: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes its own
    tokens_per_rank in the (max over ranks) time ms."""
    return world * tokens_per_rank / (ms / 1e3)


def run_profile_leg(args):
    """One leg only, `--reps` times with no timing: a small, fixed launch
    sequence for ncu captures (3 warm-up calls, then the reps)."""
    import torch

    import gated_delta_rule_attn_b200 as la
    import workloads

    torch.cuda.set_device(0)
    legs = Legs(torch, la, workloads, seed=0, names=[args.profile_leg])
    for _ in range(3 + args.reps):
        legs.run(args.profile_leg)
    torch.cuda.synchronize()
    la.check_device()
    print(json.dumps({"profile_leg": args.profile_leg, "calls": 3 + args.reps,
                      "launches": (3 + args.reps) * LEG_LAUNCHES[args.profile_leg]}), flush=True)


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import gated_delta_rule_attn_b200 as la
    import workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    legs = Legs(torch, la, workloads, seed=rank)
    stream = torch.cuda.current_stream()
    # warm-up (also checks the device error word once)
    for _ in range(max(args.warmup, 3)):
        for n in legs.names:
            legs.run(n)
    torch.cuda.synchronize()
    la.check_device()

    K = args.steps
    ev = {n: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)] for n in legs.names}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(K):
            for n in legs.names:
                ev[n][i][0].record(stream)
                legs.run(n)
                ev[n][i][1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = start.elapsed_time(end)
    leg_ms = {n: sum(a.elapsed_time(b) for a, b in ev[n]) / K for n in legs.names}
    la.check_device()

    # max over ranks
    red = max_over_ranks(dist, [total_ms] + [leg_ms[n] for n in legs.names], "cuda")
    total_ms = red[0]
    leg_ms = {n: red[i + 1] for i, n in enumerate(legs.names)}

    hbm_peak, tc_peak, peak_kind = load_peaks()
    traffic = load_traffic()
    legs_out = {}
    for n in legs.names:
        w = leg_work(n)
        s = leg_ms[n] / 1e3
        gbs = w["bytes"] / s / 1e9
        legs_out[n] = {"ms": round(leg_ms[n], 4), "tokens_per_s": round(w["tokens"] / s),
                       "alg_bytes": w["bytes"], "alg_flops": w["flops"],
                       "gbs": round(gbs, 1), "tflops": round(w["flops"] / s / 1e12, 2),
                       "hbm_frac": round(gbs / hbm_peak, 4)}
    pre = ("gla_prefill", "gdn_prefill")
    pre_ms = sum(leg_ms[n] for n in pre)
    tokens = sum(leg_work(n)["tokens"] for n in pre)
    value = job_tokens_per_s(world, tokens, pre_ms)
    # roofline of the dominant kernel (longest leg)
    dom = max(legs.names, key=lambda n: leg_ms[n])
    w = leg_work(dom)
    ach = w["bytes"] / (leg_ms[dom] / 1e3) / 1e9
    roofline = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak,
                "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "unit": "GB/s", "frac": round(ach / hbm_peak, 4),
                "traffic": traffic.get(dom),
                "tensor_frac": round(w["flops"] / (leg_ms[dom] / 1e3) / 1e12 / tc_peak, 4)}
    # roofline time = max(FLOPs at tensor peak, bytes at HBM peak) for the prefill pair
    t_roof = sum(max(leg_work(n)["flops"] / (tc_peak * 1e12), leg_work(n)["bytes"] / (hbm_peak * 1e9))
                 for n in pre)
    dec_ms = leg_ms["gla_decode"] + leg_ms["gdn_decode"]
    dec_bytes = leg_work("gla_decode")["bytes"] + leg_work("gdn_decode")["bytes"]

    out = {
        "metric": METRIC, "value": round(value), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) q/k/v and gates per the workload recipe in workloads.py; no dataset",
        "config": {"workload": "GLA + gated-delta prefill B=2 H=16 T=8192 dk=dv=128 (value); "
                               "ELU+1 prefill B=1 H=16 T=32768 dk=128 dv=64; GLA + gated-delta "
                               "decode step on state [256,16,128,128] fp32",
                   "global_batch": 2 * world, "seq_len": 8192, "chunk": CHUNK,
                   "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
                   "l2": "inputs larger than L2 (every leg streams > 126 MB between reuses)"},
        "prefill_roofline_frac": round(t_roof / (pre_ms / 1e3), 4),
        "decode_state_gbs": round(dec_bytes / (dec_ms / 1e3) / 1e9, 1),
        "legs": legs_out,
        "roofline": roofline,
        "gpu_launches": legs.launches_per_step * K,
        "clocks": clk.summary(),
    }

    # end to end through the host-buffer entry point (copies inside the timed region)
    out["e2e"] = run_e2e(torch, la, legs, min(K, args.e2e_steps), world)
    if args.variants:
        out["variants"] = run_variants(torch, la, workloads, K, hbm_peak, seed=rank)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def _time_calls(torch, run, K):
    """Mean device time (ms) of K calls of ``run`` after 3 warm-up calls, CUDA
    events on the current stream."""
    for _ in range(3):
        run()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        e0.record(stream)
        run()
        e1.record(stream)
    torch.cuda.synchronize()
    return sum(e0.elapsed_time(e1) for e0, e1 in ev) / K


def run_variants(torch, la, workloads, K, hbm_peak, seed):
    """The rule variants that run on the same kernels, at the prefill benchmark
    shape (B=2, H=16, T=8192, d=128): DeltaNet (gated delta rule, alpha = 1),
    RetNet (GLA, one constant decay per head), Lightning (GLA, g = 1) without
    and with its output RMS normalisation; KDA prefill and decode; and GLA /
    gated-delta prefill of 32 packed variable-length sequences.  Each is timed K
    times with CUDA events, after 3 warm-up calls."""
    wn = torch.ones(128, device="cuda")
    spec = {"deltanet_prefill": ("gdn", dict(gdn_alpha="ones"), {}),
            "retnet_prefill": ("gla", dict(gla_gate="retnet"), {}),
            "lightning_prefill": ("gla", dict(gla_gate="ones"), {}),
            "lightning_norm_prefill": ("gla", dict(gla_gate="ones"),
                                       dict(out_norm=True, norm_w=wn, norm_eps=1e-6))}
    res = {}
    for name, (rule, kw, fkw) in spec.items():
        p = workloads.make_problem(rule, 2, 8192, 16, 128, 128, seed=seed, **kw)
        a = [None if t is None else t.cuda() for t in (p.q, p.k, p.v, p.g, p.beta)]
        o = torch.empty(2, 8192, 16, 128, dtype=torch.bfloat16, device="cuda")
        S = torch.empty(2, 16, 128, 128, device="cuda")
        run = lambda: la.fwd(rule, *a, o=o, S_out=S, **fkw)
        for _ in range(3):
            run()
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        torch.cuda.synchronize()
        for e0, e1 in ev:
            e0.record(stream)
            run()
            e1.record(stream)
        torch.cuda.synchronize()
        la.check_device()
        ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / K
        w = leg_work(rule + "_prefill")
        gbs = w["bytes"] / (ms / 1e3) / 1e9
        res[name] = {"ms": round(ms, 4), "tokens_per_s": round(w["tokens"] / (ms / 1e3)),
                     "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm_peak, 4)}
        del a, o, S
    # the normalisation pass alone: o read and written once (bf16)
    dn = res["lightning_norm_prefill"]["ms"] - res["lightning_prefill"]["ms"]
    nb = 2 * (2 * 8192 * 16 * 128 * 2)
    res["lightning_norm_prefill"]["norm_pass_ms"] = round(dn, 4)
    res["lightning_norm_prefill"]["norm_pass_gbs"] = round(nb / (dn / 1e3) / 1e9, 1) if dn > 0 else None
    # KDA (per-channel retention): chunked prefill (kda_prep_kernel +
    # gdn_main_kernel<true>) at the benchmark shape and one decode step
    # (recurrent kernel) on the [256,16,128,128] fp32 state
    p = workloads.make_problem("kda", 2, 8192, 16, 128, 128, seed=seed)
    a = [t.cuda() for t in (p.q, p.k, p.v, p.g, p.beta)]
    o = torch.empty(2, 8192, 16, 128, dtype=torch.bfloat16, device="cuda")
    S = torch.empty(2, 16, 128, 128, device="cuda")
    Kk = K
    ms = _time_calls(torch, lambda: la.fwd("kda", *a, o=o, S_out=S), Kk)
    la.check_device()
    w = prefill_bytes("gla", 2, 8192, 16, 128, 128) + 2 * 8192 * 16 * 4   # gla's bytes + beta
    res["kda_prefill"] = {"ms": round(ms, 4), "tokens_per_s": round(2 * 8192 / (ms / 1e3)),
                          "gbs": round(w / (ms / 1e3) / 1e9, 1), "hbm_frac": round(w / (ms / 1e3) / 1e9 / hbm_peak, 4),
                          "kernel": "chunked: kda_prep_kernel + gdn_main_kernel<true>", "timed_calls": Kk}
    del a, o, S
    Sd = workloads.decode_state(seed=seed).cuda()
    pd = workloads.make_problem("kda", 256, 1, 16, 128, 128, seed=seed)
    qd, kd, vd, gd = (x[:, 0].contiguous().cuda() for x in (pd.q, pd.k, pd.v, pd.g))
    bd = pd.beta[:, 0].contiguous().cuda()
    od = torch.empty(256, 16, 128, dtype=torch.bfloat16, device="cuda")
    ms = _time_calls(torch, lambda: la.step("kda", qd, kd, vd, Sd, g=gd, beta=bd, o=od), K)
    la.check_device()
    wd = decode_bytes("gla", 256, 16, 128, 128) + 256 * 16 * 4   # gla's bytes + beta
    res["kda_decode"] = {"ms": round(ms, 4), "gbs": round(wd / (ms / 1e3) / 1e9, 1),
                         "hbm_frac": round(wd / (ms / 1e3) / 1e9 / hbm_peak, 4)}
    del Sd
    # packed variable-length prefill: 32 sequences, lengths uniform in [1, 8192]
    # (seeded), H=16, d=128, on one token axis
    import numpy as np
    lens = np.random.default_rng(1000 + seed).integers(1, 8193, size=32)
    cu_h = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64)
    Ttot, Lmax = int(cu_h[-1]), int(lens.max())
    for rule in ("gla", "gdn"):
        p = workloads.make_problem(rule, 1, Ttot, 16, 128, 128, seed=seed)
        a = [None if t is None else t.cuda() for t in (p.q, p.k, p.v, p.g, p.beta)]
        cu = cu_h.cuda()
        o = torch.empty(1, Ttot, 16, 128, dtype=torch.bfloat16, device="cuda")
        S = torch.empty(32, 16, 128, 128, device="cuda")
        run = lambda: la.fwd(rule, *a, o=o, S_out=S, cu_seqlens=cu, max_seqlen=Lmax)
        for _ in range(3):
            run()
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
        torch.cuda.synchronize()
        for e0, e1 in ev:
            e0.record(stream)
            run()
            e1.record(stream)
        torch.cuda.synchronize()
        la.check_device()
        ms = sum(e0.elapsed_time(e1) for e0, e1 in ev) / K
        nbytes = prefill_bytes(rule, 1, Ttot, 16, 128, 128) + (32 - 1) * 16 * 128 * 128 * 4
        gbs = nbytes / (ms / 1e3) / 1e9
        res[f"packed_{rule}_prefill"] = {"ms": round(ms, 4), "tokens_per_s": round(Ttot / (ms / 1e3)),
                                        "sequences": 32, "tokens": Ttot, "max_seqlen": Lmax,
                                        "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm_peak, 4)}
        del a, o, S
    return res


def run_e2e(torch, la, legs, steps, world):
    pin = lambda t: None if t is None else t.contiguous().pin_memory()
    hg = {k: pin(getattr(legs.host["gla"], k)) for k in ("q", "k", "v", "g")}
    hd = {k: pin(getattr(legs.host["gdn"], k)) for k in ("q", "k", "v", "g", "beta")}
    mk = lambda: (torch.empty(2, 8192, 16, 128, dtype=torch.bfloat16).pin_memory(),
                  torch.empty(2, 16, 128, 128).pin_memory())
    og, Sg = mk()
    od, Sd = mk()
    n = max(la.host_staging_size("gla", hg["q"], hg["k"], hg["v"], hg["g"]),
            la.host_staging_size("gdn", hd["q"], hd["k"], hd["v"], hd["g"], hd["beta"]))
    staging = torch.empty(n, dtype=torch.uint8, device="cuda")
    h2d = sum(t.numel() * t.element_size() for t in list(hg.values()) + list(hd.values()))
    d2h = sum(t.numel() * t.element_size() for t in (og, Sg, od, Sd))

    def step():
        la.fwd_host("gla", hg["q"], hg["k"], hg["v"], hg["g"], o=og, S_out=Sg, staging=staging)
        la.fwd_host("gdn", hd["q"], hd["k"], hd["v"], hd["g"], hd["beta"], o=od, S_out=Sd,
                    staging=staging)

    step()
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(s)
    for _ in range(steps):
        step()
    b.record(s)
    torch.cuda.synchronize()
    import torch.distributed as dist
    ms = max_over_ranks(dist, [a.elapsed_time(b) / steps], "cuda")[0]
    tokens = 2 * 2 * 8192
    return {"value": round(job_tokens_per_s(world, tokens, ms)), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms, 3), "api": "la_fwd_host (C ABI, pinned host buffers)"}


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------

_ORACLE_INPUTS = []


def _oracle_inputs():
    if not _ORACLE_INPUTS:
        import workloads
        _ORACLE_INPUTS.extend([workloads.gla_prefill(B=2, H=16, T=8192),
                               workloads.gdn_prefill(B=2, H=16, T=8192)])
    return _ORACLE_INPUTS


def oracle_sample(T: int, batches: int = 1, repeats: int = 1):
    """GLA + gated-delta prefill, the first `batches` batches (all 16 heads) and
    first T tokens of the d=128 T=8192 workloads, `repeats` times; returns
    (seconds, tokens processed)."""
    import oracle
    oracle.build.build()
    gla, gdn = _oracle_inputs()
    sl = lambda x: x[:batches, :T].contiguous()
    args_gla = [sl(x) for x in (gla.q, gla.k, gla.v, gla.g)]
    args_gdn = [sl(x) for x in (gdn.q, gdn.k, gdn.v, gdn.g, gdn.beta)]
    t0 = time.perf_counter()
    for _ in range(repeats):
        oracle.gla_fwd(*args_gla)
        oracle.gdn_fwd(*args_gdn)
    dt = time.perf_counter() - t0
    return dt, 2 * T * batches * repeats


def cpu_baseline(budget_s: float = 15.0):
    import oracle
    # size the sample so that the timed part takes about budget_s seconds: a
    # prefix of batch 0, or the whole workload (both batches) repeated
    t_probe, tok_probe = oracle_sample(128)
    want = tok_probe / max(t_probe, 1e-3) * budget_s
    if want <= 2 * 8192:
        T, B, R = max(64, int(want / 2) // 64 * 64), 1, 1
    else:
        T = 8192
        B = 2 if want >= 2 * 2 * 8192 else 1
        R = max(1, min(64, round(want / (2 * T * B))))
    dt, tokens = oracle_sample(T, B, R)
    what = (f"first {T} tokens of batch 0" if B == 1 and R == 1 else
            f"all {B} batch(es), all 8192 tokens, {R} time(s)")
    return {"value": round(tokens / dt, 1), "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"fp64 C oracle (OpenMP over heads): GLA + gated-delta prefill of the d=128 "
                      f"T=8192 workloads, 16 heads, {what}; {dt:.1f} s",
            "host": _or_none(host_cpu), "elu_fp32_small_ms": _or_none(oracle_elu_small_ms)}


def _or_none(fn):
    """A descriptive field of the baseline: its failure must not cost the line."""
    try:
        return fn()
    except Exception:
        return None


def host_cpu():
    """The host the oracle ran on: cores this process may use, the CPU model
    and the oracle's OpenMP threads."""
    import oracle
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    return {"affinity_cores": cores, "cpu_model": model, "omp_threads": oracle.num_threads()}


def oracle_elu_small_ms(reps: int = 5):
    """Median time of the oracle on the fp32 ELU+1 workload (B=1 H=1 T=256
    d=32): one sequence, so one thread whatever the OpenMP setting."""
    import oracle
    import workloads
    p = workloads.elu_fp32_small(seed=0)
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        oracle.elu_fwd(p.q, p.k, p.v, p.S0, p.z0, eps=p.eps)
        ts.append(time.perf_counter() - t0)
    ts.sort()
    return round(1e3 * ts[len(ts) // 2], 3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    dist = None
    if world > 1:
        # the ranks meet once at the end (gloo: CPU only), so they finish together;
        # rank 0 alone does the work and prints the line
        import torch.distributed as dist
        from datetime import timedelta
        if not dist.is_initialized():
            dist.init_process_group("gloo", timeout=timedelta(minutes=10))
        else:
            dist = None   # the caller owns the group
    try:
        if rank == 0:
            _reference_line(args, world)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


def _reference_line(args, world):
    import oracle
    T = args.ref_tokens
    for _ in range(args.warmup):
        oracle_sample(T)
    times = []
    for _ in range(args.steps):
        dt, tokens = oracle_sample(T)
        times.append(dt)
    total = sum(times)
    value = args.steps * 2 * T / total
    cores = oracle.num_threads()
    sample = (f"per step: fp64 C oracle on GLA + gated-delta prefill, batch 0, 16 heads, first {T} "
              f"tokens of each d=128 T=8192 workload ({2 * T} tokens)")
    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic: seeded inputs per workloads.py; no dataset",
           "config": {"workload": "GLA + gated-delta prefill B=2 H=16 T=8192 dk=dv=128 (sampled)",
                      "global_batch": 2, "seq_len": 8192, "parallelism": "CPU threads"},
           "impl": "reference",
           "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": cores,
                            "kind": "oracle", "sample": sample, "host": _or_none(host_cpu)},
           "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, argv):
    """One rank started by launch_ranks: the environment a torchrun launch gives
    it (one process per GPU, rendezvous on 127.0.0.1), then the bench itself."""
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    main(argv)


def launch_ranks(world: int, argv) -> None:
    """`--gpus N` without a launcher: start N ranks (spawned processes, one per
    GPU) and wait for them; a rank that fails fails the launch."""
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(world, free_port(), argv), nprocs=world, join=True,
                       start_method="spawn")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-tokens", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-leg", choices=LEG_NAMES + PROFILE_ONLY_LEGS, default=None,
                    help="run one leg 3 + --reps times without timing (for ncu captures)")
    ap.add_argument("--reps", type=int, default=1)
    ap.add_argument("--variants", action="store_true",
                    help="also time DeltaNet, RetNet and Lightning prefill (same kernels) at B=2 H=16 T=8192")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    launched = "WORLD_SIZE" in os.environ
    if args.gpus < 1:
        sys.exit("bench.py: --gpus must be >= 1")
    if launched and int(os.environ["WORLD_SIZE"]) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but the launcher started WORLD_SIZE={os.environ['WORLD_SIZE']} ranks")
    if args.gpus > 1 and not launched:
        if args.impl == "cuda" and not args.profile_leg:
            import torch
            have = torch.cuda.device_count()
            if have < args.gpus:
                sys.exit(f"bench.py: --gpus {args.gpus} needs {args.gpus} CUDA devices, this node has {have}")
        launch_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv))
        return
    if args.profile_leg:
        run_profile_leg(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
