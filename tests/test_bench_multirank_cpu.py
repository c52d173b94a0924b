"""The bench's multi-rank path on CPU: two ranks over gloo (no GPU).

With N GPUs the bench runs one process per GPU, each on its own sequences
(weak scaling, no collective on the data path); the only collectives are the
barrier and the maximum of the per-rank device times, and the whole-job value
counts every rank's tokens over that maximum.  The reference arm runs on rank
0 alone; the other ranks exit without work.  These tests drive exactly those
functions from two gloo ranks, and drive ``bench.py --gpus 2`` itself: without
a launcher it starts its two ranks (torchrun's environment, 127.0.0.1), and it
refuses to run on fewer CUDA devices than asked for.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    return dist


def _max_worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    dist = _init(rank, world, port)
    try:
        # rank r's leg times: rank 1 is slower on the first entry, rank 0 on the second
        mine = [10.0 + rank, 5.0 - rank, 7.5]
        red = bench.max_over_ranks(dist, mine, "cpu")
        value = bench.job_tokens_per_s(world, 32768, red[0])
        dist.barrier()
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"red": red, "value": value}, f)
    finally:
        dist.destroy_process_group()


def _reference_worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    dist = _init(rank, world, port)
    try:
        args = argparse.Namespace(ref_tokens=16, steps=1, warmup=1)
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(args)
        with open(os.path.join(out_dir, f"ref{rank}.txt"), "w") as f:
            f.write(buf.getvalue())
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value(tmp_path):
    world, port = 2, _free_port()
    mp.spawn(_max_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    r0 = json.load(open(tmp_path / "r0.json"))
    r1 = json.load(open(tmp_path / "r1.json"))
    assert r0["red"] == r1["red"] == [11.0, 5.0, 7.5]
    # 2 ranks x 32768 tokens in 11 ms
    assert r0["value"] == pytest.approx(2 * 32768 / 0.011)


def test_reference_arm_runs_on_rank_zero_only(tmp_path):
    world, port = 2, _free_port()
    mp.spawn(_reference_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    out0 = (tmp_path / "ref0.txt").read_text().strip().splitlines()
    out1 = (tmp_path / "ref1.txt").read_text().strip()
    assert out1 == ""
    line = json.loads(out0[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"


def _bench(*argv, timeout=300):
    import subprocess
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env["OMP_NUM_THREADS"] = "2"
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_gpus_flag_launches_the_ranks_itself():
    """`bench.py --gpus 2` without torchrun starts two ranks (torchrun's
    environment, rendezvous on 127.0.0.1; the reference arm meets over gloo) and
    prints one line, from rank 0, for the whole job."""
    r = _bench("--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-tokens", "16")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_gpus_flag_refuses_missing_devices():
    """The CUDA arm refuses, instead of running on fewer GPUs, when the node has
    fewer CUDA devices than --gpus asks for (none here)."""
    r = _bench("--gpus", "2", "--steps", "1")
    assert r.returncode != 0
    assert "needs 2 CUDA devices" in r.stderr
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


def test_gpus_flag_must_match_the_launcher():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="4", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE=4" in r.stderr
