"""Multi-rank host logic of bench.py, on CPU with the gloo backend.

The path splits into independent (sequence, head) problems, so
`bench.py --gpus N` runs one replica per GPU and the only cross-rank step is
the maximum over ranks of the timed region (and of the end-to-end time).
These tests run that step with two gloo ranks, and check the reference arm's
rank handling (rank 0 prints one line, the other ranks exit without work).
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench
    slowest = bench.max_over_ranks(times[rank], torch.device("cpu"))
    tops = bench.job_tops(world, 1e12, 10, slowest)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, slowest, tops))


@pytest.mark.parametrize("times", [(3.5, 7.25), (9.0, 2.0)])
def test_max_over_ranks_two_gloo_ranks(times):
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.exitcode is None:
            p.kill()
    assert codes == [0, 0], codes
    res = sorted(out.get() for _ in range(2))
    want = max(times)
    for rank, slowest, tops in res:
        assert slowest == want
        # both ranks' work over the slowest rank's time
        assert tops == pytest.approx(2 * 1e12 * 10 / (want * 1e-3) / 1e12)


def test_max_over_ranks_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.5, torch.device("cpu")) == 4.5
    assert bench.job_tops(1, 2e12, 5, 1000.0) == pytest.approx(10.0)


def _reference_arm(rank: int, world: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                           "--gpus", str(world), "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.2"],
                          env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_on_rank0_only():
    r1 = _reference_arm(1, 2)
    assert r1.returncode == 0, r1.stderr
    assert r1.stdout.strip() == ""
    r0 = _reference_arm(0, 2)
    assert r0.returncode == 0, r0.stderr
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "TOPS" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
