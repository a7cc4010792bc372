"""Host logic of the benchmark's multi-process path on CPU (gloo, world size 2):
the max-over-ranks timing, the whole-job throughput, and the reference arm
under torchrun, where rank 0 alone runs and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [12.5, 20.0][rank]            # this rank's timed milliseconds
        m = bench.max_over_ranks(elapsed, dist, "cpu")
        q.put((rank, m, bench.job_throughput(100, world, m)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, m, v in res:
        assert m == 20.0                       # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 100 / 0.020)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_throughput(10, 1, 1000.0) == pytest.approx(10.0)


def _run_ref(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--config", "relu1", "--steps", "2", "--warmup", "3"],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_rank0_prints_other_ranks_exit_quietly():
    r1 = _run_ref(1)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_ref(0)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_code_hash_ignores_comments_and_blank_space_only():
    base = "int f(int a) {\n    return a + 1;   // one more\n}\n"
    same = "/* header */\nint f(int a)\n{ return a + 1; }\n// trailing note\n"
    changed = "int f(int a) {\n    return a + 2;   // one more\n}\n"
    assert bench.code_hash(base) == bench.code_hash(same)
    assert bench.code_hash(base) != bench.code_hash(changed)
    assert len(bench.kernel_hash()) == 16
