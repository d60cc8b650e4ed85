"""Host logic of the multi-GPU benchmark on CPU: two gloo ranks combine their
timings as max over ranks and their work as the sum; the reference arm runs
on rank 0 only."""

import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    from shifted_window_attention_sw_b200 import replicas

    r, w = replicas.init("gloo", timeout_s=60)
    replicas.barrier()
    elapsed, units, n = replicas.combine(1.0 + r, 10.0 * (r + 1))
    replicas.shutdown()
    q.put((r, w, elapsed, units, n))


def test_two_ranks_combine_max_time_and_sum_work():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for r, (rank, w, elapsed, units, n) in enumerate(got):
        assert (rank, w, n) == (r, world, world)
        assert elapsed == 2.0  # slowest rank
        assert units == 30.0   # all ranks' work


def test_single_process_combine_is_identity():
    sys.path.insert(0, ROOT)
    from shifted_window_attention_sw_b200 import replicas

    assert replicas.combine(1.5, 7.0) == (1.5, 7.0, 1)


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_bench_refuses_a_world_size_that_is_not_gpus():
    # under torchrun the rank count must be the --gpus the line will report
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "4",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "WORLD_SIZE" in r.stderr
