"""The N > 1 bench path (independent replicas) on CPU: two gloo ranks agree on the slowest
rank's time, the job throughput counts every rank's tokens, the ranks' batches differ, and
the reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
        q.put((rank, ms, bench.job_throughput(64 * 32, world, 3, ms), bench.replica_seed(rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, s0), (r1, ms1, v1, s1) = res
    assert ms0 == ms1 == 15.0                    # the slowest rank's time on both ranks
    assert v0 == v1 == pytest.approx(64 * 32 * 2 * 3 / 0.015)
    assert s0 != s1                               # each replica generates its own batch


def test_replica_batches_differ():
    import bench
    import fg_synth
    a = fg_synth.token_ids(bench.replica_seed(0), fg_synth.S_IDS, (4, 16), 50272)
    b = fg_synth.token_ids(bench.replica_seed(1), fg_synth.S_IDS, (4, 16), 50272)
    assert not np.array_equal(a, b)


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
