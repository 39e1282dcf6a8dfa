"""The multi-rank (replica) host path of bench.py, on CPU with gloo.

With N GPUs every rank runs its own replica on its own tokens and the step
time is the maximum over ranks; these tests run that reduction and the
job-throughput arithmetic on two gloo ranks, check that a rank dying before
the collective makes the survivor fail within the process-group timeout
instead of hanging, and that the reference arm's non-zero ranks exit quietly.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    try:
        if mode == "ok":
            ms = [2.0, 3.5][rank]
            m = bench.reduce_max_over_ranks(ms, dist, "cpu")
            out[rank] = (m, bench.job_tokens_per_s(4096, world, m))
        elif mode == "dead_rank":
            if rank == 1:
                os._exit(3)          # dies before the collective
            try:
                bench.reduce_max_over_ranks(1.0, dist, "cpu")
                out[rank] = "returned"
            except Exception as e:   # the survivor must see an error, not hang
                out[rank] = f"error: {type(e).__name__}"
    finally:
        if mode == "ok":
            dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, "ok", out), nprocs=2, join=True)
        for r in range(2):
            ms, tps = out[r]
            assert ms == 3.5
            assert tps == pytest.approx(2 * 4096 / 3.5e-3)


def test_dead_rank_makes_survivor_fail_not_hang():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, "dead_rank", out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        alive = [p for p in procs if p.is_alive()]
        for p in alive:
            p.kill()
        assert not alive, "a rank hung"
        assert procs[1].exitcode == 3
        assert str(out.get(0, "")).startswith("error"), out.get(0)


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3", "--workload", "tiny"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks(1.25, None, "cpu") == 1.25
    assert bench.job_tokens_per_s(32, 1, 2.0) == pytest.approx(16000.0)
