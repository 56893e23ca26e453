"""The multi-GPU (replicas) path of bench.py on the CPU: two processes over gloo run the same
rank plumbing the GPU bench runs over NCCL -- barrier, max over ranks of the step time, the
whole-job value (every rank's work over the slowest rank's time) -- and the reference arm
prints only on rank 0."""
import io
import os
import socket
import sys
import contextlib

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    ranks = bench.Ranks.from_env("gloo")
    try:
        ranks.barrier()
        ms = 1.0 + rank  # rank r's step time: the slowest rank decides
        ms_max = ranks.max(ms)
        out[rank] = (ranks.world, ranks.rank, ms_max, bench.whole_job_tflops(ranks.world, 2e12, ms_max))
        ranks.barrier()
    finally:
        ranks.close()


def test_replicas_max_over_ranks_gloo():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r, (w, rank, ms_max, value) in res.items():
        assert (w, rank) == (2, r)
        assert ms_max == 2.0  # the max of 1.0 and 2.0, seen by both ranks
        assert value == pytest.approx(2 * 2e12 / 2e-3 / 1e12)  # 2000 TFLOP/s


def test_single_process_needs_no_process_group():
    import bench
    ranks = bench.Ranks(1, 0, 0, "gloo")
    ranks.barrier()
    assert ranks.max(3.5) == 3.5
    assert ranks.dist is None
    ranks.close()


def test_reference_arm_prints_only_on_rank_zero(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(None)  # rank 1 returns before touching its arguments
    assert buf.getvalue() == ""
