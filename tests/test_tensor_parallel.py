"""The tensor-parallel (N-split) W4A4 linear's host logic on the CPU: shard ranges of whole 128-row
blocks, slices of the folded codes and of the E8M0 scales in the MMA tile layout, and the
all-gather of the output columns over gloo with two ranks, each rank's arithmetic done by the
oracle on its shard.  The gathered result must equal the single-rank oracle result exactly (the
oracle's contraction is exact fp64, so a shard's columns are the full problem's columns)."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from online_hadamard_b200 import tensor_parallel as tp  # noqa: E402
from tests import layout  # noqa: E402


@pytest.mark.parametrize("N", [128, 130, 1000, 1024, 25600, 14336, 383])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_ranges_tile_the_rows(N, world):
    ranges = [tp.shard_range(N, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == N
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0
    for n0, n1 in ranges:
        assert n0 <= n1 and (n0 % 128 == 0 or n0 == n1 == N)  # an empty shard sits at N
        assert n1 == N or n1 % 128 == 0
    blocks = [-(-(n1 - n0) // 128) for n0, n1 in ranges if n1 > n0]
    assert max(blocks) - min(blocks) <= 1


@pytest.mark.parametrize("N,K", [(300, 1056), (1024, 512), (129, 256)])
def test_scale_slices_are_the_shards_scales(N, K):
    rng = np.random.default_rng(N + K)
    S = rng.integers(0, 255, (N, K // 32)).astype(np.uint8)
    tiled = torch.from_numpy(layout.rowmajor_to_tiled(S, N, K))
    codes = torch.from_numpy(rng.integers(0, 255, (N, K // 2)).astype(np.uint8))
    for world in (2, 3):
        for r in range(world):
            q, s, n = tp.shard_folded_weights(codes, tiled, N, K, world, r)
            n0, n1 = tp.shard_range(N, world, r)
            assert n == n1 - n0 and torch.equal(q, codes[n0:n1])
            if n:
                assert s.numel() == layout.scale_bytes(n, K)
                assert np.array_equal(layout.tiled_to_rowmajor(s.numpy(), n, K), S[n0:n1])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(9)
        M, K, N = 6, 512, 700
        x = rng.standard_normal((M, K)).astype(np.float32)
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        s = rng.uniform(0.5, 2.0, K).astype(np.float32)
        Wq, Ws, a = oracle.fold_weights(W, s)
        Aq, As = oracle.act_transform_quant(x, a)
        full = oracle.mx_gemm(Aq, As, Wq, Ws)
        tiled = torch.from_numpy(layout.rowmajor_to_tiled(Ws, N, K))
        q, sc, n = tp.shard_folded_weights(torch.from_numpy(Wq), tiled, N, K, world, rank)
        y_shard = oracle.mx_gemm(Aq, As, q.numpy(), layout.tiled_to_rowmajor(sc.numpy(), n, K))
        y = tp.gather_columns(torch.from_numpy(y_shard), N)
        out[rank] = bool(np.array_equal(y.numpy(), full)), tuple(y.shape)
    finally:
        dist.destroy_process_group()


def test_two_rank_gather_equals_single_rank_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert dict(out) == {0: (True, (6, 700)), 1: (True, (6, 700))}
