"""The tensor-parallel W4A4 linear on one GPU: a single-rank process group (the collective is the
identity) gives the plain linear's result bit for bit, and the shards of a two- and three-way
split, each run through macaq_w4a4_linear on its weight slice, put side by side match the oracle
(sampled rows) within the GEMM tolerance -- the per-rank work of a multi-GPU run, without the
collective (this pool gives one GPU per run)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import online_hadamard_b200 as m
    m.load_library()
    return m


def _layer(mq, M, K, N, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g) * 0.02
    s = torch.rand(K, generator=g) * 3 + 0.3
    Wq, Ws, am = mq.macaq_fold_weights(W.cuda(), s.cuda())
    return x, W, s, Wq, Ws, am


def test_single_rank_group_is_the_plain_linear(mq):
    import torch.distributed as dist

    from online_hadamard_b200 import tensor_parallel as tp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        x, W, s, Wq, Ws, am = _layer(mq, 300, 1024, 1000, 1)
        q, sc, n = tp.shard_folded_weights(Wq, Ws, 1000, 1024, 1, 0)
        y = tp.tp_w4a4_linear(x.cuda(), am, q, sc, 1000)
        ref = mq.macaq_w4a4_linear(x.cuda(), am, Wq, Ws, 1000)
        torch.cuda.synchronize()
        assert torch.equal(y, ref)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,K,N", [(4096, 5120, 25600), (16, 5120, 8192), (300, 1056, 1000)], ids=str)
@pytest.mark.parametrize("world", [2, 3])
def test_shards_side_by_side_match_the_oracle(mq, M, K, N, world):
    from online_hadamard_b200 import tensor_parallel as tp
    x, W, s, Wq, Ws, am = _layer(mq, M, K, N, M + N + world)
    parts = []
    for r in range(world):
        q, sc, n = tp.shard_folded_weights(Wq, Ws, N, K, world, r)
        parts.append(mq.macaq_w4a4_linear(x.cuda(), am, q, sc, n))
    y = torch.cat(parts, dim=1)
    full = mq.macaq_w4a4_linear(x.cuda(), am, Wq, Ws, N)
    torch.cuda.synchronize()
    assert gu.rel_fro(gu.to_np(y.float()), gu.to_np(full.float())) <= 1e-3
    rows = np.arange(M) if M <= 32 else np.sort(np.random.default_rng(2).choice(M, 12, replace=False))
    rWq, rWs, ra = oracle.fold_weights(W.numpy(), s.numpy())
    rAq, rAs = oracle.act_transform_quant(x.float().numpy()[rows], ra)
    ref = oracle.mx_gemm(rAq, rAs, rWq, rWs)
    assert gu.rel_fro(gu.to_np(y.float())[rows], gu.bf16_round(ref)) <= 1e-3
