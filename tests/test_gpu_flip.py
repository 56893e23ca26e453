"""GPU parity of Flip-Refinement (macaq_calib_hessian, macaq_flip_refine) against the oracle:
the Hessian bit for bit, the refined codes bit for bit and the moves per row equal.  Every
decision is taken in fp64 with the same operations in the same order on both sides (the reading
in oracle/macaq_oracle.c), so the codes must agree exactly.

"MACaQ ...", Abstract: Flip-Refinement refines the round-to-nearest codes by a greedy,
Hessian-weighted coordinate descent over single-code steps to neighbouring grid values."""
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


def _layer(N, K, C, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xcal = rng.standard_normal((C, K)).astype(np.float32)
    xcal[:, rng.choice(K, max(1, K // 100), replace=False)] *= 30.0
    xcal = torch.from_numpy(xcal).to(torch.bfloat16)
    s = oracle.calibrate_scale(xcal.float().numpy(), W)
    return W, s, xcal


@pytest.mark.parametrize("N,K,C,max_moves", [(300, 1024, 64, 10_000), (130, 1056, 40, 10_000), (64, 512, 33, 0),
                                             (64, 512, 33, 1), (200, 768, 96, 3),
                                             (2100, 256, 40, 50)],  # two chunks of rows (2048 + 52)
                         ids=lambda v: str(v))
def test_flip_refine_matches_oracle(mq, N, K, C, max_moves):
    W, s, xcal = _layer(N, K, C, N + K + C + max_moves)
    Wd, sd = torch.from_numpy(W).cuda(), torch.from_numpy(s).cuda()
    Wq, Ws, am = mq.macaq_fold_weights(Wd, sd)
    rtn = Wq.clone()
    Hs = mq.macaq_calib_hessian(xcal.cuda(), am)
    moves = mq.macaq_flip_refine(Wd, sd, Hs, Wq, Ws, max_moves)
    torch.cuda.synchronize()
    assert mq.macaq_device_status() == 0
    a, w = oracle.multipliers(s)
    rHs = oracle.calib_hessian(xcal.float().numpy(), a)
    assert np.array_equal(gu.to_np(Hs).view(np.uint64), rHs.view(np.uint64)), "Hessian"
    V = oracle.transform_f32(W, w)
    rcodes, rscales = oracle.quantize_mx(V)
    assert np.array_equal(gu.to_np(rtn), rcodes)
    ref, rmoves = oracle.flip_refine_codes(V, rcodes, rscales, rHs, max_moves)
    assert np.array_equal(gu.to_np(moves).astype(np.int64), rmoves)
    assert np.array_equal(gu.to_np(Wq), ref)
    if max_moves == 0:
        assert np.array_equal(gu.to_np(Wq), rcodes)
    print(f"N={N} K={K}: {int(rmoves.sum())} moves, {float((rmoves > 0).mean()):.2f} of rows moved")


def test_flip_refine_llama_width_sampled_rows(mq):
    """K = 4096 (the Llama-3-8B up projection's input width): the GPU refines all rows, the oracle a
    sample of them (rows are independent)."""
    N, K, C = 512, 4096, 64
    W, s, xcal = _layer(N, K, C, 17)
    Wd, sd = torch.from_numpy(W).cuda(), torch.from_numpy(s).cuda()
    Wq, Ws, am = mq.macaq_fold_weights(Wd, sd)
    Hs = mq.macaq_calib_hessian(xcal.cuda(), am)
    moves = mq.macaq_flip_refine(Wd, sd, Hs, Wq, Ws, 64)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(N, 24, replace=False))
    a, w = oracle.multipliers(s)
    rHs = oracle.calib_hessian(xcal.float().numpy(), a)
    assert np.array_equal(gu.to_np(Hs).view(np.uint64), rHs.view(np.uint64))
    V = oracle.transform_f32(W[rows], w)
    rc, rsc = oracle.quantize_mx(V)
    ref, rmoves = oracle.flip_refine_codes(V, rc, rsc, rHs, 64)
    assert np.array_equal(gu.to_np(moves)[rows].astype(np.int64), rmoves)
    assert np.array_equal(gu.to_np(Wq)[rows], ref)


def test_flip_refine_rejects_bad_arguments(mq):
    K = 12320  # above the one-row shared-memory limit
    assert mq.load_library().macaq_flip_refine_workspace_bytes(4, K) == 0
    W = torch.zeros(4, 64, device="cuda")
    s = torch.ones(64, device="cuda")
    Wq, Ws, am = mq.macaq_fold_weights(W, s)
    Hs = torch.zeros(64, 64, dtype=torch.float64, device="cuda")
    with pytest.raises(mq.MacaqError) as ei:
        mq.macaq_flip_refine(W, s, Hs, Wq, Ws, -1)
    assert ei.value.status == -1
