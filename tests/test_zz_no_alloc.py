"""macaq_w4a4_linear_noalloc, the linear layer for callers that cannot allocate device memory
(a latency-critical loop that plans its memory up front, a plugin whose host owns every
allocation, a C caller handed only input and output pointers).  It keeps the activation
scratch in a static 32 MiB device array of the library instead of a caller workspace.

Called here through the C ABI (ctypes, raw device pointers) and compared with
macaq_w4a4_linear on two calls in a row -- a larger problem, then a smaller one, so the
second runs over the first one's leftover scratch -- within the GEMM tolerance of the other
tests; and, on a problem too large for the GEMM's stream-K scratch to fit beside the
activations, with the oracle and with the data-parallel GEMM it falls back to.  This file is collected last so a stop-at-first-failure run has run the rest first."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 1e-3  # relative Frobenius error, as in tests/test_gpu_gemm.py


@pytest.fixture(scope="module")
def mq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import online_hadamard_b200 as m
    m.load_library()
    return m


def _layer(mq, M, K, N, seed):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(M, K, generator=g) * 3).to(torch.bfloat16).cuda()
    W = (torch.randn(N, K, generator=g) * 0.02).cuda()
    s = (torch.rand(K, generator=g) * 4 + 0.25).cuda()
    Wq, Ws, am = mq.macaq_fold_weights(W, s)
    return x, Wq, Ws, am


def _noalloc_via_c_abi(mq, x, am, Wq, Ws, N):
    M, K = x.shape
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = mq.load_library().macaq_w4a4_linear_noalloc(
        P(x), M, K, P(am), P(Wq), P(Ws), N, P(y), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, mq.status_str(st)
    return y


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def test_noalloc_matches_linear_on_two_calls_in_a_row(mq):
    big = _layer(mq, 300, 1024, 520, 1)
    small = _layer(mq, 5, 256, 384, 2)
    y1 = _noalloc_via_c_abi(mq, big[0], big[3], big[1], big[2], 520)
    y2 = _noalloc_via_c_abi(mq, small[0], small[3], small[1], small[2], 384)
    r1 = mq.macaq_w4a4_linear(big[0], big[3], big[1], big[2], 520)
    r2 = mq.macaq_w4a4_linear(small[0], small[3], small[1], small[2], 384)
    torch.cuda.synchronize()
    assert _rel(y1, r1) <= TOL
    assert _rel(y2, r2) <= TOL
    assert torch.count_nonzero(r1).item() > 0 and torch.count_nonzero(r2).item() > 0
    assert mq.macaq_device_status() == 0


def test_noalloc_against_oracle_and_its_data_parallel_fallback(mq):
    """A problem whose activation codes and scales fit the 32 MiB array but whose whole
    workspace (with the GEMM's stream-K scratch) does not: the GEMM then runs its
    data-parallel schedule, so the output equals, bit for bit, the data-parallel GEMM of the
    same codes.  Called right after a smaller stream-K problem, so it runs over that call's
    leftover scratch, and checked on sampled rows against the oracle's own fold,
    quantisation and fp64 contraction."""
    import oracle
    from tests import gpu_util as gu
    M, K, N = 4096, 8192, 2560
    act = M * K // 2 + mq.scale_bytes(M, K)
    assert act <= mq.NOALLOC_SCRATCH_BYTES < mq.linear_workspace_bytes(M, N, K)
    small = _layer(mq, 200, 1024, 768, 3)
    _noalloc_via_c_abi(mq, small[0], small[3], small[1], small[2], 768)
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g) * 0.02
    s = torch.rand(K, generator=g) * 4 + 0.25
    Wq, Ws, am = mq.macaq_fold_weights(W.cuda(), s.cuda())
    y = _noalloc_via_c_abi(mq, x.cuda(), am, Wq, Ws, N)
    Aq, As = mq.macaq_act_transform_quant(x.cuda(), am)
    dp = mq.macaq_mxfp4_gemm(Aq, As, Wq, Ws, M, N, K, data_parallel=True)
    torch.cuda.synchronize()
    assert mq.macaq_device_status() == 0
    assert torch.equal(y, dp)
    rows = np.sort(np.random.default_rng(5).choice(M, 16, replace=False))
    rWq, rWs, ra = oracle.fold_weights(W.numpy(), s.numpy())
    rAq, rAs = oracle.act_transform_quant(x.float().numpy()[rows], ra)
    ref = oracle.mx_gemm(rAq, rAs, rWq, rWs)
    assert gu.rel_fro(gu.to_np(y.float())[rows], gu.bf16_round(ref)) <= TOL


def test_noalloc_rejects_problems_beyond_its_scratch(mq):
    lib = mq.load_library()
    K = 8192
    M = 8192  # needs 32 MiB of codes plus scales: over the limit
    assert M * K // 2 + mq.scale_bytes(M, K) > mq.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x10000)  # validation fails before any pointer is used
    st = lib.macaq_w4a4_linear_noalloc(fake, M, K, fake, fake, fake, 64, fake, None)
    assert st == -7, mq.status_str(st)
