"""GPU parity of the grouped (mixture-of-experts) W4A4 linear.  Each expert is its own linear
layer ("MACaQ", Abstract: layer-local), so the reference is the per-expert path: the codes the
grouped quantiser writes equal the per-expert quantiser's bit for bit, and y matches the
oracle's fp64 contraction of those codes with each expert's folded weights within the GEMM
tolerance, for the transformed and the plain (NULL multiplier) activations.  The padding rows of
each expert's 128-row segment are never written: the workspace starts as 0xFF (NaN scale bytes,
-6 codes), so a padding row that reached a stored output would show as a NaN in y."""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as gu
from tests import layout

pytestmark = pytest.mark.gpu

TOL = 1e-3


@pytest.fixture(scope="module")
def mq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import online_hadamard_b200 as m
    m.load_library()
    return m


def _experts(mq, E, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    Wq, Ws, am = [], [], []
    for _ in range(E):
        W = (torch.randn(N, K, generator=g) * 0.03).cuda()
        s = (torch.rand(K, generator=g) * 3 + 0.3).cuda()
        q, sc, a = mq.macaq_fold_weights(W, s)
        Wq.append(q)
        Ws.append(sc)
        am.append(a)
    return torch.stack(Wq), torch.cat(Ws), torch.stack(am)


CASES = [
    ("decode_top8", [1, 0, 2, 0, 0, 3, 1, 1, 0, 0, 0, 0, 0, 0, 0, 0], 256, 512),
    ("decode_16max", [16, 5, 0, 9], 384, 1024),
    ("mid_128max", [128, 100, 7], 256, 1056),
    ("prefill", [300, 0, 129, 64, 1], 512, 768),
    ("one_expert", [257], 384, 2048),
]


@pytest.mark.parametrize("name,counts,N,K", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("plain", [False, True], ids=["w4a4", "plain"])
def test_grouped_matches_per_expert(mq, name, counts, N, K, plain):
    E, T = len(counts), sum(counts)
    Wq, Ws, am = _experts(mq, E, N, K, seed=E * 31 + N + K)
    g = torch.Generator().manual_seed(T + K)
    x = (torch.randn(T, K, generator=g) * 2).to(torch.bfloat16).cuda()
    ws = torch.full((mq.grouped_workspace_bytes(counts, N, K),), 0xFF, dtype=torch.uint8, device="cuda")
    y = mq.macaq_w4a4_grouped_linear(x, counts, None if plain else am, Wq, Ws, N, workspace=ws)
    torch.cuda.synchronize()
    assert mq.macaq_device_status() == 0
    assert bool(torch.isfinite(y.float()).all())
    sb = mq.scale_bytes(N, K)
    P = sum((c + 127) // 128 * 128 for c in counts)
    Aq_all = ws[:P * K // 2].view(P, K // 2)
    As_off = (P * K // 2 + 255) // 256 * 256
    As_all = gu.to_np(ws[As_off:As_off + mq.scale_bytes(P, K)])
    As_rows = layout.tiled_to_rowmajor(As_all, P, K)
    x_row = a_row = 0
    for e, c in enumerate(counts):
        if c:
            xe = x[x_row:x_row + c]
            Aq, As = mq.macaq_act_quant_plain(xe) if plain else mq.macaq_act_transform_quant(xe, am[e])
            torch.cuda.synchronize()
            assert torch.equal(Aq_all[a_row:a_row + c], Aq)  # codes bit for bit
            Asr = layout.tiled_to_rowmajor(gu.to_np(As), c, K)
            assert np.array_equal(As_rows[a_row:a_row + c], Asr)
            ref = oracle.mx_gemm(gu.to_np(Aq), Asr, gu.to_np(Wq[e]),
                                 layout.tiled_to_rowmajor(gu.to_np(Ws[e * sb:(e + 1) * sb]), N, K))
            err = gu.rel_fro(gu.to_np(y[x_row:x_row + c].float()), gu.bf16_round(ref))
            assert err <= TOL, (e, err)
        x_row += c
        a_row += (c + 127) // 128 * 128


def test_grouped_without_tokens_leaves_y_alone(mq):
    N, K = 256, 512
    Wq, Ws, am = _experts(mq, 3, N, K, seed=5)
    x = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    y = mq.macaq_w4a4_grouped_linear(x, [0, 0, 0], am, Wq, Ws, N)
    torch.cuda.synchronize()
    assert y.shape == (0, N)


@pytest.mark.parametrize("name,counts,N,K", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("dtype", [torch.int32, torch.int64], ids=["i32", "i64"])
def test_device_counts_match_host_counts(mq, name, counts, N, K, dtype):
    """The counts on the device (a GPU router's output): y matches the host-count call within the
    GEMM tolerance (the kernel choice may differ: the host call picks it from the largest expert, the
    device call from the total), and both match the oracle per expert via the test above."""
    E, T = len(counts), sum(counts)
    Wq, Ws, am = _experts(mq, E, N, K, seed=E * 31 + N + K)
    g = torch.Generator().manual_seed(T + K)
    x = (torch.randn(T, K, generator=g) * 2).to(torch.bfloat16).cuda()
    host = mq.macaq_w4a4_grouped_linear(x, counts, am, Wq, Ws, N)
    ws = torch.full((mq.grouped_device_workspace_bytes(T, E, N, K),), 0xFF, dtype=torch.uint8, device="cuda")
    cd = torch.tensor(counts, dtype=dtype, device="cuda")
    dev = mq.macaq_w4a4_grouped_linear_device(x, cd, am, Wq, Ws, N, workspace=ws)
    dev2 = mq.macaq_w4a4_grouped_linear_device(x, cd, None, Wq, Ws, N)
    # an expert capacity at the largest count picks the narrow decode kernels where it can
    devc = mq.macaq_w4a4_grouped_linear_device(x, cd, am, Wq, Ws, N, capacity=max(counts))
    plain = mq.macaq_w4a4_grouped_linear(x, counts, None, Wq, Ws, N)
    torch.cuda.synchronize()
    assert mq.macaq_device_status() == 0
    assert bool(torch.isfinite(dev.float()).all())
    assert gu.rel_fro(gu.to_np(dev.float()), gu.to_np(host.float())) <= TOL
    assert gu.rel_fro(gu.to_np(dev2.float()), gu.to_np(plain.float())) <= TOL
    assert gu.rel_fro(gu.to_np(devc.float()), gu.to_np(host.float())) <= TOL


def test_device_counts_out_of_range_are_corrected_and_reported(mq):
    """Negative counts or counts past the rows of x are corrected on the device (no access outside x
    or y) and reported as MACAQ_ECOUNTS; the rows they do cover are computed as usual."""
    N, K = 256, 512
    Wq, Ws, am = _experts(mq, 3, N, K, seed=9)
    x = (torch.randn(40, K) * 2).to(torch.bfloat16).cuda()
    ref = mq.macaq_w4a4_grouped_linear(x[:30], [10, 0, 20], am, Wq, Ws, N)
    y = torch.zeros(40, N, dtype=torch.bfloat16, device="cuda")
    mq.macaq_w4a4_grouped_linear_device(x, torch.tensor([10, -5, 1000], dtype=torch.int32, device="cuda"), am, Wq, Ws,
                                        N, y=y)
    torch.cuda.synchronize()
    assert mq.macaq_device_status(clear=True) == -8  # MACAQ_ECOUNTS
    assert mq.macaq_device_status() == 0
    # expert 2's count is cut at the 30 rows that remain after expert 0: rows 10..39
    assert gu.rel_fro(gu.to_np(y[:10].float()), gu.to_np(ref[:10].float())) <= TOL
    assert bool(torch.isfinite(y.float()).all())


def test_device_counts_above_capacity_are_not_computed(mq):
    """An expert with more rows than the capacity: its first `capacity` rows are computed, the rest
    of its rows of y are left as they were, later experts keep their place in x, and MACAQ_ECOUNTS
    is reported."""
    N, K = 256, 512
    Wq, Ws, am = _experts(mq, 3, N, K, seed=13)
    counts = [5, 12, 7]
    x = (torch.randn(sum(counts), K) * 2).to(torch.bfloat16).cuda()
    ref = mq.macaq_w4a4_grouped_linear(x, counts, am, Wq, Ws, N)
    y = torch.full((sum(counts), N), 7.0, dtype=torch.bfloat16, device="cuda")
    mq.macaq_w4a4_grouped_linear_device(x, torch.tensor(counts, device="cuda"), am, Wq, Ws, N, capacity=8, y=y)
    torch.cuda.synchronize()
    assert mq.macaq_device_status(clear=True) == -8
    done = list(range(0, 5)) + list(range(5, 13)) + list(range(17, 24))  # expert 1: rows 5..12 of 5..16
    assert gu.rel_fro(gu.to_np(y[done].float()), gu.to_np(ref[done].float())) <= TOL
    assert bool((y[13:17] == 7.0).all())
