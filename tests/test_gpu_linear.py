"""End-to-end parity of the W4A4 linear layer (fold + online transform + GEMM) against the
oracle run on its OWN codes: the oracle folds W, transforms and quantises x and contracts
in fp64 ("MACaQ", Abstract).  Because codes and scales are bit-exact, the GPU's bf16 y
must match bf16(y_oracle) within the GEMM tolerance.  The W4A4 error against the
unquantised fp64 x W^T is printed (the pages give no bound: parity unpinned)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wls
from tests import gpu_util as gu
from tests import layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import online_hadamard_b200 as m
    m.load_library()
    return m


CASES = [wls.TINY, wls.QWEN_UP_DECODE.with_m(1), wls.QWEN_UP_DECODE.with_m(16), wls.LLAMA_UP,
         wls.QWEN_DOWN, wls.stack_layer(0, "q", 32), wls.stack_layer(63, "down", 512),
         wls.stack_layer(17, "k", 4)]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: f"{w.name}_M{w.M}")
def test_linear_end_to_end(mq, wl):
    x = wls.make_x(wl)
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    Wq, Ws, am = mq.macaq_fold_weights(W.cuda(), s.cuda())
    y = mq.macaq_w4a4_linear(x.cuda(), am, Wq, Ws, wl.N)
    torch.cuda.synchronize()
    rng = np.random.default_rng(100 + wl.config)
    rows = np.arange(wl.M) if wl.M <= 64 else np.sort(rng.choice(wl.M, 16, replace=False))
    xf = x.float().numpy()
    Wf = W.numpy()
    rWq, rWs, ra = oracle.fold_weights(Wf, s.numpy())
    rAq, rAs = oracle.act_transform_quant(xf[rows], ra)
    ref = oracle.mx_gemm(rAq, rAs, rWq, rWs)
    got = gu.to_np(y.float())[rows]
    err = gu.rel_fro(got, gu.bf16_round(ref))
    exact = xf[rows].astype(np.float64) @ Wf.astype(np.float64).T
    q_err = gu.rel_fro(got, exact)
    print(f"{wl.name} M={wl.M}: vs oracle {err:.2e}; W4A4 error vs fp64 x W^T {q_err:.4f} (reported)")
    assert err <= 1e-3


# The 64-layer Qwen3-32B-shaped stack: every linear shape of a decoder layer (each from a
# different layer, so different seeds) at every token count of the stack sweep.  Each layer is
# its own problem ("MACaQ", Abstract: every linear layer is treated independently), with its own
# calibrated scale, fold and multipliers.
STACK_LAYER_OF = {"q": 5, "k": 17, "v": 29, "o": 40, "gate": 51, "up": 58, "down": 63}


@pytest.fixture(scope="module")
def stack_folds(mq):
    """Per stack linear (built once, reused for every M): s, the GPU fold and the oracle fold;
    the GPU fold is checked against the oracle's bit for bit on the way."""
    cache = {}

    def get(name):
        if name not in cache:
            wl = wls.stack_layer(STACK_LAYER_OF[name], name, 1)
            W = wls.make_w(wl)
            s = wls.make_s(wl, W)
            Wq, Ws, am = mq.macaq_fold_weights(W.cuda(), s.cuda())
            torch.cuda.synchronize()
            Wf = W.numpy()
            del W
            rWq, rWs, ra = oracle.fold_weights(Wf, s.numpy())
            assert np.array_equal(gu.to_np(am).view(np.uint32), ra.view(np.uint32))
            _, w = oracle.multipliers(s.numpy())
            gu.compare_mx(gu.to_np(Wq), gu.to_np(Ws), rWq, rWs, wl.N, wl.K, lambda: oracle.transform_f32(Wf, w),
                          label=gu.config_label(wl, "fold"))
            cache[name] = (Wq, Ws, am, rWq, rWs, ra)
        return cache[name]

    return get


@pytest.mark.parametrize("M", wls.STACK_M)
@pytest.mark.parametrize("name", list(STACK_LAYER_OF))
def test_stack_linear_matches_oracle(mq, stack_folds, name, M):
    """One linear of the stack at one token count, in the launch configuration the stack sweep
    times (the linear with a caller workspace): activation codes and scales of sampled rows bit
    for bit (near-boundary mismatches counted), y of those rows within the GEMM tolerance of
    the oracle's contraction of its own codes."""
    wl = wls.stack_layer(STACK_LAYER_OF[name], name, M)
    Wq, Ws, am, rWq, rWs, ra = stack_folds(name)
    x = wls.make_x(wl)
    xd = x.cuda()
    ws = torch.full((mq.linear_workspace_bytes(M, wl.N, wl.K),), 0xA5, dtype=torch.uint8, device="cuda")
    y = mq.macaq_w4a4_linear(xd, am, Wq, Ws, wl.N, workspace=ws)
    Aq, As = mq.macaq_act_transform_quant(xd, am)
    torch.cuda.synchronize()
    assert mq.macaq_device_status() == 0
    rng = np.random.default_rng(7 * M + wl.layer)
    rows = np.arange(M) if M <= 64 else np.unique(np.r_[0, M - 1, rng.choice(M, 22, replace=False)])
    xf = x.float().numpy()[rows]
    V = oracle.transform_f32(xf, ra)
    rAq, rAs = oracle.quantize_mx(V)
    gAs = layout.rows_of_tiled(gu.to_np(As), rows, wl.K)
    gu.compare_mx(gu.to_np(Aq)[rows], gAs, rAq, rAs, len(rows), wl.K, V, label=gu.config_label(wl, "act"))
    ref = oracle.mx_gemm(rAq, rAs, rWq, rWs)
    err = gu.rel_fro(gu.to_np(y.float())[rows], gu.bf16_round(ref))
    print(f"stack {name} M={M}: {len(rows)} rows vs oracle {err:.2e}")
    assert err <= 1e-3


def test_linear_zero_input_gives_zero(mq):
    M, K, N = 5, 256, 384
    W = torch.randn(N, K, device="cuda") * 0.02
    s = torch.rand(K, device="cuda") + 0.5
    Wq, Ws, am = mq.macaq_fold_weights(W, s)
    y = mq.macaq_w4a4_linear(torch.zeros(M, K, dtype=torch.bfloat16, device="cuda"), am, Wq, Ws, N)
    assert torch.count_nonzero(y).item() == 0


def test_linear_workspace_and_errors(mq):
    M, K, N = 3, 64, 40
    W = torch.randn(N, K, device="cuda")
    s = torch.ones(K, device="cuda")
    Wq, Ws, am = mq.macaq_fold_weights(W, s)
    x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    small = torch.empty(mq.linear_workspace_bytes(M, N, K) - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mq.MacaqError) as ei:
        mq.macaq_w4a4_linear(x, am, Wq, Ws, N, workspace=small)
    assert ei.value.status == -6
    ws = torch.full((mq.linear_workspace_bytes(M, N, K),), 0xFF, dtype=torch.uint8, device="cuda")
    y1 = mq.macaq_w4a4_linear(x, am, Wq, Ws, N, workspace=ws)
    y2 = mq.macaq_w4a4_linear(x, am, Wq, Ws, N)
    assert torch.equal(y1, y2)
    assert mq.macaq_device_status() == 0


# Shapes on both GEMM kernels (swap-AB for M <= 128, the CTA-pair kernel above), with ragged M,
# N and K tails, padded scale blocks (K = 1056), data-parallel and stream-K schedules.
LINEAR_SHAPES = [(1, 384, 256), (8, 512, 8192), (16, 1000, 6144), (3, 2000, 5120), (33, 2048, 8192), (128, 1000, 1056), (100, 520, 1024), (129, 520, 1024), (300, 777, 2048), (1000, 1024, 8192), (2049, 2304, 1056),
                 (4100, 512, 256), (3000, 4096, 768), (2500, 4608, 4352)]


@pytest.mark.parametrize("M,N,K", LINEAR_SHAPES, ids=lambda v: str(v))
def test_linear_matches_two_calls(mq, M, N, K):
    """The linear reproduces transform-then-GEMM bit for bit, for both the transformed (W4A4)
    and the plain MXFP4 activations, on a workspace that starts dirty and is reused, and
    leaves no timeout status."""
    g = torch.Generator().manual_seed(M + N + K)
    x = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16).cuda()
    W = (torch.randn(N, K, generator=g) * 0.05).cuda()
    s = (torch.rand(K, generator=g) * 3 + 0.3).cuda()
    Wq, Ws, am = mq.macaq_fold_weights(W, s)
    Aq, As = mq.macaq_act_transform_quant(x, am)
    ref = mq.macaq_mxfp4_gemm(Aq, As, Wq, Ws, M, N, K)
    ws = torch.full((mq.linear_workspace_bytes(M, N, K),), 0x5A, dtype=torch.uint8, device="cuda")
    y = mq.macaq_w4a4_linear(x, am, Wq, Ws, N, workspace=ws)
    y2 = mq.macaq_w4a4_linear(x, am, Wq, Ws, N, workspace=ws)  # reused workspace
    Pq, Ps = mq.macaq_act_quant_plain(x)
    pref = mq.macaq_mxfp4_gemm(Pq, Ps, Wq, Ws, M, N, K)
    py = mq.macaq_mxfp4_linear(x, Wq, Ws, N, workspace=ws)
    torch.cuda.synchronize()
    assert mq.macaq_device_status() == 0
    assert torch.equal(y, ref)
    assert torch.equal(y2, ref)
    assert torch.equal(py, pref)
    # the workspace starts with the activation codes the linear quantised
    assert torch.equal(ws[:M * K // 2].view(M, K // 2), Pq)


def test_plain_linear_against_oracle(mq):
    """macaq_mxfp4_linear against the oracle's plain quantiser and fp64 contraction."""
    M, K, N = 384, 1024, 640
    g = torch.Generator().manual_seed(77)
    x = (torch.randn(M, K, generator=g) * 1.5).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g) * 0.03
    Wq, Ws, _ = mq.macaq_fold_weights(W.cuda(), torch.ones(K, device="cuda"))
    y = mq.macaq_mxfp4_linear(x.cuda(), Wq, Ws, N)
    torch.cuda.synchronize()
    rows = np.arange(0, M, 7)
    rAq, rAs = oracle.act_quant_plain(x.float().numpy()[rows])
    Wc = gu.to_np(Wq)
    Wsr = layout.tiled_to_rowmajor(gu.to_np(Ws), N, K)
    ref = oracle.mx_gemm(rAq, rAs, Wc, Wsr)
    assert gu.rel_fro(gu.to_np(y.float())[rows], gu.bf16_round(ref)) <= 1e-3
