"""Parity of macaq_w4a4_linear_multi: several layers on one x (the q, k and v projections of an
attention block, the gate and up projections of an MLP), each its own MACaQ layer with its own
scale, fold and multipliers ("MACaQ ...", Abstract: every linear layer stands alone).  Per layer:
the activation codes and scales the call leaves in its workspace equal the oracle's transform and
quantisation of x with that layer's multipliers (bit for bit, 1-ulp exemption as elsewhere), and
its column block of y matches the oracle's fp64 contraction of those codes with the oracle's fold
of the layer's weights within the GEMM tolerance."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wls
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

MULTI_CONFIG = 7  # seed slot of these synthetic layer sets


@pytest.fixture(scope="module")
def mq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import online_hadamard_b200 as m
    m.load_library()
    return m


def _layers(name, K, Ns):
    """One Workload per layer: x drawn as for the llama up projection (1 % outlier channels x 50),
    W ~ N(0, 0.02), each layer its own seeds."""
    return [wls.Workload(f"{name}_{g}", MULTI_CONFIG, 1, K, N, "normal", 0.01, 50.0, layer=g)
            for g, N in enumerate(Ns)]


def _fold_all(mq, layers):
    """GPU folds (stacked as the call takes them) and the oracle folds, per layer."""
    gpu, ref = [], []
    for wl in layers:
        W = wls.make_w(wl)
        s = wls.make_s(wl, W)
        gpu.append(mq.macaq_fold_weights(W.cuda(), s.cuda()))
        ref.append(oracle.fold_weights(W.numpy(), s.numpy()))
    Wq = torch.cat([q for q, _, _ in gpu])
    Ws = torch.cat([t for _, t, _ in gpu])
    am = torch.stack([a for _, _, a in gpu])
    for (_, _, a), (_, _, ra) in zip(gpu, ref):
        assert np.array_equal(gu.to_np(a).view(np.uint32), ra.view(np.uint32))
    return Wq, Ws, am, ref


def _workspace_acts(ws, M, K, G, g):
    """Layer g's activation codes [M, K/2] and tiled scales as the header places them."""
    Mp = (M + 127) // 128 * 128
    sb = Mp * 8 * ((K + 255) // 256)
    a0 = (G * Mp * K // 2 + 255) // 256 * 256
    codes = ws[g * Mp * K // 2: g * Mp * K // 2 + M * K // 2].view(M, K // 2)
    scales = ws[a0 + g * sb: a0 + (g + 1) * sb]
    return gu.to_np(codes), gu.to_np(scales)


def _check(mq, layers, M, plain=False, col_sample=None, row_sample=None):
    K = layers[0].K
    Ns = [wl.N for wl in layers]
    G = len(Ns)
    Wq, Ws, am, ref = _fold_all(mq, layers)
    x = wls.make_x(layers[0], M)
    ws = torch.empty(mq.linear_multi_workspace_bytes(M, G, K), dtype=torch.uint8, device="cuda")
    y = mq.macaq_w4a4_linear_multi(x.cuda(), None if plain else am, Wq, Ws, Ns, workspace=ws)
    torch.cuda.synchronize()
    xf = x.float().numpy()
    yg = gu.to_np(y.float())
    rng = np.random.default_rng(7000 + M)
    rows = np.arange(M) if row_sample is None else np.sort(rng.choice(M, row_sample, replace=False))
    n0 = 0
    for g, (wl, (rWq, rWs, ra)) in enumerate(zip(layers, ref)):
        if plain:
            rAq, rAs = oracle.act_quant_plain(xf)
        else:
            rAq, rAs = oracle.act_transform_quant(xf, ra)
        if not plain or g == 0:  # plain: one shared set of codes
            codes, scales = _workspace_acts(ws, M, K, G, 0 if plain else g)
            gu.compare_mx(codes, scales, rAq, rAs, M, K,
                          (lambda: xf.astype(np.float32)) if plain else (lambda ra=ra: oracle.transform_f32(xf, ra)),
                          label=f"config {MULTI_CONFIG} stacked-layers activations")
        cols = np.arange(wl.N) if col_sample is None else np.sort(rng.choice(wl.N, col_sample, replace=False))
        want = oracle.mx_gemm(rAq, rAs, rWq[cols], rWs[cols], rows=rows)
        got = yg[rows][:, n0 + cols]
        err = gu.rel_fro(got, gu.bf16_round(want))
        print(f"layer {g} (N={wl.N}) M={M}{' plain' if plain else ''}: vs oracle {err:.2e}")
        assert err <= 1e-3
        n0 += wl.N
    return x, y, Wq, Ws, am


QKV_SMALL = _layers("qkv_small", 512, (512, 128, 128))
QKV_PAIR = _layers("qkv_pair", 768, (512, 256, 256))


@pytest.mark.parametrize("M", [1, 5, 16, 33, 64, 128, 129, 300])
def test_stacked_qkv_small(mq, M):
    """Every swap-AB tile width (M <= 128: one stacked GEMM, three activation segments) and, above
    128 tokens with a layer width that is not a multiple of 256, one GEMM per layer (ragged M, y
    written with a row stride of sum N)."""
    _check(mq, QKV_SMALL, M)


@pytest.mark.parametrize("M", [129, 300, 600])
def test_stacked_pair_gemm(mq, M):
    """Above 128 tokens with every width a multiple of 256: one CTA-pair GEMM over the stacked
    weights, each 256-row weight tile against its layer's activation segment (ragged M: the
    segments' padding rows and the next segment's rows reach only unstored output rows)."""
    _check(mq, QKV_PAIR, M)


def test_stacked_large_k_at_128_tokens(mq):
    """M * K above the half-block quantiser's range at 128 tokens (K = 33024, 129 blocks: a ragged
    last K tile): the grouped quantiser writes the segments, the swap-AB GEMM reads them."""
    _check(mq, _layers("large_k", 33024, (256, 128)), 128, col_sample=96)


def test_single_layer_stack_is_the_linear(mq):
    """G = 1: the stacked call is the single layer's linear (same codes; y within the GEMM tolerance,
    bit for bit where both take the same schedule)."""
    layers = _layers("one", 512, (384,))
    for M in (3, 200):
        x, y, Wq, Ws, am = _check(mq, layers, M)
        ys = mq.macaq_w4a4_linear(x.cuda(), am[0].contiguous(), Wq, Ws, 384)
        torch.cuda.synchronize()
        assert gu.rel_fro(gu.to_np(y.float()), gu.to_np(ys.float())) <= 1e-3


def test_stacked_gate_up_ragged(mq):
    _check(mq, _layers("gateup_small", 1056, (384, 384)), 7)  # K = 33 blocks: a ragged 256-wide K tile


@pytest.mark.parametrize("layers,M", [(QKV_SMALL, 16), (QKV_SMALL, 200), (QKV_PAIR, 300)])
def test_stacked_plain_shares_one_quantisation(mq, layers, M):
    """act_mult = NULL: plain MXFP4 of x, quantised once, contracted with every layer's weights."""
    _check(mq, layers, M, plain=True)


@pytest.mark.parametrize("M", [1, 16, 512])
def test_stacked_qwen_qkv(mq, M):
    """Qwen3-32B-shaped q, k and v projections (K = 5120; N = 8192, 1024, 1024) at decode and at
    512 tokens: one quantiser and one GEMM over 10240 stacked weight rows; sampled output columns."""
    layers = [wls.stack_layer(0, n, 1) for n in ("q", "k", "v")]
    _check(mq, layers, M, col_sample=512)


@pytest.mark.parametrize("M", [32, 4096])
def test_stacked_qwen_gate_up(mq, M):
    """Qwen3-32B-shaped gate and up projections (K = 5120, N = 25600 each): 51200 stacked weight rows,
    swap-AB at 32 tokens, the CTA-pair GEMM with stream-K at 4096; every activation code and scale
    compared, outputs on sampled rows and columns."""
    layers = [wls.stack_layer(0, n, 1) for n in ("gate", "up")]
    _check(mq, layers, M, col_sample=384, row_sample=None if M <= 64 else 48)


@pytest.mark.parametrize("layers,M", [(QKV_SMALL, 16), (QKV_SMALL, 300), (QKV_PAIR, 300)])
def test_stacked_matches_single_layer_calls(mq, layers, M):
    """Where each layer runs its own GEMM (above 128 tokens, a width not a multiple of 256) the
    schedule is the single layer's, so its column block equals macaq_w4a4_linear's output bit for
    bit; the stacked launches agree with it within the GEMM tolerance (they split the K steps over
    a different tile count)."""
    x, y, Wq, Ws, am = _check(mq, layers, M)
    K = layers[0].K
    n0, kb = 0, 8 * ((K + 255) // 256)
    per_layer = M > 128 and any(wl.N % 256 for wl in layers)
    for g, wl in enumerate(layers):
        ys = mq.macaq_w4a4_linear(x.cuda(), am[g].contiguous(), Wq[n0:n0 + wl.N].contiguous(),
                                  Ws[n0 * kb: (n0 + wl.N) * kb].contiguous(), wl.N)
        torch.cuda.synchronize()
        blk = y[:, n0:n0 + wl.N]
        if per_layer:
            assert torch.equal(blk, ys)
        else:
            assert gu.rel_fro(gu.to_np(blk.float()), gu.to_np(ys.float())) <= 1e-3
        n0 += wl.N
