"""GPU parity of the activation transform + MXFP4 quantisation and of the weight fold
against the CPU oracle: codes and E8M0 scales bit-exact (mismatches allowed only within
1 fp32 ulp of a rounding boundary, counted), multipliers bit-exact.

"MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision Weights and
Activations", Abstract: per-channel scale + block-Hadamard online on the activations,
inverse transforms folded into the weights, MXFP4 W4A4, round-to-nearest weights."""
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


ACT_CASES = [
    wls.TINY,
    wls.LLAMA_UP,
    wls.QWEN_UP_DECODE.with_m(1),
    wls.QWEN_UP_DECODE.with_m(4),
    wls.QWEN_UP_DECODE.with_m(16),
    wls.QWEN_DOWN,
]


@pytest.mark.parametrize("wl", ACT_CASES, ids=lambda w: f"{w.name}_M{w.M}")
def test_act_transform_quant_matches_oracle(mq, wl):
    x = wls.make_x(wl)
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    del W
    a, _ = oracle.multipliers(s.numpy())
    Aq, As = mq.macaq_act_transform_quant(x.cuda(), torch.from_numpy(a).cuda())
    torch.cuda.synchronize()
    xf = x.float().numpy()
    V = oracle.transform_f32(xf, a)
    rc, rs = oracle.quantize_mx(V)
    stats = gu.compare_mx(gu.to_np(Aq), gu.to_np(As), rc, rs, wl.M, wl.K, V, label=gu.config_label(wl, "act"))
    print(wl.name, wl.M, stats)


@pytest.mark.parametrize("M,K", [(1037, 4128), (4099, 1056), (64, 65600), (4099, 4128)], ids=lambda v: str(v))
def test_act_quant_large_ragged(mq, M, K):
    """Inputs above the small-input size, so the whole-block kernel (one thread per 32-element
    block, rows walked two at a time, or one row ahead for transforms of 16 M elements and
    more: the last case) runs, with row counts that leave a thread an odd last row and K that
    is not a multiple of 256 (padded scale blocks): transform and plain codes against the
    oracle."""
    assert M * K > (1 << 22)
    rng = np.random.default_rng(M + K)
    xf32 = rng.standard_t(4, (M, K)).astype(np.float32) * rng.uniform(0.1, 30.0, (1, K)).astype(np.float32)
    xb = torch.from_numpy(xf32).to(torch.bfloat16)
    s = rng.uniform(0.05, 5.0, K).astype(np.float32)
    a, _ = oracle.multipliers(s)
    Aq, As = mq.macaq_act_transform_quant(xb.cuda(), torch.from_numpy(a).cuda())
    Pq, Ps = mq.macaq_act_quant_plain(xb.cuda())
    torch.cuda.synchronize()
    xf = xb.float().numpy()
    V = oracle.transform_f32(xf, a)
    rc, rs = oracle.quantize_mx(V)
    gu.compare_mx(gu.to_np(Aq), gu.to_np(As), rc, rs, M, K, V, label="large ragged act")
    pc, ps = oracle.quantize_mx(xf)
    gu.compare_mx(gu.to_np(Pq), gu.to_np(Ps), pc, ps, M, K, xf, label="large ragged plain")


@pytest.mark.parametrize("wl", [wls.TINY, wls.LLAMA_UP, wls.QWEN_DOWN], ids=lambda w: w.name)
def test_act_quant_plain_matches_oracle(mq, wl):
    x = wls.make_x(wl)
    Aq, As = mq.macaq_act_quant_plain(x.cuda())
    torch.cuda.synchronize()
    xf = x.float().numpy()
    rc, rs = oracle.act_quant_plain(xf)
    gu.compare_mx(gu.to_np(Aq), gu.to_np(As), rc, rs, wl.M, wl.K, xf, label=gu.config_label(wl, "plain"))


@pytest.mark.parametrize("wl", [wls.TINY, wls.LLAMA_UP, wls.QWEN_UP_DECODE, wls.QWEN_DOWN], ids=lambda w: w.name)
def test_fold_weights_matches_oracle(mq, wl):
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    Wq, Ws, am = mq.macaq_fold_weights(W.cuda(), s.cuda())
    torch.cuda.synchronize()
    a, w = oracle.multipliers(s.numpy())
    assert np.array_equal(gu.to_np(am).view(np.uint32), a.view(np.uint32))
    V = oracle.transform_f32(W.numpy(), w)
    rc, rs = oracle.quantize_mx(V)
    stats = gu.compare_mx(gu.to_np(Wq), gu.to_np(Ws), rc, rs, wl.N, wl.K, V, label=gu.config_label(wl, "fold"))
    print(wl.name, stats)


def _edge_inputs():
    rng = np.random.default_rng(77)
    cases = []
    cases.append(("k32_m1", rng.standard_normal((1, 32))))
    cases.append(("k96_m3_padded_blocks", rng.standard_normal((3, 96)) * 5))
    cases.append(("k288_m130_ragged", rng.standard_normal((130, 288))))
    cases.append(("zeros", np.zeros((5, 256))))
    z = np.zeros((4, 64))
    z[1] = -0.0
    z[2, ::3] = -0.0
    z[3, 7] = -1.0
    cases.append(("signed_zeros", z))
    cases.append(("huge", rng.standard_normal((4, 256)) * 1e34))
    cases.append(("subnormal_range", rng.standard_normal((6, 256)) * 1e-38))
    cases.append(("mixed_binades", rng.standard_normal((33, 512)) * 10.0 ** rng.integers(-20, 20, (33, 1))))
    cases.append(("m257_k1056", rng.standard_t(3, (257, 1056))))
    return cases


@pytest.mark.parametrize("name,x", _edge_inputs(), ids=[c[0] for c in _edge_inputs()])
def test_act_transform_quant_edge_cases(mq, name, x):
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    M, K = xb.shape
    rng = np.random.default_rng(M * 7 + K)
    s = rng.uniform(0.05, 5.0, K).astype(np.float32)
    a, _ = oracle.multipliers(s)
    Aq, As = mq.macaq_act_transform_quant(xb.cuda(), torch.from_numpy(a).cuda())
    Pq, Ps = mq.macaq_act_quant_plain(xb.cuda())
    torch.cuda.synchronize()
    xf = xb.float().numpy()
    V = oracle.transform_f32(xf, a)
    rc, rs = oracle.quantize_mx(V)
    gu.compare_mx(gu.to_np(Aq), gu.to_np(As), rc, rs, M, K, V, label="edge cases act")
    pc, ps = oracle.quantize_mx(xf)
    gu.compare_mx(gu.to_np(Pq), gu.to_np(Ps), pc, ps, M, K, xf, label="edge cases plain")


def test_fold_rejects_invalid_scale(mq):
    W = torch.randn(8, 64, device="cuda")
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        s = torch.ones(64, device="cuda")
        s[5] = bad
        with pytest.raises(mq.MacaqError) as ei:
            mq.macaq_fold_weights(W, s)
        assert ei.value.status == -1


def test_scale_buffer_layout_roundtrip_on_device(mq):
    # a kernel-written buffer decodes through the documented index map
    x = torch.zeros(200, 512, dtype=torch.bfloat16)
    for r in range(200):
        for b in range(16):
            x[r, 32 * b] = 2.0 ** ((r + 3 * b) % 40 - 20)  # block max sets the scale byte
    Aq, As = mq.macaq_act_quant_plain(x.cuda())
    S = layout.tiled_to_rowmajor(gu.to_np(As), 200, 512)
    expect = np.array([[(r + 3 * b) % 40 - 20 + 127 - 2 for b in range(16)] for r in range(200)])
    assert np.array_equal(S, expect)


@pytest.mark.parametrize("rows,K", [(1, 32), (200, 1056), (300, 4096), (129, 96)], ids=str)
def test_scale_layout_conversions(mq, rows, K):
    """Row-major E8M0 scales to the MMA tile layout and back, against the documented index map
    (tests/layout.py), padded blocks and rows zero; and the quantiser's own scales round-trip."""
    rng = np.random.default_rng(rows + K)
    S = rng.integers(0, 255, (rows, K // 32)).astype(np.uint8)
    tiled = mq.macaq_scales_to_tiled(torch.from_numpy(S).cuda(), K)
    back = mq.macaq_scales_to_rowmajor(tiled, rows, K)
    torch.cuda.synchronize()
    assert np.array_equal(gu.to_np(tiled), layout.rowmajor_to_tiled(S, rows, K))
    assert np.array_equal(gu.to_np(back), S)
    x = (torch.randn(rows, K) * 3).to(torch.bfloat16).cuda()
    Aq, As = mq.macaq_act_quant_plain(x)
    rm = mq.macaq_scales_to_rowmajor(As, rows, K)
    torch.cuda.synchronize()
    assert np.array_equal(gu.to_np(rm), layout.tiled_to_rowmajor(gu.to_np(As), rows, K))
