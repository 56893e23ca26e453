"""GPU parity of the block-scaled MXFP4 GEMM and the fused W4A4 linear against the fp64
oracle.

Identical codes ("MACaQ", Abstract: MXFP4 W4A4 matmul): the oracle contracts the GPU's own
codes and scales exactly in fp64.  Gates (relative Frobenius error):
  * fp32 output vs the exact result                     <= 1e-3 (fp32 accumulation: ~1e-6)
  * bf16 output vs bf16-rounded exact result             <= 1e-3
The error of the bf16 output against the unrounded exact result is dominated by bf16's 8
significand bits (~1.5e-3 relative RMS); it is reported, not gated.
Shapes span several tiles with ragged M, N and K tails, both kernel orientations (swap-AB
for M <= 128, 128x256 tiles above), every MMA-N width, and both schedules: stream-K (tiles
split across CTAs, fp32 partials added by the tile's owner) and data-parallel."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wls
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


def random_mx(rng, rows, K, lo=118, hi=136):
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.integers(lo, hi, (rows, K // 32), dtype=np.uint8)
    return codes, scales


def to_device_mx(codes, scales, rows, K):
    return (torch.from_numpy(codes).cuda(),
            torch.from_numpy(layout.rowmajor_to_tiled(scales, rows, K)).cuda())


SHAPES = [
    (1, 256, 256), (1, 7, 32), (4, 136, 96), (16, 384, 512), (17, 200, 288), (33, 520, 800),
    (64, 256, 1024), (65, 130, 256), (100, 1000, 800), (128, 128, 256), (129, 300, 320),
    (256, 512, 512), (300, 520, 1056), (511, 777, 640), (1024, 2048, 2048),
    # long K, few tiles: stream-K splits tiles between CTAs (owner + 1 contributor for
    # tiles of <= 32 K steps, up to 3 for longer ones), swap-AB and CTA-pair kernels
    # (1280 x 2048: 40 tiles on 74 pairs)
    (16, 2048, 8192), (200, 1024, 8192), (70, 1100, 6144), (16, 1024, 16384), (1280, 2048, 16384),
]


@pytest.mark.parametrize("M,N,K", SHAPES, ids=lambda v: str(v))
def test_gemm_identical_codes(mq, M, N, K):
    rng = np.random.default_rng(M * 131 + N * 7 + K)
    Ac, As = random_mx(rng, M, K)
    Wc, Ws = random_mx(rng, N, K)
    Ag, Asg = to_device_mx(Ac, As, M, K)
    Wg, Wsg = to_device_mx(Wc, Ws, N, K)
    y32 = mq.macaq_mxfp4_gemm(Ag, Asg, Wg, Wsg, M, N, K, out_fp32=True)
    y16 = mq.macaq_mxfp4_gemm(Ag, Asg, Wg, Wsg, M, N, K)
    y32dp = mq.macaq_mxfp4_gemm(Ag, Asg, Wg, Wsg, M, N, K, out_fp32=True, data_parallel=True)
    torch.cuda.synchronize()
    ref = oracle.mx_gemm(Ac, As, Wc, Ws)
    # both schedules (stream-K fix-up and data-parallel) meet the gate
    assert gu.rel_fro(gu.to_np(y32dp), ref) <= TOL
    e32 = gu.rel_fro(gu.to_np(y32), ref)
    e16 = gu.rel_fro(gu.to_np(y16.float()), gu.bf16_round(ref))
    e16_raw = gu.rel_fro(gu.to_np(y16.float()), ref)
    print(f"M={M} N={N} K={K}: fp32 {e32:.2e}  bf16-vs-rounded {e16:.2e}  bf16-vs-exact {e16_raw:.2e}")
    assert e32 <= TOL
    assert e16 <= TOL
    # every output element is written (no stale memory): max abs error bounded too
    assert np.max(np.abs(gu.to_np(y32) - ref)) <= 1e-3 * np.max(np.abs(ref)) + 1e-30


# both shapes take the stream-K schedule (one-CTA swap-AB and CTA-pair kernels)
@pytest.mark.parametrize("M,N,K", [(16, 2048, 8192), (300, 2048, 16384)], ids=lambda v: str(v))
def test_streamk_workspace_reused_and_dirty(mq, M, N, K):
    """Stream-K hand-off through a workspace that is reused call after call and starts with
    arbitrary bytes (flag words only count when they hold the current launch's tag): five
    calls in a row, each bit-identical to the first."""
    rng = np.random.default_rng(M + K)
    Ac, As = random_mx(rng, M, K)
    Wc, Ws = random_mx(rng, N, K)
    Ag, Asg = to_device_mx(Ac, As, M, K)
    Wg, Wsg = to_device_mx(Wc, Ws, N, K)
    ws = torch.randint(0, 256, (mq.gemm_workspace_bytes(M, N, K),), dtype=torch.uint8, device="cuda")
    ys = [mq.macaq_mxfp4_gemm(Ag, Asg, Wg, Wsg, M, N, K, out_fp32=True, workspace=ws) for _ in range(5)]
    torch.cuda.synchronize()
    assert mq.macaq_device_status() == 0
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    assert gu.rel_fro(gu.to_np(ys[0]), oracle.mx_gemm(Ac, As, Wc, Ws)) <= TOL


@pytest.mark.parametrize("M,N,K", [(16, 2048, 8192), (300, 2048, 16384)], ids=lambda v: str(v))
def test_streamk_graph_replays_with_new_inputs(mq, M, N, K):
    """A stream-K GEMM captured in a CUDA graph is replayed with the same launch tag every
    time; each replay here gets new operand codes (copied into the captured buffers) and must
    give exactly what an eager call on those codes gives, i.e. no owner may take a flag left
    set by the previous replay for its own contributor's signal."""
    rng = np.random.default_rng(7 * M + K)
    inputs = []
    for _ in range(4):
        Ac, As = random_mx(rng, M, K)
        Wc, Ws = random_mx(rng, N, K)
        inputs.append((*to_device_mx(Ac, As, M, K), *to_device_mx(Wc, Ws, N, K)))
    bufs = [t.clone() for t in inputs[0]]
    ws = torch.empty(mq.gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    expect = [mq.macaq_mxfp4_gemm(*inp, M, N, K, out_fp32=True, workspace=ws).clone() for inp in inputs]
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        mq.macaq_mxfp4_gemm(*bufs, M, N, K, y=y, out_fp32=True, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        mq.macaq_mxfp4_gemm(*bufs, M, N, K, y=y, out_fp32=True, workspace=ws)
    for r in range(8):
        for dst, src in zip(bufs, inputs[r % 4]):
            dst.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, expect[r % 4]), f"replay {r} differs from the eager result"
    assert mq.macaq_device_status() == 0


def test_gemm_exact_small_integers(mq):
    # all elements in {0, +-0.5, +-1} and scale 127: every partial sum is exact in fp32
    rng = np.random.default_rng(5)
    M, N, K = 140, 264, 768
    pick = np.array([0x0, 0x1, 0x2, 0x9, 0xA], np.uint8)
    Ac = (pick[rng.integers(0, 5, (M, K))][:, 0::2] | (pick[rng.integers(0, 5, (M, K))][:, 1::2] << 4)).astype(np.uint8)
    Wc = (pick[rng.integers(0, 5, (N, K))][:, 0::2] | (pick[rng.integers(0, 5, (N, K))][:, 1::2] << 4)).astype(np.uint8)
    As = np.full((M, K // 32), 127, np.uint8)
    Ws = np.full((N, K // 32), 127, np.uint8)
    y = mq.macaq_mxfp4_gemm(*to_device_mx(Ac, As, M, K), *to_device_mx(Wc, Ws, N, K), M, N, K, out_fp32=True)
    assert np.array_equal(gu.to_np(y), oracle.mx_gemm(Ac, As, Wc, Ws))


@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (512, 512, 1024), (384, 768, 2048)], ids=lambda v: str(v))
def test_gemm_scale_placement(mq, M, N, K):
    # one distinct scale per (row, block) on both sides: a scale read from the wrong row,
    # block, TMEM column, lane quadrant or replica shows up as a wrong power of two in an
    # isolated product.  M <= 128 runs the one-CTA kernel, M > 128 the CTA-pair kernel.
    nb = K // 32
    Ac = np.zeros((M, K // 2), np.uint8)
    Wc = np.zeros((N, K // 2), np.uint8)
    rng = np.random.default_rng(9 + M)
    As = rng.integers(110, 140, (M, nb), dtype=np.uint8)
    Ws = rng.integers(110, 140, (N, nb), dtype=np.uint8)
    # A row m has a single 1.0 in block m % nb; W row n has a single 1.0 in block (n // 3) % nb
    for m in range(M):
        Ac[m, 16 * (m % nb)] = 0x02
    for n in range(N):
        Wc[n, 16 * ((n // 3) % nb)] = 0x02
    y = gu.to_np(mq.macaq_mxfp4_gemm(*to_device_mx(Ac, As, M, K), *to_device_mx(Wc, Ws, N, K), M, N, K,
                                     out_fp32=True))
    ref = oracle.mx_gemm(Ac, As, Wc, Ws)
    assert np.count_nonzero(ref) > 0
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("wl", [wls.LLAMA_UP, wls.QWEN_UP_DECODE.with_m(1), wls.QWEN_UP_DECODE.with_m(4),
                                wls.QWEN_UP_DECODE.with_m(16), wls.QWEN_DOWN],
                         ids=lambda w: f"{w.name}_M{w.M}")
def test_full_size_gemm_and_linear_sampled(mq, wl):
    """Full-size shapes in the launch configuration the benchmark times; the oracle checks
    a seeded sample of rows (all rows for decode) on the GPU's own codes, and the fused
    linear must reproduce the two-call path bit for bit."""
    x = wls.make_x(wl)
    W = wls.make_w(wl)
    s = wls.make_s(wl, W)
    Wq, Ws, am = mq.macaq_fold_weights(W.cuda(), s.cuda())
    del W
    xg = x.cuda()
    Aq, As = mq.macaq_act_transform_quant(xg, am)
    y32 = mq.macaq_mxfp4_gemm(Aq, As, Wq, Ws, wl.M, wl.N, wl.K, out_fp32=True)
    y16 = mq.macaq_mxfp4_gemm(Aq, As, Wq, Ws, wl.M, wl.N, wl.K)
    yl = mq.macaq_w4a4_linear(xg, am, Wq, Ws, wl.N)
    torch.cuda.synchronize()
    assert torch.equal(yl, y16), "fused linear differs from transform-then-GEMM"
    rng = np.random.default_rng(wl.config)
    rows = np.arange(wl.M) if wl.M <= 64 else np.sort(rng.choice(wl.M, 24, replace=False))
    Ac = gu.to_np(Aq)
    Asr = layout.tiled_to_rowmajor(gu.to_np(As), wl.M, wl.K)
    Wc = gu.to_np(Wq)
    Wsr = layout.tiled_to_rowmajor(gu.to_np(Ws), wl.N, wl.K)
    ref = oracle.mx_gemm(Ac, Asr, Wc, Wsr, rows)
    e32 = gu.rel_fro(gu.to_np(y32)[rows], ref)
    e16 = gu.rel_fro(gu.to_np(y16.float())[rows], gu.bf16_round(ref))
    print(f"{wl.name} M={wl.M}: fp32 {e32:.2e} bf16 {e16:.2e} ({rows.size} rows)")
    assert e32 <= TOL and e16 <= TOL
