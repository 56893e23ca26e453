"""GPU parity of the per-channel scale calibration against the oracle: bit-exact (column
maxima are exact; quotient and root are correctly rounded in double on both sides, then
rounded once to fp32)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wls

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import online_hadamard_b200 as m
    m.load_library()
    return m


@pytest.mark.parametrize("C,N,K", [(64, 128, 256), (3, 1000, 544), (64, 257, 96), (1, 1, 32)], ids=lambda v: str(v))
def test_calibrate_matches_oracle(mq, C, N, K):
    g = torch.Generator().manual_seed(C * 7 + N + K)
    xcal = (torch.randn(C, K, generator=g) * torch.rand(K, generator=g) * 30).to(torch.bfloat16)
    W = torch.randn(N, K, generator=g) * torch.rand(K, generator=g) * 0.05
    if K > 40:
        xcal[:, 5] = 0  # zero activation column -> 1
        W[:, 37] = 0    # zero weight column -> 1
        W[:, 7] = -W[:, 7]
    s = mq.macaq_calibrate_scale(xcal.cuda(), W.cuda())
    torch.cuda.synchronize()
    ref = oracle.calibrate_scale(xcal.float().numpy(), W.numpy())
    assert np.array_equal(s.cpu().numpy(), ref)


def test_calibrate_full_layer_and_config_scales(mq):
    """A Qwen3-32B-sized layer (25600 x 5120 fp32 weights), and the scales the workloads use."""
    wl = wls.QWEN_UP_DECODE.with_m(16)
    W = wls.make_w(wl)
    xcal = wls.make_xcal(wl)
    s = mq.macaq_calibrate_scale(xcal.cuda(), W.cuda())
    torch.cuda.synchronize()
    ref = oracle.calibrate_scale(xcal.float().numpy(), W.numpy())
    assert np.array_equal(s.cpu().numpy(), ref)
    assert np.array_equal(s.cpu().numpy(), wls.make_s(wl, W).numpy())
