"""A bounded device-side wait that runs out: the stream-K owner's wait for a contributor's flag.

Every wait inside the library's kernels is bounded; when one gives up, the kernel records
MACAQ_ETIMEOUT in a device status word (macaq_device_status) and finishes instead of hanging.
The product build bounds these waits at ~4 s, which no test can reach, so this test loads the
fault-injection build of the library (online_hadamard_b200/build.py: the owner's flag wait
bounded at 200 000 cycles, and a host hook that makes owners wait for a tag no contributor
writes).  The failure is made on the host: nothing faults, traps or spins without a bound.

Shape: a prefill GEMM on the CTA-pair kernel whose last wave is split along K (stream-K).  There
an owner waits for its contributors only after its own accumulator is in registers and the
split tile is the last item of its CTA, so when the wait runs out no tensor-core or copy work
of that CTA is still in flight."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

MACAQ_ETIMEOUT = -5


@pytest.fixture(scope="module")
def libs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import online_hadamard_b200 as mq
    from online_hadamard_b200 import build as b
    mq.load_library()
    fault = mq.load_library(b.build_fault_library())
    fault.macaq_test_owner_tag_offset.argtypes = [ctypes.c_int64]
    fault.macaq_test_owner_tag_offset.restype = None
    return mq, fault


def _gemm(lib, Aq, As, Wq, Ws, M, N, K, ws):
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib.macaq_mxfp4_gemm(P(Aq), P(As), M, P(Wq), P(Ws), N, K, P(y), 0, P(ws), ws.numel(),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    return y


def test_owner_flag_wait_runs_out_and_is_reported(libs):
    mq, fault = libs
    M, N, K = 3072, 1792, 16384  # 84 pair tiles of 64 K steps: stream-K over the last wave
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(M, K, generator=g) * 2).to(torch.bfloat16).cuda()
    W = (torch.randn(N, K, generator=g) * 0.02).cuda()
    Wq, Ws, am = mq.macaq_fold_weights(W, torch.ones(K, device="cuda"))
    Aq, As = mq.macaq_act_transform_quant(x, am)
    ws = torch.empty(mq.gemm_workspace_bytes(M, N, K), dtype=torch.uint8, device="cuda")
    ref = mq.macaq_mxfp4_gemm(Aq, As, Wq, Ws, M, N, K, workspace=ws)
    torch.cuda.synchronize()
    assert fault.macaq_device_status(1) == 0  # cleared

    # owners wait for a tag that no contributor writes: each owner's wait runs out
    fault.macaq_test_owner_tag_offset(1)
    try:
        _gemm(fault, Aq, As, Wq, Ws, M, N, K, ws)
        torch.cuda.synchronize()
    finally:
        fault.macaq_test_owner_tag_offset(0)
    assert fault.macaq_device_status(0) == MACAQ_ETIMEOUT  # recorded, and still set
    assert fault.macaq_device_status(1) == MACAQ_ETIMEOUT  # read and cleared
    assert fault.macaq_device_status(0) == 0

    # the context stays usable: the same call completes normally and matches the product library
    y = _gemm(fault, Aq, As, Wq, Ws, M, N, K, ws)
    torch.cuda.synchronize()
    assert fault.macaq_device_status(0) == 0
    assert torch.equal(y, ref)
    assert mq.macaq_device_status() == 0  # the product library's own status was never touched
