"""The C ABI: the library loads, exports every symbol include/macaq.h declares, and its
host-side helpers and argument validation behave as documented (no GPU needed: every
case here returns before any CUDA call)."""
import ctypes
import os
import re

import numpy as np
import pytest

import online_hadamard_b200 as mq
from tests import layout

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "macaq.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(macaq_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(mq.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = mq.load_library()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # and through the dynamic symbol table directly
    raw = ctypes.CDLL(mq._build_mod.LIB_PATH)
    for name in declared_symbols():
        assert ctypes.cast(getattr(raw, name), ctypes.c_void_p).value


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert mq.status_str(code).startswith("MACAQ")


@pytest.mark.parametrize("rows,K", [(1, 32), (16, 256), (129, 96), (2048, 4096), (300, 25600), (5, 800)])
def test_scale_layout_helpers_match_documentation(rows, K):
    assert mq.scale_bytes(rows, K) == layout.scale_bytes(rows, K)
    idx = layout.scale_index(rows, K, layout.padded_blocks(K))
    rng = np.random.default_rng(rows + K)
    for _ in range(50):
        r = int(rng.integers(rows))
        kb = int(rng.integers(layout.padded_blocks(K)))
        assert mq.scale_offset(r, kb, K) == idx[r, kb]
    # the map is a bijection onto the buffer when rows fill whole 128-row atoms
    full = layout.scale_index(((rows + 127) // 128) * 128, K, layout.padded_blocks(K))
    assert np.array_equal(np.sort(full.ravel()), np.arange(layout.scale_bytes(rows, K)))


def test_size_helpers_reject_bad_shapes():
    assert mq.scale_bytes(0, 256) == 0
    assert mq.scale_bytes(4, 48) == 0
    assert mq.scale_offset(0, 8, 256) == -1
    assert mq.linear_workspace_bytes(16, 64, 33) == 0
    assert mq.gemm_workspace_bytes(0, 64, 32) == 0


FAKE = 0x10000  # aligned, never dereferenced: every call below fails validation first
MIS = 0x10008


def _call(name, *args):
    lib = mq.load_library()
    return getattr(lib, name)(*args)


def test_validation_null_shape_alignment():
    P = ctypes.c_void_p
    # null pointers
    assert _call("macaq_act_transform_quant", None, 4, 64, P(FAKE), P(FAKE), P(FAKE), None) == -1
    assert _call("macaq_mxfp4_gemm", P(FAKE), P(FAKE), 4, P(FAKE), P(FAKE), 8, 64, None, 0, None, 0, None) == -1
    # shapes
    assert _call("macaq_act_transform_quant", P(FAKE), 4, 48, P(FAKE), P(FAKE), P(FAKE), None) == -2
    assert _call("macaq_act_quant_plain", P(FAKE), 0, 64, P(FAKE), P(FAKE), None) == -2
    assert _call("macaq_mxfp4_gemm", P(FAKE), P(FAKE), 4, P(FAKE), P(FAKE), 0, 64, P(FAKE), 0, None, 0, None) == -2
    assert _call("macaq_fold_weights", P(FAKE), 8, 16, P(FAKE), P(FAKE), P(FAKE), P(FAKE), None) == -2
    # alignment
    assert _call("macaq_act_transform_quant", P(MIS), 4, 64, P(FAKE), P(FAKE), P(FAKE), None) == -3
    assert _call("macaq_mxfp4_gemm", P(FAKE), P(FAKE), 4, P(FAKE), P(FAKE), 8, 64, P(MIS), 0, None, 0, None) == -3
    assert _call("macaq_mxfp4_gemm", P(FAKE), P(FAKE), 4, P(FAKE), P(FAKE), 8, 64, P(FAKE), 0, P(MIS), 1 << 30,
                 None) == -3
    # bad flag
    assert _call("macaq_mxfp4_gemm", P(FAKE), P(FAKE), 4, P(FAKE), P(FAKE), 8, 64, P(FAKE), 2, None, 0, None) == -1


def test_calibrate_scale_validation():
    P = ctypes.c_void_p
    assert _call("macaq_calibrate_scale", None, 64, P(FAKE), 128, 256, P(FAKE), None) == -1
    assert _call("macaq_calibrate_scale", P(FAKE), 64, P(FAKE), 128, 256, None, None) == -1
    assert _call("macaq_calibrate_scale", P(FAKE), 0, P(FAKE), 128, 256, P(FAKE), None) == -2
    assert _call("macaq_calibrate_scale", P(FAKE), 64, P(FAKE), 0, 256, P(FAKE), None) == -2
    assert _call("macaq_calibrate_scale", P(FAKE), 64, P(FAKE), 128, 200, P(FAKE), None) == -2
    assert _call("macaq_calibrate_scale", P(FAKE), 64, P(MIS), 128, 256, P(FAKE), None) == -3


def test_grouped_linear_validation_and_sizes():
    import numpy as np
    P = ctypes.c_void_p
    lib = mq.load_library()

    def counts(*c):
        a = np.array(c, dtype=np.int64)
        return a, P(a.ctypes.data)

    c, cp = counts(3, 0, 130)
    # workspace: every expert padded to whole 128-row blocks (128 + 0 + 256 rows)
    assert mq.grouped_workspace_bytes(c, 256, 512) == 384 * 256 + 384 * 16
    assert mq.grouped_workspace_bytes(c, 200, 512) == 0          # N % 128 != 0
    assert mq.grouped_workspace_bytes([-1, 4], 256, 512) == 0    # negative count
    assert mq.grouped_workspace_bytes([1] * 129, 256, 512) == 0  # more than 128 experts
    call = lambda cp_, E, N, x=FAKE, y=FAKE, ws=FAKE, wsb=1 << 30: lib.macaq_w4a4_grouped_linear(
        P(x), cp_, E, 512, P(FAKE), P(FAKE), P(FAKE), N, P(y), P(ws), wsb, None)
    assert lib.macaq_w4a4_grouped_linear(P(FAKE), None, 3, 512, P(FAKE), P(FAKE), P(FAKE), 256, P(FAKE), P(FAKE),
                                         1 << 30, None) == -1
    assert call(cp, 0, 256) == -2
    assert call(cp, 3, 200) == -2
    assert call(cp, 3, 256, x=MIS) == -3
    assert call(cp, 3, 256, wsb=1000) == -6
    z, zp = counts(0, 0, 0)
    assert call(zp, 3, 256, x=0, y=0, ws=0) == 0  # no token routed: nothing to do, nothing launched


def test_noalloc_linear_validation():
    """The no-allocation linear rejects bad arguments, and problems whose activation codes and
    scales exceed its fixed scratch, before it touches the device."""
    P = ctypes.c_void_p
    lib = mq.load_library()
    call = lambda M, K, N, x=FAKE, y=FAKE: lib.macaq_w4a4_linear_noalloc(P(x), M, K, P(FAKE), P(FAKE), P(FAKE), N,
                                                                           P(y), None)
    assert lib.macaq_w4a4_linear_noalloc(None, 4, 256, P(FAKE), P(FAKE), P(FAKE), 128, P(FAKE), None) == -1
    assert call(0, 256, 128) == -2
    assert call(4, 250, 128) == -2
    assert call(4, 256, 0) == -2
    assert call(4, 256, 128, x=MIS) == -3
    assert call(4, 256, 128, y=MIS) == -3
    # 65536 x 1024 activations: 32 MiB of codes alone, beyond the 32 MiB scratch
    assert call(65536, 1024, 128) == -7


def test_binding_refuses_host_tensors_and_short_buffers():
    """The Python binding hands the library bare pointers, so it checks what the C ABI cannot:
    host tensors are refused (there is no CPU path), and a buffer shorter than the call needs
    is refused before any pointer reaches a kernel."""
    import pytest
    import torch
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mq.macaq_act_transform_quant(x, torch.ones(256))
    with pytest.raises(ValueError, match="CUDA tensor"):
        mq.macaq_w4a4_linear(x, torch.ones(256), torch.zeros(128, 128, dtype=torch.uint8),
                             torch.zeros(mq.scale_bytes(128, 256), dtype=torch.uint8), 128)
    with pytest.raises(ValueError, match="CUDA tensor"):
        mq.macaq_w4a4_linear_multi(x, torch.ones(2, 256), torch.zeros(384, 128, dtype=torch.uint8),
                                   torch.zeros(mq.scale_bytes(256, 256) + mq.scale_bytes(128, 256), dtype=torch.uint8),
                                   (256, 128))
    with pytest.raises(ValueError, match="needs at least"):
        mq._need_numel(torch.zeros(mq.scale_bytes(128, 256) - 1, dtype=torch.uint8), "Ws", mq.scale_bytes(128, 256))
    mq._need_numel(torch.zeros(mq.scale_bytes(128, 256), dtype=torch.uint8), "Ws", mq.scale_bytes(128, 256))


def test_binding_refuses_a_stream_of_another_device():
    """Kernels run on the stream's device: a stream of another GPU than the tensors' would make
    them read this GPU's memory through pointers the other one cannot use, so it is refused
    before the call."""
    import types

    import pytest
    import torch
    dev0 = torch.device("cuda", 0)
    with pytest.raises(ValueError, match="stream belongs to cuda:1"):
        mq._check_stream_device(types.SimpleNamespace(device=torch.device("cuda", 1)), dev0)
    with pytest.raises(ValueError, match="stream belongs to cpu"):
        mq._check_stream_device(types.SimpleNamespace(device=torch.device("cpu")), dev0)
    mq._check_stream_device(types.SimpleNamespace(device=torch.device("cuda", 0)), dev0)
    mq._check_stream_device(types.SimpleNamespace(device="cuda:0"), dev0)


def test_fault_injection_hook_only_in_the_test_build():
    """The tag-offset hook exists only in the fault-injection build that one GPU test loads; the
    product library does not export it."""
    import ctypes

    from online_hadamard_b200 import build as b
    fault = ctypes.CDLL(b.build_fault_library())
    assert hasattr(fault, "macaq_test_owner_tag_offset")
    assert not hasattr(mq.load_library(), "macaq_test_owner_tag_offset")


def test_validation_of_the_offline_and_grouped_device_calls():
    """Flip-Refinement, the calibration Hessian, the device-count grouped linear and the scale-layout
    conversions refuse bad arguments before any CUDA call (fake pointers are never used)."""
    P = ctypes.c_void_p
    lib = mq.load_library()
    # sizes: pure host arithmetic
    assert lib.macaq_hessian_workspace_bytes(64, 256) == 64 * 256 * 4
    assert lib.macaq_hessian_workspace_bytes(64, 200) == 0
    assert lib.macaq_flip_refine_workspace_bytes(300, 1024) == 300 * 1024 * 12
    assert lib.macaq_flip_refine_workspace_bytes(5000, 1024) == 2048 * 1024 * 12  # one chunk of rows
    assert lib.macaq_flip_refine_workspace_bytes(4, 12320) == 0                  # K above the limit
    assert lib.macaq_grouped_device_workspace_bytes(128, 129, 256, 512) == 0      # more than 128 experts
    assert lib.macaq_grouped_device_workspace_bytes(128, 16, 200, 512) == 0       # N % 128 != 0
    assert lib.macaq_grouped_device_workspace_bytes(128, 16, 256, 512) > 0
    # macaq_calib_hessian(xcal, C, K, act_mult, Hs, ws, ws_bytes, stream)
    assert _call("macaq_calib_hessian", None, 64, 256, P(FAKE), P(FAKE), P(FAKE), 1 << 20, None) == -1
    assert _call("macaq_calib_hessian", P(FAKE), 64, 200, P(FAKE), P(FAKE), P(FAKE), 1 << 20, None) == -2
    assert _call("macaq_calib_hessian", P(FAKE), 64, 256, P(MIS), P(FAKE), P(FAKE), 1 << 20, None) == -3
    assert _call("macaq_calib_hessian", P(FAKE), 64, 256, P(FAKE), P(FAKE), P(FAKE), 100, None) == -6
    # macaq_flip_refine(W, N, K, s, Hs, Wq, Ws, max_moves, moves, ws, ws_bytes, stream)
    ok = (P(FAKE), 300, 1024, P(FAKE), P(FAKE), P(FAKE), P(FAKE))
    assert _call("macaq_flip_refine", *ok, -1, None, P(FAKE), 1 << 30, None) == -1        # negative budget
    assert _call("macaq_flip_refine", None, *ok[1:], 8, None, P(FAKE), 1 << 30, None) == -1
    assert _call("macaq_flip_refine", P(FAKE), 300, 12320, *ok[3:], 8, None, P(FAKE), 1 << 30, None) == -2
    assert _call("macaq_flip_refine", *ok, 8, P(MIS), P(FAKE), 1 << 30, None) == -3       # moves misaligned
    assert _call("macaq_flip_refine", *ok, 8, None, P(FAKE), 1000, None) == -6            # workspace too small
    # macaq_w4a4_grouped_linear_device(x, T, counts, counts_bytes, E, capacity, K, act_mult, Wq, Ws, N, y, ws,
    #                                  ws_bytes, stream)
    g = lambda **kw: _call("macaq_w4a4_grouped_linear_device", kw.get("x", P(FAKE)), kw.get("T", 128),
                           kw.get("counts", P(FAKE)), kw.get("cb", 4), kw.get("E", 16), 0, kw.get("K", 512),
                           P(FAKE), P(FAKE), P(FAKE), kw.get("N", 256), P(FAKE), P(FAKE), kw.get("wsb", 1 << 30),
                           None)
    assert g(counts=None) == -1
    assert g(cb=3) == -1
    assert g(E=129) == -2 and g(E=0) == -2
    assert g(N=200) == -2 and g(K=48) == -2 and g(T=0) == -2
    assert g(counts=P(FAKE + 2)) == -3                                                     # int32 counts misaligned
    assert g(wsb=1000) == -6
    # layout conversions
    assert _call("macaq_scales_to_tiled", None, 4, 64, P(FAKE), None) == -1
    assert _call("macaq_scales_to_rowmajor", P(FAKE), 4, 48, P(FAKE), None) == -2


def test_linear_multi_validation_and_sizes():
    """The stacked-linears call refuses bad arguments before any CUDA call: null pointers, a layer
    count or a layer width out of range, misalignment, a short workspace."""
    import numpy as np
    P = ctypes.c_void_p
    lib = mq.load_library()
    assert lib.macaq_linear_multi_workspace_bytes(16, 0, 512) == 0     # no layer
    assert lib.macaq_linear_multi_workspace_bytes(16, 129, 512) == 0   # more than 128 layers
    assert lib.macaq_linear_multi_workspace_bytes(16, 3, 48) == 0      # K % 32 != 0
    # per layer 128 padded rows of codes (K/2 bytes each) and scales (8 * ceil(K/256) bytes each)
    assert lib.macaq_linear_multi_workspace_bytes(16, 3, 512) >= 3 * 128 * (256 + 16)

    def widths(*n):
        a = np.array(n, dtype=np.int64)
        return a, P(a.ctypes.data)

    keep = []

    def call(N=(256, 128, 128), G=None, x=FAKE, am=FAKE, y=FAKE, M=16, K=512, wsb=1 << 30):
        a, ap = widths(*N)
        keep.append(a)
        return lib.macaq_w4a4_linear_multi(P(x), M, K, len(N) if G is None else G, P(am), P(FAKE), P(FAKE), ap,
                                           P(y), P(FAKE), wsb, None)

    assert lib.macaq_w4a4_linear_multi(P(FAKE), 16, 512, 3, P(FAKE), P(FAKE), P(FAKE), None, P(FAKE), P(FAKE),
                                       1 << 30, None) == -1          # no widths
    assert call(x=0) == -1 and call(y=0) == -1
    assert call(G=0) == -2 and call(N=(256, 100)) == -2 and call(N=(256, 0)) == -2
    assert call(M=0) == -2 and call(K=48) == -2
    assert call(x=MIS) == -3 and call(am=MIS) == -3
    assert call(wsb=1000) == -6
