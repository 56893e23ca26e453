"""The multi-GPU (replicas) path of bench.py on the CPU: two processes over gloo run the same
rank plumbing the GPU bench runs over NCCL -- barrier, max over ranks of the step time, the
whole-job value (every rank's work over the slowest rank's time) -- and the reference arm
prints only on rank 0."""
import io
import os
import socket
import sys
import contextlib

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import bench
    ranks = bench.Ranks.from_env("gloo")
    try:
        ranks.barrier()
        ms = 1.0 + rank  # rank r's step time: the slowest rank decides
        ms_max = ranks.max(ms)
        out[rank] = (ranks.world, ranks.rank, ms_max, bench.whole_job_tflops(ranks.world, 2e12, ms_max))
        ranks.barrier()
    finally:
        ranks.close()


def test_replicas_max_over_ranks_gloo():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r, (w, rank, ms_max, value) in res.items():
        assert (w, rank) == (2, r)
        assert ms_max == 2.0  # the max of 1.0 and 2.0, seen by both ranks
        assert value == pytest.approx(2 * 2e12 / 2e-3 / 1e12)  # 2000 TFLOP/s


def test_single_process_needs_no_process_group():
    import bench
    ranks = bench.Ranks(1, 0, 0, "gloo")
    ranks.barrier()
    assert ranks.max(3.5) == 3.5
    assert ranks.dist is None
    ranks.close()


def test_reference_arm_prints_only_on_rank_zero(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(None)  # rank 1 returns before touching its arguments
    assert buf.getvalue() == ""


def test_summary_and_mx_diff_on_fake_results():
    """The bench's end-of-line summary reads every leg's figures (a missing key would end a long
    GPU run without its line), and its code comparison counts mismatches and exempt ones."""
    import numpy as np

    import bench
    lr = {"frac": 0.6}
    leg = {"roofline": {"frac": 0.7}, "overhead": {"vs_plain_mxfp4_pct": 3.0, "vs_gemm_only_pct": 9.0}}
    out = {"value": 4000.0, "linear_roofline": lr, **leg,
           "secondary": {"flip_refinement": {"hessian_ms": 1.0, "refine_ms": 80.0, "held_out_rel_err_rtn": 0.062,
                                             "held_out_rel_err_refined": 0.056},
                         "llama3_8b_up_prefill": {"tflops": 4000.0, "linear_roofline": lr, **leg},
                         "qwen3_32b_up_decode_M1": {"gbs": 3600.0, "linear_roofline": lr, "vs_plain_mxfp4_pct": 2.0},
                         "qwen3_32b_stack": {"layers": 64, "M1": {"w4a4_ms": 6.5, "linear_roofline_frac": 0.4,
                                                                  "vs_plain_mxfp4_pct": 3.0,
                                                                  "w4a4_one_linear_at_a_time_ms": 7.0}},
                         "qwen3_moe_grouped": {"experts": 128, "up_T16": {"ms": 0.015, "linear_roofline_frac": 0.5,
                                                                          "vs_plain_mxfp4_pct": 3.0}}},
           "parity": {"ok": True, "activations": {"exempt": 0}, "weights": {"exempt": 0}, "y_rel_fro_vs_oracle": 1e-6}}
    sm = bench.summary(out)
    assert set(sm) == {"cfg4_down_prefill", "cfg2_llama_up", "cfg3_M1", "cfg5_M1", "moe_up_T16", "parity_cfg4",
                       "flip_llama_up"}
    codes = np.zeros((1, 16), np.uint8)  # one 32-element block
    codes[0, :2] = [0x21, 0x43]
    scales = np.array([[120]], np.uint8)
    V = np.zeros((1, 32), np.float32)
    V[0, :4] = [2.0 ** -8, 2.0 ** -7, 1.5 * 2.0 ** -7, 2.0 ** -6]
    same = bench._mx_diff(codes, scales, codes.copy(), scales.copy(), V)
    assert same == {"codes": 32, "code_mismatch": 0, "scales": 1, "scale_mismatch": 0, "exempt": 0}
    # element 1 differs; the oracle's value 2^-7 at scale 2^(120-127) is 1.0 on the E2M1 grid, not
    # near a rounding boundary, so the mismatch is not exempt
    other = codes.copy()
    other[0, 0] = 0x31
    diff = bench._mx_diff(other, scales, codes, scales, V)
    assert diff["code_mismatch"] == 1 and diff["exempt"] == 0
    # a value exactly on the 1.25 boundary (scaled) is exempt
    V[0, 1] = 1.25 * 2.0 ** -7
    assert bench._mx_diff(other, scales, codes, scales, V)["exempt"] == 1
