"""Shared pytest configuration: the ``gpu`` marker and import paths."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")


def pytest_terminal_summary(terminalreporter):
    """One line per config: the MXFP4 codes and scales the GPU parity tests compared with the
    oracle, their mismatches and how many of those were exempt (within 1 fp32 ulp of a
    rounding boundary).  Only the GPU tests record comparisons."""
    gpu_util = sys.modules.get("tests.gpu_util")
    log = getattr(gpu_util, "PARITY_LOG", None)
    if not log:
        return
    terminalreporter.write_line("MXFP4 parity vs oracle (codes / scales compared: mismatches, exempt):")
    for label in sorted(log):
        t = log[label]
        terminalreporter.write_line(
            f"  {label}: {t['codes']} codes {t['code_mismatch']} mismatched, {t['scales']} scales "
            f"{t['scale_mismatch']} mismatched, {t['exempt']} exempt")
