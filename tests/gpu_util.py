"""Helpers of the GPU parity tests: comparison of codes/scales with the 1-ulp exemption,
relative Frobenius errors, bf16 rounding of fp64 references."""
import numpy as np
import torch

from tests import layout

# Rounding boundaries of |v| / 2^(e-127) on the E2M1 grid (midpoints between magnitudes).
E2M1_BOUNDARIES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def unpack_nibbles(codes: np.ndarray) -> np.ndarray:
    out = np.empty(codes.shape[:-1] + (2 * codes.shape[-1],), np.uint8)
    out[..., 0::2] = codes & 0xF
    out[..., 1::2] = codes >> 4
    return out


def _near_power_of_two(a: np.ndarray) -> np.ndarray:
    """amax within 1 fp32 ulp of a change of binade."""
    a = a.astype(np.float32)
    up = np.nextafter(a, np.float32(np.inf))
    dn = np.nextafter(a, np.float32(0))
    ex = lambda v: (v.view(np.uint32) >> 23) & 0xFF
    return (ex(up) != ex(a)) | (ex(dn) != ex(a))


def _near_code_boundary(v: np.ndarray, e: np.ndarray) -> np.ndarray:
    """|v| within 1 fp32 ulp of a rounding boundary times 2^(e-127)."""
    a = np.abs(v.astype(np.float32))
    lo = np.nextafter(a, np.float32(0)).astype(np.float64)
    hi = np.nextafter(a, np.float32(np.inf)).astype(np.float64)
    scale = np.exp2(e.astype(np.float64) - 127)
    res = np.zeros(a.shape, bool)
    for t in E2M1_BOUNDARIES:
        b = t * scale
        res |= (lo <= b) & (b <= hi)
    return res


# Comparisons of codes and scales made in this test session, per label (the config they cover):
# printed at the end of the run by the terminal-summary hook in tests/conftest.py, so the
# counts of exempt near-boundary mismatches appear in the run's log.
PARITY_LOG: dict = {}


def config_label(wl, what: str) -> str:
    """Label of a comparison: the workload's config number and what was compared."""
    return f"config {wl.config} {what}"


def _record(label, stats):
    if label is None:
        return
    tot = PARITY_LOG.setdefault(label, {"codes": 0, "scales": 0, "code_mismatch": 0, "scale_mismatch": 0,
                                        "exempt": 0})
    for k in tot:
        tot[k] += stats[k]


def compare_mx(gpu_codes, gpu_scales_tiled, ref_codes, ref_scales, rows, K, V=None, label=None):
    """Bit-exact comparison of MXFP4 codes and E8M0 scales.  Mismatches are allowed only
    where the fp32 pre-rounding value (oracle V) lies within 1 ulp of a rounding boundary
    (or the block max within 1 ulp of a power of two); those are counted and returned, and
    recorded under `label` for the session summary.  V may be a callable that returns it
    (computed only when there is a mismatch)."""
    gs = layout.tiled_to_rowmajor(gpu_scales_tiled, rows, K)
    pad = layout.padded_block_bytes(gpu_scales_tiled, rows, K)
    assert np.all(pad == 0), "padded scale blocks of real rows must be zero"
    bad_s = gs != ref_scales
    gn = unpack_nibbles(gpu_codes)
    rn = unpack_nibbles(ref_codes)
    bad_c = gn != rn
    stats = {"codes": int(bad_c.size), "scales": int(bad_s.size), "code_mismatch": int(bad_c.sum()),
             "scale_mismatch": int(bad_s.sum()), "exempt": 0}
    if not bad_c.any() and not bad_s.any():
        _record(label, stats)
        return stats
    if callable(V):
        V = V()
    assert V is not None, f"mismatches without oracle values: {stats}"
    Vb = V.reshape(rows, K // 32, 32)
    amax = np.abs(Vb).max(-1)
    ok_s = ~bad_s | _near_power_of_two(amax)
    e_full = np.repeat(ref_scales, 32, axis=1)
    ok_c = ~bad_c | _near_code_boundary(V, e_full) | np.repeat(bad_s & ok_s, 32, axis=1)
    stats["exempt"] = int((bad_c & ok_c).sum() + (bad_s & ok_s).sum())
    assert ok_s.all() and ok_c.all(), f"non-exempt mismatches: {stats}"
    _record(label, stats)
    return stats


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def bf16_round(y64: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (RN) -> bf16 (RNE), back to fp64 (the rounding the epilogue performs,
    applied to the exact result)."""
    t = torch.from_numpy(np.asarray(y64, np.float64)).to(torch.float32).to(torch.bfloat16)
    return t.to(torch.float64).numpy()
