"""Pins for the CPU oracle: each check ties it to something other than itself.

Method: "MACaQ: Fast, Model Agnostic Calibrated Quantization for Low-Precision Weights and
Activations", Abstract -- per-channel scale and block-Hadamard applied online to the
activations, inverse transforms absorbed into the weights, MXFP4 W4A4 with round-to-nearest
weights.  MX format: OCP Microscaling v1.0 (E2M1 elements, one E8M0 scale per 32).

A plausible slip anywhere in the oracle fails at least one test here:
  * wrong butterfly index/sign/order        -> Sylvester matrix, involution, explicit matmul
  * wrong scale direction or normalisation  -> fold identity (fp64 and fp32)
  * wrong E8M0 rule (floor vs ceil, bias)   -> exponent closed forms, [4, 8) range
  * wrong rounding (ties, saturation, sign) -> threshold table, brute force, sign cases
  * wrong nibble order or scale indexing    -> hand-derived golden block, pack test
  * wrong GEMM decode or transposition      -> exact contraction of independent decode
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
C = 1.0 / math.sqrt(32.0)
E2M1_SET = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)  # OCP MX v1.0 FP4 E2M1 magnitudes


def sylvester(n=32):
    """H[i][j] = (-1)^popcount(i & j), built from its closed form."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    return np.where(pc % 2 == 0, 1.0, -1.0)


# ----------------------------------------------------------------------------- Hadamard


def test_hadamard_matches_sylvester_matrix():
    H = sylvester()
    assert np.array_equal(H @ H.T, 32 * np.eye(32))
    # transform of each unit vector (mult = 1) is the corresponding column of H
    X = np.eye(32, dtype=np.float32)
    V = oracle.transform_f32(X, np.ones(32, np.float32))
    assert np.array_equal(V, H.T.astype(np.float32))  # row j of V = H e_j = column j


def test_hadamard_is_involution_up_to_32():
    rng = np.random.default_rng(1)
    u = rng.integers(-8, 9, size=(16, 96)).astype(np.float32)  # exact in fp32 throughout
    one = np.ones(96, np.float32)
    v = oracle.transform_f32(oracle.transform_f32(u, one), one)
    assert np.array_equal(v, 32 * u)


def test_butterfly_equals_explicit_product_and_parseval():
    rng = np.random.default_rng(2)
    u = rng.standard_normal((8, 128))
    H = sylvester()
    v = oracle.transform_f64(u, np.ones(128))
    ref = np.concatenate([u[:, 32 * b:32 * b + 32] @ H.T for b in range(4)], axis=1)
    assert np.max(np.abs(v - ref)) <= 1e-13 * np.max(np.abs(ref))
    blocks_u = u.reshape(8, 4, 32)
    blocks_v = v.reshape(8, 4, 32)
    np.testing.assert_allclose((blocks_v ** 2).sum(-1), 32 * (blocks_u ** 2).sum(-1), rtol=1e-13)


def test_fp32_transform_within_rounding_bound_of_fp64():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 256)).astype(np.float32)
    mult = rng.uniform(0.01, 2.0, 256).astype(np.float32)
    v32 = oracle.transform_f32(x, mult).astype(np.float64)
    v64 = oracle.transform_f64(x.astype(np.float64), mult.astype(np.float64))
    # 1 rounding for the scale + 5 butterfly stages, each at most 2^-24 relative to a
    # partial sum bounded by sum_j |u_j| of the block
    absu = np.abs(x.astype(np.float64) * mult).reshape(64, 8, 32).sum(-1)
    bound = 6 * 2.0 ** -24 * np.repeat(absu, 32, axis=1) * 1.0001
    assert np.all(np.abs(v32 - v64) <= bound)


# ------------------------------------------------------------------------- multipliers


def test_multipliers_closed_forms():
    s = np.array([1.0, 2.0, 0.25, 2.0 ** 20, 3.0, 0.7], np.float32)
    a, w = oracle.multipliers(s)
    base = np.float32(C)  # fl32(1/sqrt(32))
    # powers of two scale exactly
    assert a[0] == base and w[0] == base
    assert a[1] == base / 2 and w[1] == base * 2
    assert a[2] == base * 4 and w[2] == base / 4
    assert a[3] == np.float32(base * 2.0 ** -20) and w[3] == np.float32(base * 2.0 ** 20)
    # product a * w is c^2 = 1/32 to within two fp32 roundings
    prod = a.astype(np.float64) * w.astype(np.float64)
    assert np.all(np.abs(prod * 32 - 1) <= 2 * 2.0 ** -24 + 1e-15)
    # a_k * s_k * sqrt(32) == 1 within one fp32 rounding
    assert np.all(np.abs(a.astype(np.float64) * s * math.sqrt(32) - 1) <= 2.0 ** -24 + 1e-15)


# ----------------------------------------------------------------------- fold identity


@pytest.mark.parametrize("M,K,N", [(16, 256, 128), (5, 64, 7), (3, 32 * 37, 11)])
def test_fold_identity_fp64(M, K, N):
    """(x diag(c/s) H)(W diag(c s) H)^T == x W^T with no rounding (Abstract: the inverse
    transforms absorbed into the weights cancel the online ones)."""
    rng = np.random.default_rng(M * 1000 + K)
    x = rng.standard_normal((M, K))
    W = rng.standard_normal((N, K)) * 0.02
    s = rng.uniform(0.05, 20.0, K)
    Ap = oracle.transform_f64(x, C / s)
    Wp = oracle.transform_f64(W, C * s)
    ref = x @ W.T
    err = np.linalg.norm(Ap @ Wp.T - ref) / np.linalg.norm(ref)
    assert err <= 1e-12
    # the opposite scale direction does not reproduce it
    bad = oracle.transform_f64(x, C * s) @ Wp.T
    assert np.linalg.norm(bad - ref) / np.linalg.norm(ref) > 1e-2


def test_fold_identity_fp32_multipliers():
    import workloads
    wl = workloads.TINY
    x = workloads.make_x(wl).float().numpy()
    W = workloads.make_w(wl).numpy()
    s = workloads.make_s(wl, workloads.make_w(wl)).numpy()
    a, w = oracle.multipliers(s)
    Ap = oracle.transform_f32(x, a).astype(np.float64)
    Wp = oracle.transform_f32(W, w).astype(np.float64)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    err = np.linalg.norm(Ap @ Wp.T - ref) / np.linalg.norm(ref)
    assert err <= 1e-5


# ------------------------------------------------------------------------------ E8M0


def test_e8m0_closed_forms():
    f = oracle.e8m0_from_amax
    assert f(0.0) == 0
    assert f(1.0) == 125  # floor(log2 1) - 2 + 127
    assert f(4.0) == 127
    assert f(7.999) == 127
    assert f(8.0) == 128
    assert f(0.17677669) == 122
    assert f(np.float32(2.0 ** -126)) == 0  # E = 1 -> clamped
    assert f(np.float32(2.0 ** -125)) == 0  # E = 2 -> clamped
    assert f(np.float32(2.0 ** -124)) == 1  # E = 3
    assert f(np.float32(1e-40)) == 0  # subnormal
    assert f(np.finfo(np.float32).max) == 252


def test_e8m0_puts_block_max_in_4_to_8():
    rng = np.random.default_rng(4)
    for amax in np.exp(rng.uniform(-80, 80, 2000)).astype(np.float32):
        e = oracle.e8m0_from_amax(amax)
        q = float(amax) * 2.0 ** (127 - e)
        assert 4.0 <= q < 8.0


# ------------------------------------------------------------------------------ E2M1


def threshold_index(t):
    """Hand-derived boundaries of round-half-to-even-code onto E2M1, saturating at 6:
    ties at .25 -> 0 (even), .75 -> 1.0 (code 2), 1.25 -> 1.0, 1.75 -> 2.0, 2.5 -> 2,
    3.5 -> 4, 5 -> 4."""
    t = np.asarray(t, np.float64)
    return ((t > 0.25).astype(int) + (t >= 0.75) + (t > 1.25) + (t >= 1.75)
            + (t > 2.5) + (t >= 3.5) + (t > 5.0))


def brute_force_index(t):
    """Nearest E2M1 magnitude by exhaustive search; among equidistant ones the even code."""
    ds = [abs(t - m) for m in E2M1_SET]
    dmin = min(ds)
    ties = [i for i, d in enumerate(ds) if d == dmin]
    even = [i for i in ties if i % 2 == 0]
    return even[0] if even else ties[0]


def test_e2m1_scalar_against_threshold_table_and_brute_force():
    pts = [0.0, 0.1, 0.25, 0.2500001, 0.5, 0.74999, 0.75, 1.0, 1.25, 1.2500001, 1.5, 1.75,
           1.7499999, 2.0, 2.5, 2.5000002, 3.0, 3.5, 3.4999998, 4.0, 5.0, 5.0000005, 6.0, 7.9, 100.0]
    for t in pts:
        assert oracle.e2m1_index(t) == threshold_index(t) == brute_force_index(t), t


def _quantize_values_at_unit_scale(t):
    """Quantise values t (fp32, |t| < 8) under scale byte 127 (X = 1): each row holds one
    anchor 4.0 (amax in [4, 8) fixes e = 127) followed by 31 test values."""
    t = np.asarray(t, np.float32)
    n = t.size
    rows = -(-n // 31)
    V = np.zeros((rows, 32), np.float32)
    V[:, 0] = 4.0
    flat = np.zeros(rows * 31, np.float32)
    flat[:n] = t
    V[:, 1:] = flat.reshape(rows, 31)
    codes, scales = oracle.quantize_mx(V)
    assert np.all(scales == 127)
    nib = np.empty((rows, 32), np.uint8)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    return nib[:, 1:].reshape(-1)[:n]


def test_e2m1_exhaustive_over_threshold_binades():
    # every fp32 value in [0.25, 8): the binades holding all rounding boundaries
    lo = np.float32(0.25).view(np.uint32)
    hi = np.float32(8.0).view(np.uint32)
    t = np.arange(lo, hi, dtype=np.uint32).view(np.float32)
    got = _quantize_values_at_unit_scale(t)
    assert np.array_equal(got & 7, threshold_index(t))
    assert np.all(got >> 3 == 0)
    # and their negatives carry the sign bit only
    got_neg = _quantize_values_at_unit_scale(-t[::97])
    assert np.array_equal(got_neg, (threshold_index(t[::97]) | 8).astype(np.uint8))


def test_e2m1_brute_force_fine_grid_with_ties():
    grid = np.concatenate([np.linspace(0, 7.99, 4001),
                           np.array(E2M1_SET[1:]) - 0.0, [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]])
    grid = grid.astype(np.float32)
    ulp_up = np.nextafter(grid, np.float32(np.inf))
    ulp_dn = np.nextafter(grid, np.float32(0))
    t = np.concatenate([grid, ulp_up, ulp_dn])
    got = _quantize_values_at_unit_scale(t) & 7
    ref = np.array([brute_force_index(float(v)) for v in t])
    assert np.array_equal(got, ref)


def test_e2m1_codes_lie_in_representable_set():
    rng = np.random.default_rng(5)
    V = (rng.standard_t(3, (300, 256)) * 10 ** rng.uniform(-3, 3, (300, 1))).astype(np.float32)
    codes, scales = oracle.quantize_mx(V)
    dec = oracle.mx_decode(codes, scales)
    X = 2.0 ** (np.repeat(scales.astype(np.float64), 32, axis=1) - 127)
    mags = np.abs(dec / X)
    assert np.all(np.isin(mags, E2M1_SET))
    # each block's amax quantises to 4 or 6 (amax / X in [4, 8))
    amax_q = mags.reshape(300, 8, 32).max(-1)
    assert np.all(np.isin(amax_q, (4.0, 6.0)))


def test_sign_of_zero_and_pack_order():
    assert oracle.e2m1_code(-0.0, 127) == 0x8
    assert oracle.e2m1_code(0.0, 127) == 0x0
    assert oracle.e2m1_code(-0.1, 127) == 0x8
    assert oracle.e2m1_code(-6.5, 127) == 0xF
    V = np.zeros((1, 32), np.float32)
    V[0, :8] = [4.0, 0.5, -1.0, 1.5, 2.0, -3.0, 6.0, -0.25]
    codes, scales = oracle.quantize_mx(V)
    assert scales[0, 0] == 127
    # element 2j in the low nibble
    assert list(codes[0, :4]) == [0x16, 0x3A, 0xD4, 0x87]


# ------------------------------------------------------------------ worked example / golden


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def test_golden_onehot_block():
    g = _read_golden("onehot_block_j5.txt")
    x = np.zeros((1, 32), np.float32)
    x[0, 5] = 1.0
    a, _ = oracle.multipliers(np.ones(32, np.float32))
    codes, scales = oracle.act_transform_quant(x, a)
    assert scales[0, 0] == int(g["scale"][0])
    assert [f"{b:02X}" for b in codes[0]] == g["codes"]


@pytest.mark.parametrize("j", range(32))
def test_onehot_closed_form_every_position(j):
    x = np.zeros((1, 64), np.float32)
    x[0, 32 + j] = 1.0  # second block; first block all zero
    a, _ = oracle.multipliers(np.ones(64, np.float32))
    codes, scales = oracle.act_transform_quant(x, a)
    assert scales[0, 0] == 0 and np.all(codes[0, :16] == 0)  # zero block: e = 0, +0 codes
    assert scales[0, 1] == 122
    H = sylvester()
    expect = np.where(H[:, j] > 0, 0x7, 0xF)
    got = np.empty(32, int)
    got[0::2] = codes[0, 16:] & 0xF
    got[1::2] = codes[0, 16:] >> 4
    assert np.array_equal(got, expect)


# ----------------------------------------------------------------------- invariants


def _tiny_inputs(seed=6, M=24, K=320):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, 7] *= 40
    a = rng.uniform(0.02, 0.5, K).astype(np.float32)
    return x, a


def test_power_of_two_scaling_shifts_only_the_scale():
    x, a = _tiny_inputs()
    c0, s0 = oracle.act_transform_quant(x, a)
    for j in (-5, 3, 11):
        c1, s1 = oracle.act_transform_quant(x * np.float32(2.0 ** j), a)
        assert np.array_equal(c0, c1)
        assert np.array_equal(s1.astype(int), s0.astype(int) + j)


def test_negation_flips_only_sign_bits():
    x, a = _tiny_inputs(7)
    c0, s0 = oracle.act_transform_quant(x, a)
    c1, s1 = oracle.act_transform_quant(-x, a)
    assert np.array_equal(s0, s1)
    assert np.array_equal(c1, c0 ^ 0x88)


def test_block_permutation_permutes_outputs():
    x, a = _tiny_inputs(8)
    nb = x.shape[1] // 32
    perm = np.random.default_rng(9).permutation(nb)
    cols = np.concatenate([np.arange(32 * b, 32 * b + 32) for b in perm])
    c0, s0 = oracle.act_transform_quant(x, a)
    c1, s1 = oracle.act_transform_quant(x[:, cols], a[cols])
    ccols = np.concatenate([np.arange(16 * b, 16 * b + 16) for b in perm])
    assert np.array_equal(c1, c0[:, ccols])
    assert np.array_equal(s1, s0[:, perm])


def test_fold_equals_transform_of_weights_with_weight_multiplier():
    rng = np.random.default_rng(10)
    W = (rng.standard_normal((40, 128)) * 0.02).astype(np.float32)
    s = rng.uniform(0.1, 10, 128).astype(np.float32)
    codes, scales, act_mult = oracle.fold_weights(W, s)
    a, w = oracle.multipliers(s)
    assert np.array_equal(act_mult, a)
    c2, s2 = oracle.quantize_mx(oracle.transform_f32(W, w))
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)


# ------------------------------------------------------------------------------ GEMM


def independent_decode(codes, scales):
    """Decode from the E2M1 value set and 2^(e-127), written independently of the oracle."""
    R, K2 = codes.shape
    nib = np.empty((R, 2 * K2), np.int64)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    mag = np.array(E2M1_SET)[nib & 7]
    val = np.where(nib & 8, -mag, mag)
    return val * np.exp2(np.repeat(scales.astype(np.float64), 32, axis=1) - 127)


def test_decode_matches_independent_decode():
    rng = np.random.default_rng(11)
    codes = rng.integers(0, 256, (13, 48), dtype=np.uint8)
    scales = rng.integers(100, 150, (13, 3), dtype=np.uint8)
    assert np.array_equal(oracle.mx_decode(codes, scales), independent_decode(codes, scales))


def test_gemm_is_exact_contraction():
    rng = np.random.default_rng(12)
    M, N, K = 9, 21, 320
    Aq = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    As = rng.integers(110, 140, (M, K // 32), dtype=np.uint8)
    Wq = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    Ws = rng.integers(110, 140, (N, K // 32), dtype=np.uint8)
    ref = independent_decode(Aq, As) @ independent_decode(Wq, Ws).T
    y = oracle.mx_gemm(Aq, As, Wq, Ws)
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
    rows = np.array([8, 0, 3])
    np.testing.assert_array_equal(oracle.mx_gemm(Aq, As, Wq, Ws, rows), y[rows])


def test_gemm_closed_form_all_ones():
    # every element 1.0 (code 2) at scale 127: y = K exactly; a transposed or mis-scaled
    # contraction would not give the per-row factors below
    M, N, K = 3, 5, 96
    Aq = np.full((M, K // 2), 0x22, np.uint8)
    As = np.full((M, K // 32), 127, np.uint8)
    As[1] = 128  # row 1 doubled
    Wq = np.full((N, K // 2), 0x22, np.uint8)
    Ws = np.full((N, K // 32), 127, np.uint8)
    Ws[4] = 125  # column 4 quartered
    y = oracle.mx_gemm(Aq, As, Wq, Ws)
    expect = np.full((M, N), float(K))
    expect[1] *= 2
    expect[:, 4] /= 4
    assert np.array_equal(y, expect)


def test_end_to_end_quantisation_error_is_reported():
    """Parity unpinned: the pages give no bound on W4A4 error; only sanity is checked."""
    import workloads
    wl = workloads.TINY
    x = workloads.make_x(wl).float().numpy()
    W = workloads.make_w(wl).numpy()
    s = workloads.make_s(wl, workloads.make_w(wl)).numpy()
    Wq, Ws, a = oracle.fold_weights(W, s)
    Aq, As = oracle.act_transform_quant(x, a)
    y = oracle.mx_gemm(Aq, As, Wq, Ws)
    ref = x.astype(np.float64) @ W.astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel < 0.5  # W4A4 on a 256-wide dot product: a few percent is typical
    print(f"tiny: W4A4 relative Frobenius error vs fp64 x W^T = {rel:.4f}")


# ---- calibration of the per-channel scale (the step before the fold) ----

def test_calibrate_scale_hand_values():
    # column maxima (ignoring sign) 4/1, 1/4, 9/1, 3/3, and zero columns -> 1
    xcal = np.array([[4.0, -1.0, 9.0, 3.0, 0.0, 2.0],
                     [-2.0, 0.5, 1.0, -3.0, 0.0, 1.0]], np.float32)
    W = np.array([[1.0, 4.0, -1.0, 3.0, 5.0, 0.0],
                  [-0.5, -2.0, 0.25, 1.0, 1.0, 0.0]], np.float32)
    s = oracle.calibrate_scale(xcal, W)
    assert s.tolist() == [2.0, 0.5, 3.0, 1.0, 1.0, 1.0]


def test_calibrate_scale_power_of_two_and_sign_invariance():
    rng = np.random.default_rng(3)
    xcal = (rng.standard_normal((64, 96)) * 3).astype(np.float32)
    W = (rng.standard_normal((40, 96)) * 0.02).astype(np.float32)
    s = oracle.calibrate_scale(xcal, W)
    # W x 4 halves s exactly, x x 4 doubles it; signs do not matter
    assert np.array_equal(oracle.calibrate_scale(xcal, W * 4), s / 2)
    assert np.array_equal(oracle.calibrate_scale(xcal * 4, W), s * 2)
    assert np.array_equal(oracle.calibrate_scale(-xcal, -W), s)
    # permuting channels permutes s
    perm = rng.permutation(96)
    assert np.array_equal(oracle.calibrate_scale(xcal[:, perm], W[:, perm]), s[perm])


def test_calibrate_scale_balances_activation_and_weight_ranges():
    # the purpose of the rule: after scaling, each channel's activation range max|x/s| and
    # weight range max|W s| coincide (up to rounding s to fp32)
    rng = np.random.default_rng(4)
    xcal = (rng.standard_normal((64, 128)) * rng.uniform(0.1, 50, 128)).astype(np.float32)
    W = (rng.standard_normal((200, 128)) * rng.uniform(0.001, 0.1, 128)).astype(np.float32)
    s = oracle.calibrate_scale(xcal, W).astype(np.float64)
    xr = np.abs(xcal.astype(np.float64)).max(0) / s
    wr = np.abs(W.astype(np.float64)).max(0) * s
    np.testing.assert_allclose(xr, wr, rtol=2.0 ** -22)
