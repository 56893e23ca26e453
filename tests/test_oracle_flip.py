"""Pins of the oracle's Flip-Refinement (CPU, no GPU): the Hessian against a plain matrix product,
hand-derived worked cases, and properties that hold for any greedy descent of this objective,
checked against an objective written here from its definition (not the oracle's incremental
arithmetic).

"MACaQ ...", Abstract: Flip-Refinement refines the round-to-nearest codes by a greedy,
Hessian-weighted coordinate descent over single-code steps to neighbouring grid values.  Reading (oracle/macaq_oracle.c): per weight row the objective is
L = (q - v) Hs (q - v)^T with Hs = Xt^T Xt of the transformed calibration activations; block
scales are kept; each step applies the single most-improving one-step move on the ordered E2M1
value line; ties go to the smaller k, then the downward move."""
import itertools

import numpy as np
import pytest

import oracle

LINE = np.array([-6, -4, -3, -2, -1.5, -1, -0.5, 0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
MAG = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def decode(codes, scales):
    """Values of MXFP4 codes [N][K/2] (even k low nibble) with E8M0 scales [N][K/32]."""
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(codes.shape[0], -1)
    val = np.where(nib & 8, -MAG[nib & 7], MAG[nib & 7])
    return val * np.exp2(np.repeat(scales.astype(np.float64), 32, axis=1) - 127)


def objective(codes, scales, V, Hs):
    r = decode(codes, scales) - V.astype(np.float64)
    return np.einsum("nk,kj,nj->n", r, Hs, r)


def pack(nibbles):
    nibbles = np.asarray(nibbles, np.uint8).reshape(1, -1)
    return (nibbles[:, 0::2] | (nibbles[:, 1::2] << 4)).astype(np.uint8)


def test_hessian_is_the_gram_matrix():
    rng = np.random.default_rng(1)
    Xt = (rng.standard_normal((48, 96)) * rng.uniform(0.1, 5, 96)).astype(np.float32)
    Hs = oracle.hessian_of(Xt)
    ref = Xt.astype(np.float64).T @ Xt.astype(np.float64)
    assert np.max(np.abs(Hs - ref)) <= 1e-12 * np.max(np.abs(ref))
    assert np.array_equal(Hs, Hs.T)  # bitwise symmetric: fma(a, b, c) == fma(b, a, c)
    one = np.zeros((1, 64), np.float32)
    one[0, 5], one[0, 40] = 3.0, -0.5
    assert np.array_equal(oracle.hessian_of(one), np.outer(one[0], one[0]).astype(np.float64))


def _two_coupled(v0, v1, rho, K=32):
    V = np.zeros((1, K), np.float32)
    V[0, 0], V[0, 1] = v0, v1
    Hs = np.zeros((K, K))
    Hs[0, 0] = Hs[1, 1] = 1.0
    Hs[0, 1] = Hs[1, 0] = rho
    return V, Hs


def test_worked_case_one_move_up():
    """Scale byte 127 (unit 1), targets 1.2 and 1.2, RTN codes 1.0 (0x2) with residuals -0.2 each,
    Hs = [[1, .9], [.9, 1]] on those two channels.  g = Hs r = (-0.38, -0.38).  Moving channel 0
    to 1.5 changes L by 0.5 (0.5 - 0.76) = -0.13 (channel 1 ties; the smaller k wins); afterwards
    g = (0.12, 0.07) and every move raises L (by 0.37, 0.13, 0.32, 0.18): one move, L 0.152 ->
    0.022."""
    V, Hs = _two_coupled(1.2, 1.2, 0.9)
    codes = pack([2, 2] + [0] * 30)
    scales = np.full((1, 1), 127, np.uint8)
    out, moves = oracle.flip_refine_codes(V, codes, scales, Hs, 100)
    assert moves.tolist() == [1]
    assert out.tolist() == pack([3, 2] + [0] * 30).tolist()
    assert objective(codes, scales, V, Hs)[0] == pytest.approx(0.152, abs=1e-6)
    assert objective(out, scales, V, Hs)[0] == pytest.approx(0.022, abs=1e-6)


def test_worked_case_move_to_zero_keeps_the_sign_bit():
    """Targets -0.3 and 0.35 (RTN -0.5 = 0x9 and 0.5 = 0x1), Hs = [[1, -.9], [-.9, 1]]:
    g = (-0.335, 0.33); channel 0 up to zero lowers L by 0.085, channel 1 down by 0.08, so channel 0
    moves, and its code becomes 0x8 (the negative zero: the sign bit is kept).  Then every move
    raises L."""
    V, Hs = _two_coupled(-0.3, 0.35, -0.9)
    codes = pack([9, 1] + [0] * 30)
    scales = np.full((1, 1), 127, np.uint8)
    out, moves = oracle.flip_refine_codes(V, codes, scales, Hs, 100)
    assert moves.tolist() == [1]
    assert out.tolist() == pack([8, 1] + [0] * 30).tolist()


def test_exact_tie_goes_to_the_smaller_index():
    """Two identical, uncoupled copies of the first worked case (channels 0, 1 and 2, 3): the
    first move has the same dL bit for bit at channels 0 and 2 and goes to channel 0; the second
    goes to channel 2."""
    K = 32
    V = np.zeros((1, K), np.float32)
    V[0, :4] = 1.2
    Hs = np.zeros((K, K))
    for a in (0, 2):
        Hs[a, a] = Hs[a + 1, a + 1] = 1.0
        Hs[a, a + 1] = Hs[a + 1, a] = 0.9
    codes = pack([2] * 4 + [0] * 28)
    scales = np.full((1, 1), 127, np.uint8)
    first, m1 = oracle.flip_refine_codes(V, codes, scales, Hs, 1)
    assert m1.tolist() == [1] and first.tolist() == pack([3, 2, 2, 2] + [0] * 28).tolist()
    out, m = oracle.flip_refine_codes(V, codes, scales, Hs, 100)
    assert m.tolist() == [2] and out.tolist() == pack([3, 2, 3, 2] + [0] * 28).tolist()


def test_diagonal_hessian_keeps_round_to_nearest():
    """With Hs diagonal the objective separates per code and the nearest value is optimal, so no
    move lowers it (ties at a midpoint change L by exactly zero): zero moves."""
    rng = np.random.default_rng(2)
    V = (rng.standard_normal((6, 128)) * 0.03).astype(np.float32)
    codes, scales = oracle.quantize_mx(V)
    Hs = np.diag(rng.uniform(0.5, 2.0, 128))
    out, moves = oracle.flip_refine_codes(V, codes, scales, Hs, 1000)
    assert moves.tolist() == [0] * 6
    assert np.array_equal(out, codes)


def _random_layer(seed, N=8, K=128, C=40):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    s = rng.uniform(0.3, 3.0, K).astype(np.float32)
    xcal = rng.standard_normal((C, K)).astype(np.float32)
    xcal[:, rng.choice(K, 3, replace=False)] *= 20.0
    a, w = oracle.multipliers(s)
    V = oracle.transform_f32(W, w)
    codes, scales = oracle.quantize_mx(V)
    Hs = oracle.calib_hessian(xcal, a)
    return V, codes, scales, Hs


def test_refinement_lowers_the_objective_and_ends_in_a_local_minimum():
    V, codes, scales, Hs = _random_layer(3)
    out, moves = oracle.flip_refine_codes(V, codes, scales, Hs, 10_000)
    L0 = objective(codes, scales, V, Hs)
    L1 = objective(out, scales, V, Hs)
    assert np.all(L1 <= L0) and np.any(L1 < L0) and moves.sum() > 0
    # codes stay MXFP4 codes with the same scales; only code nibbles changed
    assert out.dtype == np.uint8 and out.shape == codes.shape
    # local minimum: no single one-step move lowers the objective (brute force, from the definition)
    N, K = V.shape
    nib = np.stack([out & 15, out >> 4], -1).reshape(N, -1)
    for n in range(N):
        base = L1[n]
        for k in range(K):
            m, sgn = int(nib[n, k] & 7), int(nib[n, k] >> 3)
            p = 7 - m if sgn else 7 + m
            for q in (p - 1, p + 1):
                if 0 <= q <= 14:
                    trial = nib[n].copy()
                    trial[k] = (sgn << 3) if LINE[q] == 0 else (q - 7 if LINE[q] > 0 else 8 | (7 - q))
                    L = objective(pack(trial), scales[n:n + 1], V[n:n + 1], Hs)[0]
                    assert L >= base - 1e-9 * abs(base), (n, k, q)


def test_move_budget_is_a_prefix_of_the_descent():
    V, codes, scales, Hs = _random_layer(4)
    full, m_full = oracle.flip_refine_codes(V, codes, scales, Hs, 10_000)
    two, m_two = oracle.flip_refine_codes(V, codes, scales, Hs, 2)
    assert np.all(m_two == np.minimum(m_full, 2))
    L0, L2, Lf = (objective(c, scales, V, Hs) for c in (codes, two, full))
    assert np.all(L2 <= L0) and np.all(Lf <= L2)
    changed = (np.stack([two & 15, two >> 4], -1) != np.stack([codes & 15, codes >> 4], -1)).reshape(len(V), -1)
    assert np.all(changed.sum(1) <= 2)


def test_brute_force_on_three_coupled_codes():
    """Hs supported on channels 3, 10 and 17 of one block (a random positive definite 3 x 3): all
    15^3 value combinations of those three codes give the global optimum L*; the greedy result
    lies between L* and round-to-nearest, moves only those three codes, and is a local minimum."""
    rng = np.random.default_rng(5)
    K, idx = 32, [3, 10, 17]
    A = rng.standard_normal((3, 3))
    Hs = np.zeros((K, K))
    Hs[np.ix_(idx, idx)] = A @ A.T + 0.05 * np.eye(3)
    V = (rng.standard_normal((1, K)) * 1.5).astype(np.float32)
    codes, scales = oracle.quantize_mx(V)
    out, _ = oracle.flip_refine_codes(V, codes, scales, Hs, 1000)
    nib0 = np.stack([codes & 15, codes >> 4], -1).reshape(-1)
    nib1 = np.stack([out & 15, out >> 4], -1).reshape(-1)
    others = np.setdiff1d(np.arange(K), idx)
    assert np.array_equal(nib0[others], nib1[others])
    unit = np.exp2(float(scales[0, 0]) - 127)
    v = V[0, idx].astype(np.float64)
    Hsub = Hs[np.ix_(idx, idx)]
    best = min(((np.array(c) * unit - v) @ Hsub @ (np.array(c) * unit - v))
               for c in itertools.product(LINE, repeat=3))
    Lg, L0 = objective(out, scales, V, Hs)[0], objective(codes, scales, V, Hs)[0]
    assert best - 1e-12 <= Lg <= L0
