"""Pins for the CPU oracle: each checks it against something other than itself.

  * SVD closed form: for X0 = U diag(sigma) V^T the matrix iteration equals
    U p(sigma) V^T with p the scalar polynomial iterated on each singular value
    (a theorem about odd matrix polynomials; SVD from numpy.linalg).
  * Exact rational orbits: on a diagonal matrix the iteration must reproduce
    the scalar orbit computed with fractions.Fraction (no floating point).
  * Cubic (1.5, -0.5, 0) converges to the polar factor U V^T.
  * Hand-unrolled three-step recurrences for both momenta and the EMA.
  * Invariants: transpose, gradient scale, permutations, G = 0, rank one.
  * The page constants in tests/golden/pages_constants.json.
  * bf16 rounding against torch's float32 -> bfloat16 conversion.
  * Whole-step closed forms: rank one (Muon), diagonal matrices (SGD form,
    with and without Nesterov), tall rank one with zero rows (ANVIL).
  * The flop count against a count of a small case's multiply-adds.
  * Sensitivity: plausible mistakes (wrong sign, dropped term, transposed
    Gram) make the closed-form pin fail; test_oracle_mutants plants one-line
    mistakes in every function and names the pin that catches each.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)


def _random_svd(rows, cols, sigmas, seed):
    rng = np.random.default_rng(seed)
    r = min(rows, cols)
    U, _ = np.linalg.qr(rng.standard_normal((rows, r)))
    V, _ = np.linalg.qr(rng.standard_normal((cols, r)))
    return U, np.asarray(sigmas, dtype=np.float64), V


def _scalar_orbit(sig, coeffs):
    s = np.array(sig, dtype=np.float64)
    for a, b, c in coeffs:
        s = a * s + b * s ** 3 + c * s ** 5
    return s


SHAPES = [(5, 9), (9, 5), (16, 16), (24, 40), (40, 24), (1, 7), (7, 1)]
COEFF_SETS = {
    "quintic5": [QUINTIC] * 5,
    "quintic6": [QUINTIC] * 6,
    "cubic5": [CUBIC] * 5,
    "schedule": [(3.0, -3.2, 1.2), (2.0, -1.5, 0.5), (1.5, -0.5, 0.0)],
}


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("cname", sorted(COEFF_SETS))
def test_svd_closed_form(shape, cname):
    rows, cols = shape
    r = min(rows, cols)
    # skewed spectrum: one large value, a geometric tail
    sig = 3.0 * 0.55 ** np.arange(r)
    U, s, V = _random_svd(rows, cols, sig, seed=rows * 100 + cols)
    G = U @ np.diag(s) @ V.T
    eps = 1e-7
    coeffs = COEFF_SETS[cname]
    O = oracle.orthogonalize(G, coeffs, eps)
    s0 = s / (np.sqrt(np.sum(s ** 2)) + eps)
    expect = U @ np.diag(_scalar_orbit(s0, coeffs)) @ V.T
    assert O.shape == (rows, cols)
    assert np.max(np.abs(O - expect)) < 1e-12
    # singular values of O are |p^k(sigma_i)| (O O^T eigenvalues are p^k(sigma)^2)
    sv = np.sort(np.linalg.svd(O, compute_uv=False))
    assert np.allclose(sv, np.sort(np.abs(_scalar_orbit(s0, coeffs))), atol=1e-12)


def test_exact_rational_orbit():
    """diag(d) in, diag(p^k(d / ||d||)) out, with exact rationals for p^k."""
    d = [Fraction(3, 4), Fraction(1, 2), Fraction(-1, 8), Fraction(1, 16)]
    coeffs = [(Fraction(3, 2), Fraction(-1, 2), Fraction(0))] * 3 + \
             [(Fraction(17, 5), Fraction(-19, 4), Fraction(2))] * 2
    # X0 is fed to newton_schulz directly, so every entry stays rational
    x0 = [x / 2 for x in d]  # all |x| < 1
    exact = []
    for x in x0:
        for a, b, c in coeffs:
            x = a * x + b * x ** 3 + c * x ** 5
        exact.append(x)
    X0 = np.zeros((4, 6))
    X0[np.arange(4), np.arange(4)] = [float(x) for x in x0]
    out = oracle.newton_schulz(X0, [tuple(float(v) for v in t) for t in coeffs])
    got = np.diag(out[:, :4])
    assert np.allclose(got, [float(e) for e in exact], rtol=1e-13, atol=1e-15)
    assert np.all(out[:, 4:] == 0.0)


@pytest.mark.parametrize("shape", [(2, 2), (3, 5), (5, 3), (4, 8), (8, 16), (16, 8)])
def test_cubic_converges_to_polar_factor(shape):
    rows, cols = shape
    r = min(rows, cols)
    sig = np.linspace(1.0, 0.35, r)  # sigma_min / ||sigma||_2 >= 0.1
    U, s, V = _random_svd(rows, cols, sig, seed=7 * rows + cols)
    assert s.min() / np.linalg.norm(s) >= 0.1
    G = U @ np.diag(s) @ V.T
    O = oracle.orthogonalize(G, [CUBIC] * 40, 0.0)
    assert np.max(np.abs(O - U @ V.T)) < 1e-10


def test_quintic_does_not_converge_to_one():
    """The quintic overshoots: its fixed-point orbit from 1 oscillates."""
    x = 1.0
    orbit = []
    for _ in range(4):
        x = QUINTIC[0] * x + QUINTIC[1] * x ** 3 + QUINTIC[2] * x ** 5
        orbit.append(x)
    assert abs(orbit[0] - 0.701) < 1e-3 and abs(orbit[1] - 1.114) < 2e-3
    X = np.eye(3, 4)
    out = oracle.newton_schulz(X, [QUINTIC] * 2)
    assert np.allclose(np.diag(out[:, :3]), orbit[1])


def test_momentum_three_step_unroll():
    rng = np.random.default_rng(3)
    G1, G2, G3 = (rng.standard_normal((2, 3)) for _ in range(3))
    mu = 0.95
    M = np.zeros((2, 3))
    for G in (G1, G2, G3):
        M = oracle.momentum_update(M, G, mu)
    M3 = (1 - mu) * (G3 + mu * G2 + mu * mu * G1)
    assert np.max(np.abs(M - M3)) < 1e-15
    U = oracle.nesterov_lookahead(M, G3, mu, True)
    U3 = (1 - mu) * G3 + mu * (1 - mu) * (G3 + mu * G2 + mu * mu * G1)
    assert np.max(np.abs(U - U3)) < 1e-15
    assert oracle.nesterov_lookahead(M, G3, mu, False) is M


def test_sgd_form_three_step_unroll_and_step():
    rng = np.random.default_rng(31)
    G1, G2, G3 = (rng.standard_normal((2, 3)) for _ in range(3))
    mu = 0.9
    M = np.zeros((2, 3))
    for G in (G1, G2, G3):
        M = oracle.momentum_update_sgd(M, G, mu)
    assert np.max(np.abs(M - (G3 + mu * G2 + mu * mu * G1))) < 1e-15
    U = oracle.nesterov_lookahead_sgd(M, G3, mu, True)
    assert np.max(np.abs(U - (G3 + mu * (G3 + mu * G2 + mu * mu * G1)))) < 1e-15
    # through muon_step: the SGD buffer is (1 - mu)^-1 times the moving average
    # and the orthogonalised update is the same
    th = rng.standard_normal((6, 10))
    G = rng.standard_normal((6, 10))
    hp = dict(lr=0.02, mu=mu, weight_decay=0.0, nesterov=1, coeffs=[QUINTIC] * 5, eps=0.0)
    t_ma, M_ma, O_ma = oracle.muon_step(th, G, np.zeros((6, 10)), hp, "f32")
    t_sg, M_sg, O_sg = oracle.muon_step(th, G, np.zeros((6, 10)), dict(hp, sgd_momentum=1), "f32")
    assert np.allclose(M_sg * (1 - mu), M_ma, atol=1e-14)
    assert np.max(np.abs(O_sg - O_ma)) < 1e-12
    assert np.array_equal(t_sg, t_ma)


@pytest.mark.parametrize("nesterov", [0, 1])
def test_sgd_form_step_on_diagonal_matrices_closed_form(nesterov):
    """On 'diagonal' 4 x 6 matrices every product of the iteration stays
    diagonal, so O is the scalar orbit of each entry of U / ||U||_F. From a
    momentum that is not a multiple of the gradient the SGD form gives
    M' = mu M + G and U = G + mu M' with Nesterov (else U = M'): two
    directions the normalisation cannot make equal."""
    def diag(d):
        return np.eye(4, 6) * d[:, None]

    g = np.array([1.0, -2.0, 0.5, 3.0])
    m0 = np.array([4.0, 1.0, -2.0, 0.5])
    mu, lr, wd = 0.9, 0.02, 0.3
    th = np.arange(24, dtype=np.float64).reshape(4, 6) / 10.0
    hp = dict(lr=lr, mu=mu, weight_decay=wd, nesterov=nesterov, coeffs=[QUINTIC] * 5, eps=0.0,
              sgd_momentum=1)
    t1, M1, O = oracle.muon_step(th, diag(g), diag(m0), hp, "f32")
    m1 = mu * m0 + g
    u = g + mu * m1 if nesterov else m1
    assert np.max(np.abs(M1 - diag(m1))) < 1e-15
    O_exp = diag(_scalar_orbit(u / np.linalg.norm(u), [QUINTIC] * 5))
    assert np.max(np.abs(O - O_exp)) < 1e-12
    th_exp = th * (1 - lr * wd) - lr * 1.0 * O_exp
    assert np.max(np.abs(t1 - th_exp)) <= 1e-6 * np.max(np.abs(th_exp))


def test_sgd_momentum_form_gives_the_same_update():
    """From zero state the SGD form M' = mu M' + G is M / (1 - mu); the
    normalisation removes the factor, so O is the same (reading R1)."""
    rng = np.random.default_rng(11)
    mu = 0.9
    M = np.zeros((6, 10))
    Ms = np.zeros((6, 10))
    for _ in range(4):
        G = rng.standard_normal((6, 10))
        M = oracle.momentum_update(M, G, mu)
        Ms = mu * Ms + G
    assert np.allclose(Ms * (1 - mu), M, atol=1e-13)
    a = oracle.orthogonalize(M, [QUINTIC] * 5, 0.0)
    b = oracle.orthogonalize(Ms, [QUINTIC] * 5, 0.0)
    assert np.max(np.abs(a - b)) < 1e-12


def test_anvil_momenta_and_ema_unroll():
    rng = np.random.default_rng(5)
    Gs = [rng.standard_normal((2, 3)) for _ in range(3)]
    bf, bs = 0.9, 0.99
    Mf = np.zeros((2, 3))
    Ms = np.zeros((2, 3))
    for G in Gs:
        Mf = oracle.momentum_update(Mf, G, bf)
        Ms = oracle.momentum_update(Ms, G, bs)
    G1, G2, G3 = Gs
    assert np.max(np.abs(Mf - (1 - bf) * (G3 + bf * G2 + bf ** 2 * G1))) < 1e-15
    assert np.max(np.abs(Ms - (1 - bs) * (G3 + bs * G2 + bs ** 2 * G1))) < 1e-15
    th = [rng.standard_normal((2, 3)) for _ in range(4)]
    beta = 0.99
    e = th[0].copy()
    for t in th[1:]:
        e = oracle.ema_update(e, t, beta)
    expect = beta ** 3 * th[0] + (1 - beta) * (beta ** 2 * th[1] + beta * th[2] + th[3])
    assert np.max(np.abs(e - expect)) < 1e-15


def test_page_constants():
    with open(os.path.join(GOLDEN, "pages_constants.json")) as f:
        pc = json.load(f)
    wf = pc["readout_final_weight"]["value"]
    wa = pc["readout_average_weight"]["value"]
    assert abs(wf + wa - 1.0) < 1e-12
    th = np.full((2, 2), 1.0)
    ema = np.zeros((2, 2))
    assert np.allclose(oracle.readout_blend(th, ema), wf)
    assert np.allclose(oracle.readout_blend(ema, th), wa)
    lo, hi = pc["ema_beta_range"]["value"]
    # beta = 0 keeps only the current weights
    assert np.allclose(oracle.ema_update(ema, th, lo), th)
    assert pc["anvil_polynomial_applications"]["value"] == 6
    assert hi == 1.0


@pytest.mark.parametrize("shape", [(6, 10), (10, 6)])
def test_transpose_and_permutation_invariance(shape):
    rng = np.random.default_rng(21)
    G = rng.standard_normal(shape)
    c = [QUINTIC] * 5
    O = oracle.orthogonalize(G, c, 1e-7)
    assert np.max(np.abs(oracle.orthogonalize(G.T, c, 1e-7) - O.T)) < 1e-12
    P = rng.permutation(shape[0])
    Q = rng.permutation(shape[1])
    Op = oracle.orthogonalize(G[P][:, Q], c, 1e-7)
    assert np.max(np.abs(Op - O[P][:, Q])) < 1e-12
    # gradient scale drops out of the normalised iteration (up to eps)
    O7 = oracle.orthogonalize(7.0 * G, c, 0.0)
    O1 = oracle.orthogonalize(G, c, 0.0)
    assert np.max(np.abs(O7 - O1)) < 1e-12


def test_zero_gradient_only_decays():
    th = np.random.default_rng(1).standard_normal((4, 8))
    hp = dict(lr=0.02, mu=0.95, weight_decay=1.6, nesterov=1, coeffs=[QUINTIC] * 5, eps=1e-7)
    t1, M1, O = oracle.muon_step(th, np.zeros((4, 8)), np.zeros((4, 8)), hp, "f32")
    assert np.all(O == 0.0) and np.all(M1 == 0.0)
    assert np.allclose(t1, (th * (1 - 0.02 * 1.6)).astype(np.float32))


@pytest.mark.parametrize("shape", [(3, 12), (12, 3), (8, 8)])
def test_rank_one_update_closed_form(shape):
    """G = u v^T: O = p^k(s0) u^ v^T and theta' = theta (1 - lr wd) - lr s O."""
    rows, cols = shape
    rng = np.random.default_rng(rows * cols)
    u = rng.standard_normal(rows)
    v = rng.standard_normal(cols)
    G = np.outer(u, v)
    th = rng.standard_normal(shape)
    eps = 1e-7
    hp = dict(lr=0.03, mu=0.5, weight_decay=0.25, nesterov=0, coeffs=[QUINTIC] * 5, eps=eps)
    t1, M1, O = oracle.muon_step(th, G, np.zeros(shape), hp, "f32")
    # M1 = 0.5 G, still rank one with the same singular vectors
    nrm = 0.5 * np.linalg.norm(u) * np.linalg.norm(v)
    s0 = nrm / (nrm + eps)
    p = _scalar_orbit([s0], [QUINTIC] * 5)[0]
    O_exp = p * np.outer(u / np.linalg.norm(u), v / np.linalg.norm(v))
    assert np.max(np.abs(O - O_exp)) < 1e-12
    s = math.sqrt(max(1.0, rows / cols))
    th_exp = th * (1 - 0.03 * 0.25) - 0.03 * s * O_exp
    assert np.max(np.abs(t1 - th_exp)) <= 1e-6 * np.max(np.abs(th_exp))


def test_cautious_mask_closed_form():
    """Positive rank-one momentum gives O > 0 everywhere, so the mask is the
    sign pattern of the slow momentum."""
    rows, cols = 4, 6
    u = np.linspace(1.0, 2.0, rows)
    v = np.linspace(0.5, 1.5, cols)
    G = np.outer(u, v)
    Ms0 = np.where(np.arange(rows * cols).reshape(rows, cols) % 3 == 0, -50.0, 50.0)
    th = np.full((rows, cols), 0.5)
    hp = dict(lr=0.05, beta_fast=0.9, beta_slow=0.99, weight_decay=0.1,
              coeffs=[QUINTIC] * 6, eps=1e-7)
    t1, Mf, Ms, O, mask = oracle.anvil_step(th, G, np.zeros_like(G), Ms0, hp, "f32")
    assert np.all(O > 0)
    assert np.array_equal(mask, (Ms > 0).astype(float))
    assert np.array_equal(mask, (Ms0 > 0).astype(float))  # slow momentum keeps its sign
    expect = th - 0.05 * 0.1 * mask * th - 0.05 * 1.0 * O
    assert np.max(np.abs(t1 - expect)) < 1e-6


def test_anvil_tall_rank_one_with_zero_rows_closed_form():
    """A tall rank-one gradient G = u v^T with two exactly-zero rows, both
    momenta starting at zero: Mf = (1 - beta_fast) G, Ms = (1 - beta_slow) G,
    O = p^6(s0) u^ v^T, so O * Ms > 0 wherever G != 0 and is exactly 0 on the
    zero rows. The sign-agreement rule is strict there (no sign, no decay):
    those rows of theta come back unchanged. Elsewhere theta decays and takes
    the update scaled by max(1, R/C)^(1/2) = 2 for a 12 x 3 matrix."""
    rows, cols = 12, 3
    rng = np.random.default_rng(1203)
    u = rng.standard_normal(rows)
    u[[4, 9]] = 0.0
    v = rng.uniform(0.5, 1.5, cols) * np.array([1.0, -1.0, 1.0])
    G = np.outer(u, v)
    th = rng.standard_normal((rows, cols))
    lr, wd, bf, bs, eps = 0.05, 0.4, 0.9, 0.99, 1e-7
    hp = dict(lr=lr, beta_fast=bf, beta_slow=bs, weight_decay=wd, coeffs=[QUINTIC] * 6, eps=eps)
    t1, Mf, Ms, O, mask = oracle.anvil_step(th, G, np.zeros_like(G), np.zeros_like(G), hp, "f32")
    nrm = (1 - bf) * np.linalg.norm(u) * np.linalg.norm(v)
    p = _scalar_orbit([nrm / (nrm + eps)], [QUINTIC] * 6)[0]
    assert p > 0
    O_exp = p * np.outer(u / np.linalg.norm(u), v / np.linalg.norm(v))
    assert np.max(np.abs(O - O_exp)) < 1e-12
    assert np.array_equal(mask, (G != 0).astype(float))
    th_exp = np.where(G != 0, th * (1 - lr * wd), th) - lr * 2.0 * O_exp
    assert np.array_equal(t1[[4, 9]], th[[4, 9]].astype(np.float32).astype(np.float64))
    assert np.max(np.abs(t1 - th_exp)) <= 1e-6 * np.max(np.abs(th_exp))


def test_round_to_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-20, 20, 20000),
                        np.array([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e38])])
    x32 = x.astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).float().numpy().astype(np.float64)
    got = oracle.round_to_bf16(x32.astype(np.float64))
    assert np.array_equal(got, want)


def test_flop_count_matches_dense_count_minus_symmetry():
    r, c = 768, 3072
    f = oracle.ns_flops_algorithmic(c, r, 1)  # tall, same as wide
    assert f == oracle.ns_flops_algorithmic(r, c, 1)
    dense = 4 * r * r * c + 2 * r ** 3
    assert f < dense and f > 0.7 * dense


@pytest.mark.parametrize("shape", [(1, 1), (3, 5), (4, 4), (7, 2)])
def test_flop_count_by_counting_operations(shape):
    """Count the multiply-adds one iteration performs when A = X X^T and
    A A are computed on and above the diagonal only (each entry a dot
    product of length c, resp. r) and B X in full, two flops each."""
    r, c = min(shape), max(shape)
    flops = 0
    for i in range(r):
        for j in range(i, r):
            flops += 2 * c          # A_ij = <x_i, x_j>
            flops += 2 * r          # (A A)_ij
    for i in range(r):
        for j in range(c):
            flops += 2 * r          # (B X)_ij
    assert oracle.ns_flops_algorithmic(*shape, 3) == 3 * flops


# ---- sensitivity: plausible mistakes must break the closed-form pin -------
def _closed_form_error(ns_impl):
    rows, cols = 9, 14
    U, s, V = _random_svd(rows, cols, 2.0 * 0.6 ** np.arange(rows), seed=99)
    X0 = U @ np.diag(s / np.linalg.norm(s)) @ V.T
    c = [QUINTIC] * 5
    expect = U @ np.diag(_scalar_orbit(s / np.linalg.norm(s), c)) @ V.T
    return np.max(np.abs(ns_impl(X0, c) - expect))


def test_pin_catches_plausible_mistakes():
    assert _closed_form_error(oracle.newton_schulz) < 1e-12

    def wrong_sign(X0, c):
        return oracle.newton_schulz(X0, [(a, -b, c_) for a, b, c_ in c])

    def dropped_square(X0, c):
        return oracle.newton_schulz(X0, [(a, b, 0.0) for a, b, _ in c])

    def gram_transposed(X0, c):  # A = X^T X on the long side, product order swapped
        X = X0.copy()
        for a, b, c_ in c:
            A = X.T @ X
            X = a * X + X @ (b * A + c_ * A @ A) * 0.5
        return X

    with np.errstate(all="ignore"):
        for bad in (wrong_sign, dropped_square, gram_transposed):
            err = _closed_form_error(bad)
            assert not (err < 1e-3), bad.__name__


# ---- ANVIL: which momentum gets which beta, and what each one feeds --------
def test_anvil_step_wiring_three_steps_closed_form():
    """Three anvil_step calls from non-zero momenta with beta_fast != beta_slow,
    against closed forms written out by hand.

    The gradient is the same positive rank-one matrix G = u v^T every step and
    both momenta start as multiples of it (M_fast) or of a fixed sign pattern
    (M_slow), so after step t
      M_fast_t = beta_f^t M_fast_0 + (1 - beta_f^t) G          (a multiple of G)
      M_slow_t = beta_s^t M_slow_0 + (1 - beta_s^t) G.
    O is the Newton-Schulz image of the rank-one fast momentum: sign(k) times
    p^6(s0) times the unit rank-one direction. The start values are chosen so
    that the sign of k and the slow momentum's sign on part of the entries
    both flip if the two betas are exchanged ("ANVIL II와 가중치 평균": the fast
    momentum is the update, the slow one only picks where the decay applies).
    """
    rows, cols = 4, 6
    u = np.linspace(1.0, 2.0, rows)
    v = np.linspace(0.5, 1.5, cols)
    G = np.outer(u, v)                      # entries in [0.5, 3]
    bf, bs = 0.9, 0.99
    k0 = -0.08                              # M_fast_0 = k0 G
    pattern = np.where(np.arange(rows * cols).reshape(rows, cols) % 2 == 0, -0.5, 0.5)
    th = np.full((rows, cols), 0.25)
    lr, wd, eps = 0.05, 0.4, 1e-7
    coeffs = [QUINTIC] * 6
    hp = dict(lr=lr, beta_fast=bf, beta_slow=bs, weight_decay=wd, coeffs=coeffs, eps=eps)
    Mf, Ms = k0 * G, pattern.copy()
    unit = np.outer(u / np.linalg.norm(u), v / np.linalg.norm(v))
    gnorm = np.linalg.norm(u) * np.linalg.norm(v)
    flipped = 0
    for t in (1, 2, 3):
        th_new, Mf, Ms, O, mask = oracle.anvil_step(th, G, Mf, Ms, hp, "f32")
        k = bf ** t * k0 + (1 - bf ** t)
        assert np.max(np.abs(Mf - k * G)) < 1e-14
        Ms_exp = bs ** t * pattern + (1 - bs ** t) * G
        assert np.max(np.abs(Ms - Ms_exp)) < 1e-14
        s0 = abs(k) * gnorm / (abs(k) * gnorm + eps)
        O_exp = np.sign(k) * _scalar_orbit([s0], coeffs)[0] * unit
        assert np.max(np.abs(O - O_exp)) < 1e-12
        mask_exp = (O_exp * Ms_exp > 0).astype(float)
        assert np.array_equal(mask, mask_exp)
        th_exp = th - lr * wd * mask_exp * th - lr * 1.0 * O_exp
        assert np.max(np.abs(th_new - th_exp.astype(np.float32))) <= 1e-7
        # with the betas exchanged the fast coefficient changes sign and the
        # slow momentum changes sign on some entries
        k_sw = bs ** t * k0 + (1 - bs ** t)
        Ms_sw = bf ** t * pattern + (1 - bf ** t) * G
        assert np.sign(k_sw) != np.sign(k)
        flipped += int(np.sum(np.sign(Ms_sw) != np.sign(Ms_exp)))
        th = th_new
    assert flipped > 0


# ---- weighted checkpoint average ------------------------------------------
def test_weighted_average_three_checkpoints_by_hand():
    """theta_1 = (1, 2), theta_2 = (3, -1), theta_3 = (0, 4), w = (1, 2, 5):
    (1*(1,2) + 2*(3,-1) + 5*(0,4)) / 8 = (7/8, 20/8)."""
    thetas = [np.array([1.0, 2.0]), np.array([3.0, -1.0]), np.array([0.0, 4.0])]
    got = oracle.weighted_average(thetas, [1.0, 2.0, 5.0])
    assert np.array_equal(got, np.array([0.875, 2.5]))
    # the running form: beta = (0, 1 - 2/3, 1 - 5/8)
    betas = oracle.weighted_average_betas([1.0, 2.0, 5.0])
    assert betas[0] == 0.0 and abs(betas[1] - 1.0 / 3.0) < 1e-16 and betas[2] == 0.375
    e = thetas[0]
    for b, th in zip(betas, thetas):
        e = oracle.ema_update(e, th, b)
    assert np.max(np.abs(e - np.array([0.875, 2.5]))) < 1e-15


def test_weighted_average_running_form_exact_rationals():
    """The beta schedule reproduces the weighted average exactly (Fraction)."""
    rng = np.random.default_rng(4)
    ths = [[Fraction(int(x), 7) for x in rng.integers(-20, 20, 3)] for _ in range(6)]
    ws = [Fraction(int(x), 3) for x in rng.integers(1, 9, 6)]
    W = sum(ws)
    exact = [sum(w * t[j] for w, t in zip(ws, ths)) / W for j in range(3)]
    e = list(ths[0])
    Wn = Fraction(0)
    for w, t in zip(ws, ths):
        Wn += w
        beta = 1 - w / Wn
        e = [beta * a + (1 - beta) * b for a, b in zip(e, t)]
    assert e == exact
    got = oracle.weighted_average([np.array([float(x) for x in t]) for t in ths],
                                  [float(w) for w in ws])
    assert np.allclose(got, [float(x) for x in exact], rtol=1e-14, atol=1e-15)
    betas = oracle.weighted_average_betas([float(w) for w in ws])
    e = np.array([float(x) for x in ths[0]])
    for b, t in zip(betas, ths):
        e = oracle.ema_update(e, np.array([float(x) for x in t]), b)
    assert np.allclose(e, [float(x) for x in exact], rtol=1e-13, atol=1e-14)


def test_ema_is_a_weighted_average():
    """The EMA from theta_bar_0 = theta_0 equals the weighted average with
    w_0 = beta^n and w_i = (1 - beta) beta^(n - i)."""
    rng = np.random.default_rng(8)
    ths = [rng.standard_normal((3, 4)) for _ in range(5)]
    beta = 0.9
    e = ths[0].copy()
    for th in ths[1:]:
        e = oracle.ema_update(e, th, beta)
    n = len(ths) - 1
    w = [beta ** n] + [(1 - beta) * beta ** (n - i) for i in range(1, n + 1)]
    assert np.max(np.abs(oracle.weighted_average(ths, w) - e)) < 1e-14
    with pytest.raises(ValueError):
        oracle.weighted_average(ths, [0.0] * len(ths))
