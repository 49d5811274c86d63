"""Pins for the float64 oracle: closed forms, textbook special cases, brute
force and LAPACK.  None of these re-types the oracle's own formula; each
would fail on a dropped term, a wrong sign or index, or a transposed operand
somewhere in the oracle."""
import json
import os
from math import sqrt

import numpy as np
import pytest

from oracle import prism_ref as o

HERE = os.path.dirname(os.path.abspath(__file__))


def rot(n, seed):
    Q, Rq = np.linalg.qr(np.random.default_rng(seed).standard_normal((n, n)))
    return Q * np.sign(np.diag(Rq))


def spd(n, lam, seed):
    Q = rot(n, seed)
    return (Q * lam) @ Q.T, Q


# ---------------------------------------------------------------- Gram EMA
def test_ema_rank_one_closed_form():
    m, n, i, j, s, beta, eps, e0 = 6, 4, 2, 3, 1.7, 0.95, 1e-3, 0.25
    G = np.zeros((m, n)); G[i, j] = s
    L, R = o.gram_ema_ref(G, e0 * np.eye(m), e0 * np.eye(n), beta, eps)
    for k in range(m):
        want = beta * e0 + eps + ((1 - beta) * s * s if k == i else 0.0)
        assert L[k, k] == pytest.approx(want, rel=1e-15)
    for k in range(n):
        want = beta * e0 + eps + ((1 - beta) * s * s if k == j else 0.0)
        assert R[k, k] == pytest.approx(want, rel=1e-15)
    assert np.count_nonzero(L - np.diag(np.diag(L))) == 0
    assert np.count_nonzero(R - np.diag(np.diag(R))) == 0


def test_ema_orthogonal_gradient_closed_form():
    n, s, beta, eps = 12, 0.3, 0.9, 1e-8
    Q = rot(n, 1)
    L = R = eps * np.eye(n)
    ell = eps
    for _ in range(7):
        L, R = o.gram_ema_ref(s * Q, L, R, beta, eps)
        ell = beta * ell + (1 - beta) * s * s + eps       # scalar recursion
    np.testing.assert_allclose(L, ell * np.eye(n), atol=1e-15)
    np.testing.assert_allclose(R, ell * np.eye(n), atol=1e-15)


def test_ema_trace_symmetry_psd():
    rng = np.random.default_rng(3)
    m, n, beta, eps = 9, 5, 0.95, 1e-6
    G = rng.standard_normal((m, n))
    L0, R0 = eps * np.eye(m), eps * np.eye(n)
    L, R = o.gram_ema_ref(G, L0, R0, beta, eps)
    fro2 = np.sum(G * G)
    assert np.trace(L - beta * L0) - m * eps == pytest.approx((1 - beta) * fro2, rel=1e-13)
    assert np.trace(R - beta * R0) - n * eps == pytest.approx((1 - beta) * fro2, rel=1e-13)
    assert np.array_equal(L, L.T) and np.array_equal(R, R.T)
    assert np.linalg.eigvalsh(L).min() > 0 and np.linalg.eigvalsh(R).min() > 0


def test_ema_row_vs_column_covariance():
    # L is the row covariance (m x m) and R the column covariance (n x n):
    # a gradient whose rows are identical has a rank-one R direction set by the row.
    m, n = 5, 3
    row = np.array([1.0, -2.0, 0.5])
    G = np.tile(row, (m, 1))
    L, R = o.gram_ema_ref(G, np.zeros((m, m)), np.zeros((n, n)), 0.0, 0.0)
    np.testing.assert_allclose(R, m * np.outer(row, row), rtol=1e-15)
    np.testing.assert_allclose(L, np.full((m, m), row @ row), rtol=1e-15)


# ---------------------------------------------------------- polynomials
def test_taylor_series_of_inverse_sqrt():
    # (1 - x)^(-1/2) = 1 + x/2 + 3x^2/8 + 5x^3/16 + 35x^4/128 + ...
    np.testing.assert_allclose(o.taylor_coeffs(4), [1, 0.5, 0.375, 0.3125, 35 / 128], rtol=0)


def test_golden_interval_is_taylor_to_one():
    page = json.load(open(os.path.join(HERE, "golden", "page_constants.json")))
    lo, hi = page["alpha_interval_d1"]["value"]
    # alpha = lo must reproduce the plain Taylor update (classic Newton-Schulz)
    assert o.taylor_coeffs(1)[1] == lo
    np.testing.assert_allclose(o.g_coeffs(1, lo), [1.0, 0.5])
    assert hi == 1.0
    assert page["root_exponent"]["value"] == -0.25


def test_classic_newton_schulz_residual():
    # d=1, alpha=1/2: g = (3 - x)/2 in terms of x = 1 - xi; textbook residual 3/4 xi^2 + 1/4 xi^3
    np.testing.assert_allclose(o.residual_coeffs(1, 0.5), [0, 0, 0.75, 0.25], atol=1e-15)
    # d=2, alpha=3/8 is the third-order Newton-Schulz (15 - 10 x + 3 x^2)/8: no xi^2 term
    r = o.residual_coeffs(2, 0.375)
    assert abs(r[2]) < 1e-15 and abs(r[0]) < 1e-15 and abs(r[1]) < 1e-15
    x = np.linspace(-0.3, 1.0, 17)
    g_textbook = (15 - 10 * x + 3 * x * x) / 8
    np.testing.assert_allclose(np.polynomial.polynomial.polyval(1 - x, o.g_coeffs(2, 0.375)),
                               g_textbook, rtol=1e-14)


@pytest.mark.parametrize("d", [1, 2, 3])
def test_residual_table_matches_polynomial(d):
    T = o.residual_alpha_table(d)
    for a in (0.0, 0.3, 0.5, 1.0, -0.7):
        via_table = T[:, 0] + T[:, 1] * a + T[:, 2] * a * a
        np.testing.assert_allclose(via_table, o.residual_coeffs(d, a), atol=1e-14)
    # r vanishes below degree d for every alpha, and r(1; alpha) = 1 (X = 0 is a fixed point)
    assert np.all(T[:d] == 0)
    for a in (0.2, 0.9):
        assert np.polynomial.polynomial.polyval(1.0, o.residual_coeffs(d, a)) == pytest.approx(1.0)


def ideal_alpha(d, xi):
    """alpha that makes (1 - xi) g(xi)^2 = 1 exactly for a scalar residual xi."""
    f = sum(o.taylor_coeffs(d)[j] * xi ** j for j in range(d))
    return (1 / sqrt(1 - xi) - f) / xi ** d


@pytest.mark.parametrize("d,xi,want", [
    (1, 0.5, 2 * sqrt(2) - 2),        # 0.828427...
    (1, 0.75, 1.0),                   # ideal 4/3, clamped to the upper end
    (1, -0.5, 0.5),                   # ideal 0.367, clamped to the lower end
    (2, 0.5, (sqrt(2) - 1.25) * 4),   # 0.656854...
    (2, 0.1, None),
])
def test_alpha_closed_form_scalar_residual(d, xi, want):
    n, p = 8, 3
    lo, hi = (0.5, 1.0) if d == 1 else (0.375, 1.0)
    S = np.random.default_rng(7).standard_normal((n, p))
    a, coef = o.prism_alpha_ref(xi * np.eye(n), S, d, lo, hi)
    if want is None:
        want = ideal_alpha(d, xi)
        assert lo < want < hi
    assert a == pytest.approx(want, abs=1e-9)


def _grid_alpha(Rk, S, d, lo, hi, step=1e-6):
    """Brute force: evaluate ||(I - (I - R) g(R)^2) S||_F^2 on a grid, from the
    matrix identity itself (no coefficient table, no Gram matrix)."""
    n = Rk.shape[0]
    I = np.eye(n)
    f = np.eye(n) if d == 1 else I + 0.5 * Rk
    Rd = np.linalg.matrix_power(Rk, d)
    F, Fd = f @ S, Rd @ S
    # g(R) S = F + a Fd, and (I-R) g(R)^2 S = (I-R) g(R) (F + a Fd)
    gF, gFd = f @ F, f @ Fd
    RdF, RdFd = Rd @ F, Rd @ Fd
    A0 = S - (I - Rk) @ gF
    A1 = -(I - Rk) @ (gFd + RdF)
    A2 = -(I - Rk) @ RdFd
    grid = np.arange(lo, hi + step / 2, step)
    best, besta = np.inf, None
    for chunk in np.array_split(grid, 50):
        a = chunk[:, None, None]
        vals = np.sum((A0[None] + a * A1[None] + a * a * A2[None]) ** 2, axis=(1, 2))
        k = int(np.argmin(vals))
        if vals[k] < best:
            best, besta = vals[k], chunk[k]
    return besta


@pytest.mark.parametrize("kind", ["diag", "rotated", "symmetric", "nonsymmetric"])
@pytest.mark.parametrize("p", [1, 2, 4, 8])
@pytest.mark.parametrize("d", [1, 2])
def test_alpha_brute_force_8x8(kind, p, d):
    rng = np.random.default_rng(100 * p + d + len(kind))
    n = 8
    lam = rng.uniform(0.05, 0.95, n)
    if kind == "diag":
        Rk = np.diag(lam)
    elif kind == "rotated":
        Q = rot(n, 5)
        Rk = (Q * lam) @ Q.T
    elif kind == "symmetric":
        M = rng.standard_normal((n, n)); Rk = 0.15 * (M + M.T)
    else:
        Rk = np.diag(lam) + 0.05 * rng.standard_normal((n, n))
    S = rng.standard_normal((n, p))
    lo, hi = (0.5, 1.0) if d == 1 else (0.375, 1.0)
    a, _ = o.prism_alpha_ref(Rk, S, d, lo, hi)
    assert a == pytest.approx(_grid_alpha(Rk, S, d, lo, hi), abs=2e-6)


@pytest.mark.parametrize("d", [1, 2])
def test_alpha_exact_trace_objective(d):
    # p = n with an orthogonal sketch: the sketched objective is the exact
    # spectral least-squares objective sum_i r(lambda_i; alpha)^2.
    n = 10
    rng = np.random.default_rng(11)
    M = rng.standard_normal((n, n)); Rk = 0.2 * (M + M.T)
    S = rot(n, 12)
    _, coef = o.prism_alpha_ref(Rk, S, d, 0.3, 1.0)
    lam = np.linalg.eigvalsh(Rk)
    P = np.polynomial.polynomial
    for a in (0.1, 0.4, 0.8, 1.3):
        r_of_lam = 1 - (1 - lam) * P.polyval(lam, o.g_coeffs(d, a)) ** 2
        assert P.polyval(a, coef) == pytest.approx(np.sum(r_of_lam ** 2), rel=1e-10)


def test_alpha_constant_objective_takes_lower_end():
    a, coef = o.prism_alpha_ref(np.zeros((6, 6)), np.ones((6, 2)), 2, 0.375, 1.0)
    assert a == 0.375


# ------------------------------------------------------- Newton-Schulz passes
def scalar_coupled(lam, alphas, d):
    """Eigenvalue-domain recurrence: y <- y g(1 - z y), z <- g(1 - z y) z."""
    y, z = lam.copy(), np.ones_like(lam)
    for a in alphas:
        xi = 1 - z * y
        c = o.taylor_coeffs(d).copy(); c[d] = a
        g = sum(c[j] * xi ** j for j in range(d + 1))
        y, z = y * g, g * z
    return y, z


@pytest.mark.parametrize("d", [1, 2])
@pytest.mark.parametrize("rotated", [False, True])
def test_coupled_matches_scalar_recurrence(d, rotated):
    n = 16
    lam = np.exp(np.random.default_rng(2).uniform(np.log(1e-3), 0, n))
    Q = rot(n, 4) if rotated else np.eye(n)
    B = (Q * lam) @ Q.T
    opts = o.PrismOpts(d=d, p=4, lo=0.5 if d == 1 else 0.375, tol=1e-13, max_iter=60,
                       stall_below=0.0)
    S = np.random.default_rng(5).standard_normal((200, n, 4))
    Y, Z, info = o.coupled_ref(B, opts, S)
    assert info.status == o.OK
    y, z = scalar_coupled(lam, info.alpha, d)
    np.testing.assert_allclose(Y, (Q * y) @ Q.T, atol=1e-12)
    np.testing.assert_allclose(Z, (Q * z) @ Q.T, atol=1e-9 * np.max(z))
    np.testing.assert_allclose(y, np.sqrt(lam), rtol=1e-11)
    np.testing.assert_allclose(z, 1 / np.sqrt(lam), rtol=1e-11)


def test_textbook_coupled_newton_schulz():
    # d=1 with alpha fixed at 1/2:  Y <- Y (3I - ZY)/2,  Z <- (3I - ZY) Z / 2
    n = 12
    B, _ = spd(n, np.linspace(0.2, 0.9, n), 8)
    opts = o.PrismOpts(d=1, p=2, lo=0.5, hi=1.0, tol=0.0, max_iter=6, fixed_alpha=True,
                       stall_below=0.0)
    Y, Z, info = o.coupled_ref(B, opts, None)
    Yt, Zt = B.copy(), np.eye(n)
    for _ in range(6):
        T = 3 * np.eye(n) - Zt @ Yt
        Yt, Zt = Yt @ T / 2, T @ Zt / 2
    np.testing.assert_allclose(Y, Yt, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(Z, Zt, rtol=1e-14, atol=1e-15)
    assert info.iters == 6 and info.status == o.ENOCONV


@pytest.mark.parametrize("d", [1, 2])
def test_inverse_roots_vs_eigh_and_identities(d):
    n = 32
    lam = np.exp(np.random.default_rng(9).uniform(np.log(1e-2), np.log(3.0), n))
    A, Q = spd(n, lam, 10)
    opts = o.PrismOpts(d=d, p=4, lo=0.5 if d == 1 else 0.375, tol=1e-13, max_iter=60,
                       stall_below=0.0)
    S = np.random.default_rng(6).standard_normal((200, n, 4))
    X4, infos = o.inv_root_ref(A, o.POW_INV4, opts, S)
    assert [i.status for i in infos] == [o.OK, o.OK]
    np.testing.assert_allclose(X4, (Q * lam ** -0.25) @ Q.T, atol=1e-10)
    np.testing.assert_allclose(X4 @ X4 @ X4 @ X4 @ A, np.eye(n), atol=1e-9)
    np.testing.assert_allclose(X4 @ A, A @ X4, atol=1e-9)
    np.testing.assert_allclose(X4, X4.T, atol=1e-10)
    X2, _ = o.inv_root_ref(A, o.POW_INV2, opts, S)
    np.testing.assert_allclose(X2 @ X2 @ A, np.eye(n), atol=1e-9)
    Xs, _ = o.inv_root_ref(A, o.POW_SQRT, opts, S)
    np.testing.assert_allclose(Xs @ Xs, A, atol=1e-10)


def test_inverse_root_takes_symmetric_part():
    """A non-symmetric input whose symmetric part is the SPD matrix with a
    known spectrum: the root is that of the symmetric part, from the
    closed form Q diag(lambda^(-1/4)) Q^T (an antisymmetric addition leaves
    the symmetric part unchanged)."""
    n = 24
    lam = np.exp(np.random.default_rng(11).uniform(np.log(1e-2), np.log(1.0), n))
    A, Q = spd(n, lam, 12)
    K = np.random.default_rng(13).standard_normal((n, n)) * 0.05
    opts = o.PrismOpts(d=2, p=4, lo=0.375, tol=1e-13, max_iter=60, stall_below=0.0)
    S = np.random.default_rng(14).standard_normal((200, n, 4))
    X, infos = o.inv_root_ref(A + (K - K.T), o.POW_INV4, opts, S)
    assert [i.status for i in infos] == [o.OK, o.OK]
    np.testing.assert_allclose(X, (Q * lam ** -0.25) @ Q.T, atol=1e-10)


def test_eigh_reference_on_diagonal():
    lam = np.array([4.0, 1.0, 0.0625, 16.0])
    np.testing.assert_allclose(o.spd_power_eigh(np.diag(lam), -0.25),
                               np.diag([1 / sqrt(2), 1.0, 2.0, 0.5]), atol=1e-15)


# ---------------------------------------------------------------- polar
@pytest.mark.parametrize("shape", [(40, 12), (12, 40), (16, 16)])
def test_polar_orthonormal_and_svd(shape):
    rng = np.random.default_rng(sum(shape))
    G = rng.standard_normal(shape)
    opts = o.PrismOpts(d=2, p=4, lo=0.375, tol=1e-13, max_iter=60, stall_below=0.0)
    S = rng.standard_normal((100, min(shape), 4))
    X, infos = o.polar_ref(G, opts, S)
    assert infos[0].status == o.OK
    k = min(shape)
    XtX = X.T @ X if shape[0] >= shape[1] else X @ X.T
    np.testing.assert_allclose(XtX, np.eye(k), atol=1e-11)
    np.testing.assert_allclose(X, o.polar_svd(G), atol=1e-10)


def test_polar_error_bounded_by_residual():
    rng = np.random.default_rng(21)
    G = rng.standard_normal((30, 10))
    U = o.polar_svd(G)
    for it in (2, 4, 6):
        opts = o.PrismOpts(d=1, p=3, lo=0.5, tol=0.0, max_iter=it, stall_below=0.0)
        X, infos = o.polar_ref(G, opts, rng.standard_normal((10, 10, 3)))
        resid = np.linalg.norm(np.eye(10) - X.T @ X)
        assert np.linalg.norm(X - U) <= resid + 1e-14


def test_polar_of_orthonormal_is_itself():
    Q = rot(20, 30)[:, :8]
    opts = o.PrismOpts(d=2, p=4, lo=0.375, tol=1e-13, max_iter=60, stall_below=0.0)
    X, _ = o.polar_ref(Q, opts, np.random.default_rng(1).standard_normal((60, 8, 4)))
    np.testing.assert_allclose(X, Q, atol=1e-12)


def test_polar_textbook_and_singular_value_recurrence():
    # d=1, alpha=1/2: X <- X (3I - X^T X)/2 ; on a diagonal input each singular
    # value follows s <- s (3 - s^2)/2.
    sig = np.array([3.0, 1.0, 0.2, 0.05])
    G = np.zeros((6, 4)); G[:4, :4] = np.diag(sig)
    opts = o.PrismOpts(d=1, p=2, lo=0.5, tol=0.0, max_iter=5, fixed_alpha=True, stall_below=0.0)
    X, _ = o.polar_ref(G, opts, None)
    s = sig / np.linalg.norm(sig)
    for _ in range(5):
        s = s * (3 - s * s) / 2
    want = np.zeros((6, 4)); want[:4, :4] = np.diag(s)
    np.testing.assert_allclose(X, want, atol=1e-15)


# ---------------------------------------------------------------- adaptive degree
def test_adaptive_degree_limits_reduce_to_fixed_degrees():
    """raise_above = inf never raises (the degree-1 run with [1/2, 1]);
    raise_above = 0 raises at the first step (the degree-2 run with [3/8, 1])."""
    rng = np.random.default_rng(41)
    A, _ = spd(24, np.logspace(-3, 0, 24), 41)
    S = rng.standard_normal((120, 24, 4))
    base = dict(p=4, tol=1e-10, max_iter=50, stall_below=0.0)
    never = o.PrismOpts(d=2, adaptive_degree=True, raise_above=np.inf, **base)
    always = o.PrismOpts(d=2, adaptive_degree=True, raise_above=0.0, **base)
    d1 = o.PrismOpts(d=1, lo=0.5, **base)
    d2 = o.PrismOpts(d=2, lo=0.375, **base)
    for ad, fixed in ((never, d1), (always, d2)):
        Xa, ia = o.inv_root_ref(A, o.POW_INV4, ad, S)
        Xf, if_ = o.inv_root_ref(A, o.POW_INV4, fixed, S)
        for pa, pf in zip(ia, if_):
            assert pa.degree == [fixed.d] * pa.iters
            np.testing.assert_allclose(pa.alpha, pf.alpha, atol=1e-14)
        np.testing.assert_allclose(Xa, Xf, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("xi,raised", [(0.9, False), (0.99, True)])
def test_adaptive_degree_rule_on_scalar_residual(xi, raised):
    """B = (1 - xi) I gives R_0 = xi I: the degree-1 fit's predicted ratio is
    min over alpha in [1/2, 1] of |r(xi; alpha)| / xi, attained at alpha = 1
    for these xi: 0.71 at xi = 0.9 (kept below raise_above = 0.9) and 0.9701
    at xi = 0.99 (raised)."""
    n = 6
    opts = o.PrismOpts(d=2, p=3, adaptive_degree=True, raise_above=0.9, tol=1e-12,
                       max_iter=30, stall_below=0.0)
    S = np.random.default_rng(42).standard_normal((30, n, 3))
    info = o.coupled_ref((1 - xi) * np.eye(n), opts, S)[2]
    q = abs((1 - 2) + (2 - 1) * xi + xi * xi)  # r(xi; 1) / xi
    assert (q > 0.9) == raised
    assert info.degree[0] == (2 if raised else 1)
    assert info.alpha[0] == pytest.approx(1.0 if not raised else info.alpha[0])
    # the degree never goes back down within a pass
    assert all(b >= a for a, b in zip(info.degree, info.degree[1:]))


# ---------------------------------------------------------------- sigma_min sweep
def test_prism_fewer_steps_than_taylor_across_sigma_min():
    """The pages' claim as a property: on polar inputs with singular values
    log-uniform on [sigma_min, 1], PRISM d = 2 reaches the residual in fewer
    steps than the fixed-coefficient d = 2 iteration, at every sigma_min, and
    the fixed iterations need more steps as sigma_min falls."""
    from second_order_optimizer_shampoo_b200 import synth
    S = np.random.default_rng(43).standard_normal((80, 32, 4))
    taylor_prev = 0
    for smin in (1e-1, 1e-2, 1e-3):
        G = synth.singular_spectrum(48, 32, smin, 1, 44)[0]
        base = dict(d=2, p=4, tol=1e-10, max_iter=80, stall_below=0.0)
        _, pr = o.polar_ref(G, o.PrismOpts(lo=0.375, **base), S)
        _, ty = o.polar_ref(G, o.PrismOpts(lo=0.375, fixed_alpha=True, **base), None)
        assert pr[0].status == o.OK and ty[0].status == o.OK
        assert pr[0].iters < ty[0].iters, (smin, pr[0].iters, ty[0].iters)
        assert ty[0].iters >= taylor_prev
        taylor_prev = ty[0].iters


# ---------------------------------------------------------------- sign
def test_sign_of_indefinite_matches_eigh():
    """sign(A) of a symmetric indefinite matrix: involutory (X^2 = I), commutes
    with A, and equals Q sign(Lambda) Q^T."""
    rng = np.random.default_rng(31)
    Q = rot(12, 7)
    lam = np.array([3.0, -2.0, 0.5, -0.1, 1.0, -1.0, 0.05, -4.0, 2.5, -0.3, 0.7, -0.02])
    A = (Q * lam) @ Q.T
    opts = o.PrismOpts(d=2, p=4, lo=0.375, tol=1e-13, max_iter=80, stall_below=0.0)
    X, infos = o.sign_ref(A, opts, rng.standard_normal((100, 12, 4)))
    assert infos[0].status == o.OK
    np.testing.assert_allclose(X @ X, np.eye(12), atol=1e-11)
    np.testing.assert_allclose(X @ A, A @ X, atol=1e-11)
    np.testing.assert_allclose(X, (Q * np.sign(lam)) @ Q.T, atol=1e-10)
    np.testing.assert_allclose(o.sign_eigh(A), (Q * np.sign(lam)) @ Q.T, atol=1e-12)


def test_sign_textbook_and_eigenvalue_recurrence():
    """d = 1, alpha = 1/2: X <- X (3I - X^2)/2; on a diagonal input each
    eigenvalue follows x <- x (3 - x^2)/2 with its sign kept."""
    lam = np.array([2.0, -1.0, 0.3, -0.05])
    opts = o.PrismOpts(d=1, p=2, lo=0.5, tol=0.0, max_iter=6, fixed_alpha=True, stall_below=0.0)
    X, _ = o.sign_ref(np.diag(lam), opts, None)
    x = lam / np.linalg.norm(lam)
    for _ in range(6):
        x = x * (3 - x * x) / 2
    np.testing.assert_allclose(X, np.diag(x), atol=1e-15)


def test_sign_of_spd_is_identity_and_equals_polar():
    """An SPD input has sign I; for a symmetric input the sign iteration and
    the polar iteration (R = I - X^T X) coincide step by step."""
    rng = np.random.default_rng(32)
    Q = rot(10, 3)
    A = (Q * np.linspace(0.1, 2.0, 10)) @ Q.T
    opts = o.PrismOpts(d=2, p=4, lo=0.375, tol=1e-13, max_iter=60, stall_below=0.0)
    S = rng.standard_normal((60, 10, 4))
    X, _ = o.sign_ref(A, opts, S)
    np.testing.assert_allclose(X, np.eye(10), atol=1e-11)
    B = (Q * np.array([1.0, -2.0, 0.5, -0.5, 3.0, -0.2, 0.9, -1.1, 0.3, -0.7])) @ Q.T
    opts5 = o.PrismOpts(d=2, p=4, lo=0.375, tol=0.0, max_iter=5, stall_below=0.0)
    Xs, si = o.sign_ref(B, opts5, S)
    Xp, pi = o.polar_ref(B, opts5, S)
    np.testing.assert_allclose(si[0].alpha, pi[0].alpha, atol=1e-12)
    np.testing.assert_allclose(Xs, Xp, atol=1e-12)


# ---------------------------------------------------------------- apply / step
def test_apply_closed_forms():
    rng = np.random.default_rng(4)
    W, G = rng.standard_normal((5, 3)), rng.standard_normal((5, 3))
    np.testing.assert_allclose(o.apply_ref(W, G, np.eye(5), np.eye(3), 0.1), W - 0.1 * G)
    a, b = rng.uniform(1, 2, 5), rng.uniform(1, 2, 3)
    got = o.apply_ref(W, G, np.diag(a), np.diag(b), 0.01)
    for i in range(5):
        for j in range(3):
            assert got[i, j] == pytest.approx(W[i, j] - 0.01 * a[i] * G[i, j] * b[j], rel=1e-15)


def test_apply_momentum_closed_form():
    """[Shampoo] §5.2 with a constant gradient and identity preconditioners:
    M_t = sum_{i<t} gamma^i G = (1 - gamma^t)/(1 - gamma) G, so after T steps
    W_T = W_0 - lr G sum_{t=1..T} (1 - gamma^t)/(1 - gamma)."""
    rng = np.random.default_rng(5)
    W0, G = rng.standard_normal((4, 6)), rng.standard_normal((4, 6))
    lr, gamma, T = 0.05, 0.9, 5
    W, M = W0, np.zeros_like(W0)
    for _ in range(T):
        W, M, acc = o.apply_variant_ref(W, G, np.eye(4), np.eye(6), lr, M=M, gamma=gamma)
        assert acc is None
    geo = sum((1 - gamma ** t) / (1 - gamma) for t in range(1, T + 1))
    np.testing.assert_allclose(W, W0 - lr * geo * G, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(M, (1 - gamma ** T) / (1 - gamma) * G, rtol=1e-13)
    # gamma = 0 is the plain update
    W1, M1, _ = o.apply_variant_ref(W0, G, np.eye(4), np.eye(6), lr, M=np.ones_like(W0),
                                    gamma=0.0)
    np.testing.assert_allclose(W1, W0 - lr * G, rtol=1e-15)


def test_apply_adaptive_step_closed_form():
    """[Shampoo] §5.1: eta_t = lr / sqrt(1 + sum_{i<=t} ||G_i||^2).  With
    G_t = c_t E (E a unit matrix entry) and identity preconditioners,
    W_T = W_0 - sum_t lr c_t / sqrt(1 + sum_{i<=t} c_i^2) E."""
    W0 = np.zeros((3, 3))
    E = np.zeros((3, 3))
    E[1, 2] = 1.0
    lr, cs = 0.1, [2.0, 0.5, 3.0, 1.0]
    W, acc, want, run = W0, 0.0, 0.0, 0.0
    for c in cs:
        W, M, acc = o.apply_variant_ref(W, c * E, np.eye(3), np.eye(3), lr, acc=acc)
        assert M is None
        run += c * c
        want += lr * c / np.sqrt(1.0 + run)
    assert acc == pytest.approx(sum(c * c for c in cs), rel=1e-15)
    np.testing.assert_allclose(W, -want * E, rtol=1e-14, atol=1e-16)


def test_apply_variants_diagonal_preconditioners():
    """P = PL G PR in that order (diagonal PL, PR: P_ij = a_i G_ij b_j), both
    variants together: a transposed or swapped factor fails this."""
    rng = np.random.default_rng(6)
    m, n, lr, gamma = 5, 3, 0.01, 0.8
    W0, G, M0 = (rng.standard_normal((m, n)) for _ in range(3))
    a, b = rng.uniform(1, 2, m), rng.uniform(1, 2, n)
    acc0 = 2.5
    W, M, acc = o.apply_variant_ref(W0, G, np.diag(a), np.diag(b), lr, M=M0, gamma=gamma,
                                    acc=acc0)
    eta = lr / np.sqrt(1.0 + acc0 + np.sum(G * G))
    for i in range(m):
        for j in range(n):
            mij = gamma * M0[i, j] + a[i] * G[i, j] * b[j]
            assert M[i, j] == pytest.approx(mij, rel=1e-14)
            assert W[i, j] == pytest.approx(W0[i, j] - eta * mij, rel=1e-14)


def test_shampoo_step_vs_eigh():
    rng = np.random.default_rng(8)
    m, n, eps, beta, lr = 16, 8, 1e-6, 0.95, 1e-3
    W = 0.02 * rng.standard_normal((m, n))
    Gs = [0.02 * rng.standard_normal((m, n)) for _ in range(4)]
    opts = o.PrismOpts(d=2, p=4, lo=0.375, tol=1e-13, max_iter=80, stall_below=0.0)
    S = rng.standard_normal((200, n, 4))
    # L is m x m and R is n x n, so each gets a sketch of its own size
    L, R = eps * np.eye(m), eps * np.eye(n)
    for G in Gs:
        L = beta * L + (1 - beta) * G @ G.T + eps * np.eye(m)
        R = beta * R + (1 - beta) * G.T @ G + eps * np.eye(n)
    SL = rng.standard_normal((200, m, 4))
    PL, _ = o.inv_root_ref(L, o.POW_INV4, opts, SL)
    PR, _ = o.inv_root_ref(R, o.POW_INV4, opts, S)
    np.testing.assert_allclose(PL, o.spd_power_eigh(L, -0.25), rtol=1e-8, atol=1e-8 * np.abs(PL).max())
    np.testing.assert_allclose(PR, o.spd_power_eigh(R, -0.25), rtol=1e-8, atol=1e-8 * np.abs(PR).max())
    Wn = o.apply_ref(W, Gs[-1], PL, PR, lr)
    want = W - lr * o.spd_power_eigh(L, -0.25) @ Gs[-1] @ o.spd_power_eigh(R, -0.25)
    np.testing.assert_allclose(Wn - W, want - W, rtol=1e-7, atol=1e-9 * np.abs(want - W).max())


def test_shampoo_step_ref_square():
    rng = np.random.default_rng(18)
    n, eps, beta, lr = 12, 1e-6, 0.95, 1e-3
    W = 0.02 * rng.standard_normal((n, n))
    Gs = [0.02 * rng.standard_normal((n, n)) for _ in range(3)]
    opts = o.PrismOpts(d=2, p=4, lo=0.375, tol=1e-13, max_iter=80, stall_below=0.0)
    S = rng.standard_normal((200, n, 4))
    W1, L, R, PL, PR, infos = o.shampoo_step_ref(W, Gs, eps * np.eye(n), eps * np.eye(n),
                                                 beta, eps, lr, opts, S)
    want = W - lr * o.spd_power_eigh(L, -0.25) @ Gs[-1] @ o.spd_power_eigh(R, -0.25)
    np.testing.assert_allclose(W1 - W, want - W, rtol=1e-7, atol=1e-9 * np.abs(want - W).max())


# ---------------------------------------------------------------- stop rules
def test_stop_rules():
    S = np.random.default_rng(0).standard_normal((10, 4, 2))
    opts = o.PrismOpts(d=1, p=2, lo=0.5, tol=1e-12, max_iter=1)
    B = np.diag([0.5, 0.2, 0.1, 0.9])
    _, _, info = o.coupled_ref(B, opts, S)
    assert info.status == o.ENOCONV and info.iters == 1 and len(info.res) == 2
    Bn = B.copy(); Bn[1, 1] = np.nan
    _, _, info = o.coupled_ref(Bn, opts, S)
    assert info.status == o.ENONFINITE and info.iters == 0
    Y, Z, info = o.coupled_ref(np.eye(4), opts, S)
    assert info.status == o.OK and info.iters == 0 and info.res == [0.0]
    np.testing.assert_array_equal(Y, np.eye(4))


# The stall rule (stop with ESTALL when the previous residual is below
# stall_below and the new one is above stall_ratio times it), pinned on a
# residual sequence worked out by hand.  B = (1 - 0.9) I with Z_0 = I gives
# R_k = xi_k I, so ||R_k||_F / sqrt(n) = xi_k, and a fixed alpha = 1/4 at d = 1
# maps xi to 0.5 xi + 0.4375 xi^2 + 0.0625 xi^3:
#   xi = 0.9, 0.84994, 0.77939, 0.68504, 0.56793, 0.43652
# (successive ratios 0.944, 0.917, 0.879, 0.829, 0.769).
STALL_XI0 = 0.9


@pytest.mark.parametrize("stall_below,stall_ratio,max_iter,status,iters", [
    # the first residual below 0.8 is xi_2; xi_3 / xi_2 = 0.879 > 0.75: stop at k = 3
    # (a rule reading the residual before the previous one would stop at k = 4)
    (0.8, 0.75, 10, o.ESTALL, 3),
    # below 0.9 already at xi_1; xi_2 / xi_1 = 0.917 > 0.75: stop at k = 2
    (0.86, 0.75, 10, o.ESTALL, 2),
    # no ratio exceeds 0.9 once below 0.8: no stall, max_iter ends the pass
    # (a reversed comparison would stop at k = 3)
    (0.8, 0.9, 5, o.ENOCONV, 5),
    # never below 0.5 within 4 steps: no stall
    (0.5, 0.75, 4, o.ENOCONV, 4),
])
def test_stall_rule_on_scalar_residual(stall_below, stall_ratio, max_iter, status, iters):
    n = 4
    opts = o.PrismOpts(d=1, p=2, lo=0.25, hi=1.0, tol=1e-12, max_iter=max_iter,
                       fixed_alpha=True, stall_below=stall_below, stall_ratio=stall_ratio)
    B = (1.0 - STALL_XI0) * np.eye(n)
    _, _, info = o.coupled_ref(B, opts, None)
    assert info.status == status and info.iters == iters, (info.status, info.iters)
    want = [0.9, 0.8499375, 0.7793903636596528, 0.6850442777023162, 0.5679272072594314,
            0.4365241771417045]
    np.testing.assert_allclose(info.res, want[: iters + 1], rtol=1e-12)


# Chebyshev's third-order root-finding step, x <- x - f/f' - f'' f^2 / (2 f'^3)
# (Traub, Iterative Methods for the Solution of Equations, 1964), applied to
# f(x) = x^-2 - a, whose root is a^(-1/2): written here from f and its
# derivatives, not from any polynomial of the oracle.
def chebyshev_inv_sqrt_step(x, a):
    f = x ** -2 - a
    f1 = -2.0 * x ** -3
    f2 = 6.0 * x ** -4
    return x - f / f1 - f2 * f * f / (2.0 * f1 ** 3)


@pytest.mark.parametrize("rotated", [False, True])
def test_chebyshev_is_the_fixed_degree2_taylor_step(rotated):
    """The Chebyshev variant PRISM accelerates is the d = 2 step with the top
    coefficient fixed at its Taylor value 3/8: on B = Q diag(lam) Q^T the
    oracle's Z_k (fixed_alpha, d = 2, lo = 3/8) has eigenvalues that follow
    Chebyshev's step for a^(-1/2), a = lam, from z_0 = 1."""
    n, steps = 6, 5
    lam = np.array([0.9, 0.6, 0.35, 0.2, 0.08, 0.03])
    Q = rot(n, 21) if rotated else np.eye(n)
    B = (Q * lam) @ Q.T
    opts = o.PrismOpts(d=2, p=2, lo=0.375, hi=1.0, tol=0.0, max_iter=steps, fixed_alpha=True,
                       stall_below=0.0)
    _, Z, info = o.coupled_ref(B, opts, None)
    z = np.ones(n)
    for _ in range(steps):
        z = chebyshev_inv_sqrt_step(z, lam)
    np.testing.assert_allclose(Q.T @ Z @ Q, np.diag(z), rtol=1e-12, atol=1e-13)
    assert info.iters == steps and all(a == 0.375 for a in info.alpha)
    # third order: one step maps the residual eigenvalue xi = 1 - lam z^2 to
    # 5/8 xi^3 + 15/64 xi^4 + 9/64 xi^5 (worked out by hand from r = 1 - (1-xi) g^2
    # with g = 1 + xi/2 + 3 xi^2/8: no xi^2 term), and so does the oracle's table
    xi = 1.0 - lam
    xi1 = 1.0 - lam * chebyshev_inv_sqrt_step(np.ones(n), lam) ** 2
    np.testing.assert_allclose(xi1, 5 / 8 * xi ** 3 + 15 / 64 * xi ** 4 + 9 / 64 * xi ** 5,
                               rtol=1e-12)
    np.testing.assert_allclose(o.residual_coeffs(2, 0.375), [0, 0, 0, 5 / 8, 15 / 64, 9 / 64],
                               atol=1e-15)
