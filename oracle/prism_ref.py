"""Float64 CPU oracle for the Shampoo preconditioner step with PRISM-accelerated
Newton-Schulz matrix functions.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module; only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg do.  It shares no code with the CUDA library.

Every function follows one passage of the source pages, cited in its
docstring by page title and section:

* [Shampoo]  "深度学习中的优化器之Shampoo算法原理与二阶优化机制"
  (algorithm.idocdown.com), sections 2.2, 2.3, 3.1, 5.1, 5.2, 6.3.
* [PRISM-it] "Sintesi Tecnica: PRISM" (gist.science), "Parte I" and
  "Parte II" (residual-form iteration, adaptive polynomial, alpha fit,
  clamp, randomized sketch; R_k = I - X_k^2 for sign functions).
* [PRISM-zh] "PRISM：分布无关的自适应矩阵函数计算" (euno.news), "方法论"
  (item 3: adaptive degree selection).

Readings taken where the pages are silent:
* The residual series is the Taylor series of (1 - xi)^(-1/2); the printed
  interval [1/2, 1] for d = 1 fixes its first coefficient at 1/2.
* A^(-1/4) is two nested coupled square-root passes: pass 1 on B = A/||A||_F
  gives Y1 ~ B^(1/2); pass 2 on Y1 gives Z2 ~ Y1^(-1/2) = B^(-1/4).
* The inverse root is stated for symmetric A: a non-symmetric input is
  replaced by its symmetric part, B = (A + A^T) / (2 ||A||_F).
* alpha minimises the sketched objective ||r(R_k; alpha) S_k||_F^2 over
  [lo, hi] (global minimum of a quartic; ties go to the smaller alpha; a
  constant objective gives alpha = lo).
* Sketch slices: pass 1 iteration k uses S[k]; pass 2 iteration k uses
  S[max_iter + k]; the polar iteration k uses S[k].
* The momentum variant follows the recursion the page prints
  (M_t = gamma M_{t-1} + P_t, W -= eta M_t), which is heavy-ball although
  the page calls it Nesterov.
* Stopping: residual ||R_k||_F / sqrt(n) <= tol, checked before the update;
  at most max_iter updates; a non-finite residual stops with ENONFINITE; a
  residual that stops shrinking once small stops with ESTALL.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, textbook special cases, brute force or LAPACK; no
function is "parity unpinned".
"""
from __future__ import annotations

from dataclasses import dataclass, field
from math import comb, sqrt

import numpy as np

# Per-block outcome codes (same numeric values as the C library's report).
OK = 0
ENOCONV = 16
ESTALL = 17
ENONFINITE = 18

POW_INV4 = 0   # A^(-1/4)
POW_INV2 = 1   # A^(-1/2)
POW_SQRT = 2   # A^(1/2)


@dataclass
class PrismOpts:
    """Knobs of one PRISM Newton-Schulz pass.

    d: degree of the update polynomial g_d; p: sketch width; [lo, hi]: alpha
    interval; tol: stop when ||R_k||_F/sqrt(n) <= tol; max_iter: update cap;
    fixed_alpha: use alpha = lo every step (the plain Taylor Newton-Schulz
    baseline); stall_below/stall_ratio: stop with ESTALL when the previous
    residual is below stall_below and the new one is not smaller than
    stall_ratio times it; adaptive_degree: each pass starts at degree 1 and
    raises to d once the sketched degree-1 fit predicts a contraction above
    raise_above (see fit_step).
    """
    d: int = 2
    p: int = 8
    lo: float = 0.375
    hi: float = 1.0
    tol: float = 1e-3
    max_iter: int = 40
    fixed_alpha: bool = False
    stall_below: float = 0.05
    stall_ratio: float = 0.75
    adaptive_degree: bool = False
    raise_above: float = 0.9


@dataclass
class PassInfo:
    alpha: list = field(default_factory=list)
    res: list = field(default_factory=list)
    J_coef: list = field(default_factory=list)
    degree: list = field(default_factory=list)
    iters: int = 0
    status: int = OK


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Shampoo statistics and update  ([Shampoo] §2.2, §2.3, §6.3)
# ---------------------------------------------------------------------------

def gram_ema_ref(G, L, R, beta, eps):
    """One EMA step of the Kronecker factors ([Shampoo] §2.3 step 2):
    L_t = beta L_{t-1} + (1-beta) G G^T + eps I,
    R_t = beta R_{t-1} + (1-beta) G^T G + eps I."""
    G, L, R = _f64(G), _f64(L), _f64(R)
    m, n = G.shape
    L_new = beta * L + (1.0 - beta) * (G @ G.T) + eps * np.eye(m)
    R_new = beta * R + (1.0 - beta) * (G.T @ G) + eps * np.eye(n)
    return L_new, R_new


def apply_ref(W, G, PL, PR, lr):
    """Preconditioned update ([Shampoo] §2.3 step 4):
    W_{t+1} = W_t - lr * L^(-1/4) G R^(-1/4), with PL = L^(-1/4), PR = R^(-1/4)."""
    W, G, PL, PR = _f64(W), _f64(G), _f64(PL), _f64(PR)
    return W - lr * (PL @ G @ PR)


def apply_variant_ref(W, G, PL, PR, lr, M=None, gamma=0.0, acc=None):
    """The update variants of [Shampoo] §5 on P = L^(-1/4) G R^(-1/4):

    §5.1 adaptive step: the running sum of squared gradient norms grows by
    ||G_t||_F^2 and the step is lr / sqrt(1 + that sum), so with `acc` (the
    sum before this step) eta = lr / sqrt(1 + acc + ||G||_F^2);
    §5.2 momentum, in the recursion the page prints: M_t = gamma M_{t-1} + P_t
    and W_{t+1} = W_t - eta M_t.

    Without M the step is W - eta P; without acc, eta = lr.  Returns
    (W, M, acc) after the step (M and acc None when not used)."""
    W, G, PL, PR = _f64(W), _f64(G), _f64(PL), _f64(PR)
    P = PL @ G @ PR
    eta = lr
    if acc is not None:
        acc = float(acc) + float(np.sum(G * G))
        eta = lr / sqrt(1.0 + acc)
    if M is not None:
        M = gamma * _f64(M) + P
        return W - eta * M, M, acc
    return W - eta * P, None, acc


# ---------------------------------------------------------------------------
# Residual-form polynomials  ([PRISM-it] Parte I, Parte II.1)
# ---------------------------------------------------------------------------

def taylor_coeffs(d):
    """Coefficients c_0..c_d of the Taylor series of f(xi) = (1 - xi)^(-1/2)
    about xi = 0: c_j = binom(2j, j) / 4^j  (1, 1/2, 3/8, 5/16, ...)."""
    return np.array([comb(2 * j, j) / 4.0 ** j for j in range(d + 1)], dtype=np.float64)


def g_coeffs(d, alpha):
    """Ascending coefficients of g_d(xi; alpha) = f_{d-1}(xi) + alpha xi^d:
    the degree-d Taylor polynomial with its top coefficient replaced by alpha."""
    c = taylor_coeffs(d).copy()
    c[d] = alpha
    return c


def residual_coeffs(d, alpha):
    """Ascending coefficients of the next residual r(xi; alpha) = 1 - (1-xi) g_d(xi; alpha)^2.

    For the square-root family, one update X <- X g(R) with R = I - X^2 (or
    R = I - Z Y in the coupled form, R = I - X^T X for the polar factor)
    maps an eigenvalue xi of R to r(xi; alpha)."""
    P = np.polynomial.polynomial
    g = g_coeffs(d, alpha)
    r = P.polysub([1.0], P.polymul([1.0, -1.0], P.polymul(g, g)))
    out = np.zeros(2 * d + 2)
    out[: len(r)] = r
    return out


def residual_alpha_table(d):
    """T with r(xi; alpha) = sum_j (T[j,0] + T[j,1] alpha + T[j,2] alpha^2) xi^j.

    Split g = f + alpha xi^d (f = f_{d-1}); then
    r = [1 - (1-xi) f^2] + alpha [-2 (1-xi) xi^d f] + alpha^2 [-(1-xi) xi^(2d)]."""
    P = np.polynomial.polynomial
    f = taylor_coeffs(d)[:d]
    one_minus = np.array([1.0, -1.0])
    xd = np.zeros(d + 1); xd[d] = 1.0
    x2d = np.zeros(2 * d + 1); x2d[2 * d] = 1.0
    parts = [
        P.polysub([1.0], P.polymul(one_minus, P.polymul(f, f))),
        -2.0 * P.polymul(one_minus, P.polymul(xd, f)),
        -1.0 * P.polymul(one_minus, x2d),
    ]
    T = np.zeros((2 * d + 2, 3))
    for a, part in enumerate(parts):
        part = np.trim_zeros(np.asarray(part, dtype=np.float64), "b")
        T[: len(part), a] = part
    return T


def matrix_poly(coeffs, Rk):
    """sum_j coeffs[j] Rk^j by Horner's rule (float64)."""
    n = Rk.shape[0]
    I = np.eye(n)
    acc = coeffs[-1] * I
    for c in coeffs[-2::-1]:
        acc = acc @ Rk + c * I
    return acc


# ---------------------------------------------------------------------------
# Sketched alpha fit  ([PRISM-it] Parte II.1 and II.2; [PRISM-zh] 方法论 2)
# ---------------------------------------------------------------------------

def _argmin_quartic(coef, lo, hi):
    """Global minimiser on [lo, hi] of J(a) = sum_s coef[s] a^s (s = 0..4).

    Candidates: the endpoints and the real roots of J' inside (lo, hi),
    each polished by two Newton steps.  The smallest J wins; values within
    1e-12 (relative) of the best count as ties and go to the smaller alpha."""
    P = np.polynomial.polynomial
    scale = max(np.max(np.abs(coef[1:])), 0.0)
    if scale == 0.0:
        return float(lo)
    dJ = P.polyder(coef)
    d2J = P.polyder(dJ)
    cands = [float(lo), float(hi)]
    for rt in P.polyroots(dJ):
        if abs(rt.imag) > 1e-9 * max(1.0, abs(rt.real)):
            continue
        a = float(rt.real)
        for _ in range(2):
            h = P.polyval(a, d2J)
            if h != 0.0:
                a -= P.polyval(a, dJ) / h
        if lo < a < hi:
            cands.append(a)
    vals = [float(P.polyval(a, coef)) for a in cands]
    best = min(vals)
    thr = best + 1e-12 * max(abs(best), 1e-300)
    return float(min(a for a, v in zip(cands, vals) if v <= thr))


def prism_alpha_ref(Rk, S, d, lo, hi):
    """alpha_k = argmin over [lo, hi] of ||r(R_k; alpha) S||_F^2.

    This is the Gaussian-sketched version of minimising ||I - X_{k+1}^2||_F^2
    (a least-squares fit of g_d to the spectrum of R_k), constrained to
    [lo, hi].  With V_j = R_k^j S and r_j(alpha) the coefficients of
    r(xi; alpha):  J(alpha) = sum_{i,j} r_i(alpha) r_j(alpha) <V_i, V_j>_F,
    and r_j = 0 outside j = d..2d+1.  Returns (alpha, J coefficients a^0..a^4)."""
    Rk, S = _f64(Rk), _f64(S)
    V = [S]
    for _ in range(2 * d + 1):
        V.append(Rk @ V[-1])
    js = list(range(d, 2 * d + 2))
    M = np.array([[np.sum(V[i] * V[j]) for j in js] for i in js])
    T = residual_alpha_table(d)[d: 2 * d + 2]
    coef = np.zeros(5)
    for a in range(3):
        for b in range(3):
            coef[a + b] += T[:, a] @ M @ T[:, b]
    return _argmin_quartic(coef, lo, hi), coef


def fit_step(Rk, Sk, deg, opts: PrismOpts):
    """alpha of one iteration at the current degree, and the degree itself.

    Adaptive degree ([PRISM-zh] 方法论 3: the sketch's residual is monitored
    and the degree raised only when needed): the pass starts at degree 1; the
    degree-1 fit predicts the next sketched residual sqrt(J_1(alpha*)), and
    when its ratio to the current one, ||R_k S_k||_F, exceeds raise_above the
    degree becomes opts.d for this and every later iteration of the pass.
    The interval of degree e is [c_e, hi] with c_e its Taylor coefficient
    (1/2, 3/8), as for the fixed degrees.  Returns (alpha, coef, degree)."""
    if opts.fixed_alpha:
        return float(opts.lo), np.full(5, np.nan), deg
    if not opts.adaptive_degree:
        a, coef = prism_alpha_ref(Rk, Sk, deg, opts.lo, opts.hi)
        return a, coef, deg
    a, coef = prism_alpha_ref(Rk, Sk, deg, taylor_coeffs(deg)[deg], opts.hi)
    if deg < opts.d:
        J = float(np.polynomial.polynomial.polyval(a, coef))
        base = float(np.sum((_f64(Rk) @ _f64(Sk)) ** 2))
        if base > 0.0 and sqrt(max(J, 0.0) / base) > opts.raise_above:
            deg = opts.d
            a, coef = prism_alpha_ref(Rk, Sk, deg, taylor_coeffs(deg)[deg], opts.hi)
    return a, coef, deg


# ---------------------------------------------------------------------------
# Newton-Schulz passes  ([PRISM-it] Parte I: X_{k+1} = X_k f(R_k); [Shampoo] §3.1)
# ---------------------------------------------------------------------------

def _stop(info, rk, k, opts, force=None):
    if force is not None:
        # same-recurrence mode: run exactly `force` updates, ignoring tol/stall
        if k >= force:
            info.status = OK if rk <= opts.tol else ENOCONV
            return True
        return False
    if not np.isfinite(rk):
        info.status = ENONFINITE
        return True
    if rk <= opts.tol:
        info.status = OK
        return True
    if k >= opts.max_iter:
        info.status = ENOCONV
        return True
    if k >= 1:
        prev = info.res[-2]
        if prev < opts.stall_below and rk > opts.stall_ratio * prev:
            info.status = ESTALL
            return True
    return False


def coupled_ref(B, opts: PrismOpts, S, s_offset=0, force_iters=None):
    """Coupled Newton-Schulz square root with PRISM alpha.

    Y_0 = B, Z_0 = I; for k = 0, 1, ...:
        R_k = I - Z_k Y_k;  stop test on ||R_k||_F / sqrt(n);
        alpha_k from the sketch S[s_offset + k];
        g = g_d(R_k; alpha_k);  Y_{k+1} = Y_k g;  Z_{k+1} = g Z_k.
    Y -> B^(1/2), Z -> B^(-1/2) for SPD B with spectrum in (0, 1].
    force_iters: run exactly that many updates (the iteration count another
    implementation took), for same-recurrence comparisons."""
    B = _f64(B)
    n = B.shape[0]
    I = np.eye(n)
    Y, Z = B.copy(), I.copy()
    info = PassInfo()
    deg = 1 if opts.adaptive_degree else opts.d
    k = 0
    while True:
        Rk = I - Z @ Y
        rk = float(np.linalg.norm(Rk) / sqrt(n))
        info.res.append(rk)
        if _stop(info, rk, k, opts, force_iters):
            break
        a, coef, deg = fit_step(Rk, None if S is None else S[s_offset + k], deg, opts)
        info.alpha.append(a)
        info.J_coef.append(coef)
        info.degree.append(deg)
        g = matrix_poly(g_coeffs(deg, a), Rk)
        Y, Z = Y @ g, g @ Z
        k += 1
    info.iters = k
    return Y, Z, info


def inv_root_ref(A, power, opts: PrismOpts, S, force_iters=None):
    """A^(-1/4), A^(-1/2) or A^(1/2) of an SPD matrix by PRISM Newton-Schulz.

    c = ||A||_F (>= lambda_max, so B = A/c has spectrum in (0, 1]);
    the method is stated for a symmetric A, so B is taken as the symmetric
    part (A + A^T) / (2c), which is A / c itself for a symmetric input;
    pass 1: (Y1, Z1) = coupled(B) -> A^(1/2) = sqrt(c) Y1, A^(-1/2) = Z1 / sqrt(c);
    pass 2 (A^(-1/4) only): (Y2, Z2) = coupled(Y1) -> A^(-1/4) = c^(-1/4) Z2.
    force_iters: optional (updates in pass 1, updates in pass 2).
    Returns (X, [PassInfo, ...])."""
    A = _f64(A)
    f1, f2 = (None, None) if force_iters is None else (list(force_iters) + [None])[:2]
    c = np.float64(np.linalg.norm(A))  # numpy arithmetic: c = 0 gives non-finite, not an error
    with np.errstate(divide="ignore", invalid="ignore"):
        B = 0.5 * (A + A.T) / c
    Y1, Z1, i1 = coupled_ref(B, opts, S, 0, f1)
    if power == POW_SQRT:
        return np.sqrt(c) * Y1, [i1]
    if power == POW_INV2:
        return Z1 / np.sqrt(c), [i1]
    Y2, Z2, i2 = coupled_ref(Y1, opts, S, opts.max_iter, f2)
    with np.errstate(divide="ignore", invalid="ignore"):
        return c ** -0.25 * Z2, [i1, i2]


def polar_ref(G, opts: PrismOpts, S, force_iters=None):
    """Polar factor U V^T of G = U Sigma V^T by PRISM Newton-Schulz.

    A wide G (m < n) is handled as G^T.  X_0 = G / ||G||_F; for k = 0, 1, ...:
    R_k = I - X_k^T X_k; stop test; alpha_k from S[k]; X_{k+1} = X_k g_d(R_k; alpha_k)."""
    G = _f64(G)
    wide = G.shape[0] < G.shape[1]
    if wide:
        G = G.T
    n = G.shape[1]
    I = np.eye(n)
    X = G / np.linalg.norm(G)
    info = PassInfo()
    deg = 1 if opts.adaptive_degree else opts.d
    k = 0
    while True:
        Rk = I - X.T @ X
        rk = float(np.linalg.norm(Rk) / sqrt(n))
        info.res.append(rk)
        if _stop(info, rk, k, opts, force_iters):
            break
        a, coef, deg = fit_step(Rk, None if S is None else S[k], deg, opts)
        info.alpha.append(a)
        info.J_coef.append(coef)
        info.degree.append(deg)
        X = X @ matrix_poly(g_coeffs(deg, a), Rk)
        k += 1
    info.iters = k
    return (X.T if wide else X), [info]


def sign_ref(A, opts: PrismOpts, S, force_iters=None):
    """Matrix sign function of a symmetric A by PRISM Newton-Schulz, the
    residual R_k = I - X_k^2 that [PRISM-it] Parte I names for sign functions:
    X_0 = A / ||A||_F; for k = 0, 1, ...: R_k = I - X_k X_k; stop test;
    alpha_k from S[k]; X_{k+1} = X_k g_d(R_k; alpha_k).  The scalar map is
    x -> x (1 - (1 - x^2))^(-1/2) = sign(x), so the same Taylor family and
    alpha objective apply as for the polar factor."""
    A = _f64(A)
    n = A.shape[0]
    I = np.eye(n)
    X = A / np.linalg.norm(A)
    info = PassInfo()
    deg = 1 if opts.adaptive_degree else opts.d
    k = 0
    while True:
        Rk = I - X @ X
        rk = float(np.linalg.norm(Rk) / sqrt(n))
        info.res.append(rk)
        if _stop(info, rk, k, opts, force_iters):
            break
        a, coef, deg = fit_step(Rk, None if S is None else S[k], deg, opts)
        info.alpha.append(a)
        info.J_coef.append(coef)
        info.degree.append(deg)
        X = X @ matrix_poly(g_coeffs(deg, a), Rk)
        k += 1
    info.iters = k
    return X, [info]


# ---------------------------------------------------------------------------
# Exact references  ([Shampoo] §3.1: eigendecomposition; SVD for the polar factor)
# ---------------------------------------------------------------------------

def spd_power_eigh(A, q):
    """A^q = Q diag(lambda^q) Q^T from a symmetric eigendecomposition."""
    w, Q = np.linalg.eigh(_f64(A))
    return (Q * w[None, :] ** q) @ Q.T


def sign_eigh(A):
    """sign(A) = Q diag(sign(lambda)) Q^T from a symmetric eigendecomposition."""
    w, Q = np.linalg.eigh(_f64(A))
    return (Q * np.sign(w)[None, :]) @ Q.T


def polar_svd(G):
    """U V^T from the thin SVD G = U Sigma V^T."""
    U, _, Vt = np.linalg.svd(_f64(G), full_matrices=False)
    return U @ Vt


# ---------------------------------------------------------------------------
# One whole Shampoo step  ([Shampoo] §2.3, §6.3)
# ---------------------------------------------------------------------------

def shampoo_step_ref(W, Gs, L0, R0, beta, eps, lr, opts: PrismOpts, S):
    """EMA over every gradient in Gs, then L^(-1/4), R^(-1/4) by
    :func:`inv_root_ref` (both use the same sketch stack S), then the update
    with the last gradient.  Returns (W_new, L, R, PL, PR, infos)."""
    L, R = _f64(L0), _f64(R0)
    for G in Gs:
        L, R = gram_ema_ref(G, L, R, beta, eps)
    PL, iL = inv_root_ref(L, POW_INV4, opts, S)
    PR, iR = inv_root_ref(R, POW_INV4, opts, S)
    W_new = apply_ref(W, Gs[-1], PL, PR, lr)
    return W_new, L, R, PL, PR, (iL, iR)
