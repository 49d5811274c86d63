"""The five workloads at their full sizes, in the launch configuration the
benchmark uses, checked on outputs the oracle can compute (sampled blocks) or
on properties that hold at any size."""
import numpy as np
import pytest

from oracle import prism_ref as o
from second_order_optimizer_shampoo_b200 import synth

from helpers import bf16_to_dev, relerr, to_dev, to_host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def prism():
    from second_order_optimizer_shampoo_b200 import prism as p
    return p


def oracle_opts(opts):
    return o.PrismOpts(d=opts.d, p=opts.p, lo=opts.lo, hi=opts.hi, tol=opts.tol,
                       max_iter=opts.max_iter, stall_below=opts.stall_below,
                       stall_ratio=opts.stall_ratio)


def test_config2_shampoo_step():
    """One Shampoo step on a 1024 x 1024 weight: 10 EMA steps (fresh G), both
    inverse 4th roots (TF32, d = 2, p = 8), then the update.  TF32 target 1e-3."""
    P = prism()
    n, beta, eps, lr = 1024, 0.95, 1e-6, 1e-3
    W = synth.gaussian((1, n, n), 0.02, 102, index=0)
    Gs = [synth.gaussian((1, n, n), 0.02, 102, index=t + 1) for t in range(10)]
    L = torch.full((1, n, n), 0.0, device="cuda")
    L[0].fill_diagonal_(eps)
    R = L.clone()
    for G in Gs:
        P.shampoo_gram_ema(to_dev(torch, G), L, R, beta, eps, "tf32")
    S = synth.sketch_stack(60, n, 8, 1002)
    opts = P.make_opts(d=2, p=8, tol=1e-3, max_iter=30, prec="tf32")
    LR = torch.cat([L, R])
    roots, rep = P.matfn_inv_root(LR, "inv4", opts, to_dev(torch, S))
    Wd = to_dev(torch, W)
    P.shampoo_apply(Wd, to_dev(torch, Gs[-1]), roots[0:1].contiguous(), roots[1:2].contiguous(),
                    lr, "tf32")
    status = to_host(rep["status"])
    assert all(s in (o.OK, o.ESTALL) for s in status), status
    # oracle: the same step in float64
    Lr, Rr = eps * np.eye(n), eps * np.eye(n)
    for G in Gs:
        Lr, Rr = o.gram_ema_ref(G[0], Lr, Rr, beta, eps)
    assert relerr(to_host(L)[0], Lr) <= 1e-3 and relerr(to_host(R)[0], Rr) <= 1e-3
    PL, PR = o.spd_power_eigh(Lr, -0.25), o.spd_power_eigh(Rr, -0.25)
    rt = to_host(roots)
    assert relerr(rt[0], PL) <= 1e-3
    assert relerr(rt[1], PR) <= 1e-3
    dW_ref = o.apply_ref(W[0], Gs[-1][0], PL, PR, lr) - W[0]
    dW = to_host(Wd)[0].astype(np.float64) - W[0]
    assert relerr(dW, dW_ref) <= 1e-3


def subspace_err(X, A, frac=1e-2):
    """Relative error of X against A^(-1/4) restricted to the eigenvectors
    with lambda >= frac * lambda_max (components TF32/fp32 products keep)."""
    w, Q = np.linalg.eigh(A.astype(np.float64))
    Xe = (Q * w ** -0.25) @ Q.T
    Pk = Q[:, w >= frac * w.max()]
    return relerr(X @ Pk, Xe @ Pk), relerr(X, Xe)


def test_config3_batched_inverse_root():
    """64 SPD blocks 1024^2, cond 1e6, d = 2, p = 8, tol 1e-3 per pass, split
    path (TF32 rounding of A/||A|| makes these blocks indefinite).  Sampled
    blocks against the oracle; alpha parity on identical residuals."""
    P = prism()
    n, batch = 1024, 64
    A = synth.spd_batch(n, batch, 1e-6, 1.0, 103)
    S = synth.sketch_stack(48, n, 8, 1003)
    opts = P.make_opts(d=2, p=8, tol=1e-3, max_iter=24, prec="3xtf32")
    X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    assert np.all(rep["status"] == o.OK), rep["status"]
    assert np.all(rep["resid"][np.arange(batch), 0, rep["iters"][:, 0]] <= 1e-3)
    for b in (0, 1, batch // 2, batch - 1):
        _, free = o.inv_root_ref(A[b], o.POW_INV4, oracle_opts(opts), S)
        assert all(abs(f.iters - int(g)) <= 1 for f, g in zip(free, rep["iters"][b]))
        sub, full = subspace_err(X[b], A[b])
        assert sub <= 1e-3, (b, sub, full)
        assert full <= 1e-1, (b, sub, full)
    # alpha on identical residuals: the oracle's R_k of block 0, rounded to fp32
    B0 = A[0].astype(np.float64) / np.linalg.norm(A[0].astype(np.float64))
    Y, Z = B0.copy(), np.eye(n)
    Rs, Ss = [], []
    for k in range(4):
        Rk = np.eye(n) - Z @ Y
        Rs.append(Rk.astype(np.float32))
        Ss.append(S[k])
        a, _ = o.prism_alpha_ref(Rk, S[k], 2, 0.375, 1.0)
        g = o.matrix_poly(o.g_coeffs(2, a), Rk)
        Y, Z = Y @ g, g @ Z
    for Rk, Sk in zip(Rs, Ss):
        ag, _ = P.prism_alpha_fit(to_dev(torch, Rk[None]), to_dev(torch, Sk), 2, 0.375, 1.0)
        ar, _ = o.prism_alpha_ref(Rk, Sk, 2, 0.375, 1.0)
        assert abs(float(to_host(ag)[0]) - ar) <= 1e-4


def test_config4_polar_bf16():
    """96 matrices 4096 x 1024, rank-64 signal + 0.01 noise, bf16 storage,
    d = 2, p = 8, until ||I - X^T X||_F / sqrt(n) <= 1e-2.  bf16 rounding of
    the iterate scrambles the noise subspace, so the check is the residual and
    the error on the 64-dimensional signal subspace."""
    P = prism()
    m, n, batch, r = 4096, 1024, 96, 64
    bits, G16 = synth.lowrank_noise_batch(m, n, r, 0.01, batch, 104)
    S = synth.sketch_stack(40, n, 8, 1004)
    opts = P.make_opts(d=2, p=8, tol=1e-2, max_iter=40, prec="bf16")
    X, rep = P.matfn_polar(bf16_to_dev(torch, bits), opts, to_dev(torch, S))
    rep = {k: to_host(v) for k, v in rep.items()}
    assert np.all(rep["status"] == o.OK), rep["status"]
    for b in (0, 1, batch // 2, batch - 1):
        Xb = to_host(X[b]).astype(np.float64)
        res = np.linalg.norm(np.eye(n) - Xb.T @ Xb) / np.sqrt(n)
        assert res <= 1e-2 + 2 ** -8, res   # + the bf16 rounding of the stored output
        U, s, Vt = np.linalg.svd(G16[b].astype(np.float64), full_matrices=False)
        V64 = Vt[:r].T
        sig = np.linalg.norm((Xb - U @ Vt) @ V64) / np.sqrt(r)
        assert sig <= 1e-2, sig
    # alpha on identical residuals (R_0 of two sampled inputs, fp32)
    for b in (0, batch - 1):
        X0 = G16[b].astype(np.float64) / np.linalg.norm(G16[b].astype(np.float64))
        R0 = (np.eye(n) - X0.T @ X0).astype(np.float32)
        ag, _ = P.prism_alpha_fit(to_dev(torch, R0[None]), to_dev(torch, S[0]), 2, 0.375, 1.0)
        ar, _ = o.prism_alpha_ref(R0, S[0], 2, 0.375, 1.0)
        assert abs(float(to_host(ag)[0]) - ar) <= 1e-4


# The tensor cores add into their fp32 accumulator with truncation: measured on
# all-positive products, one fp32-grade (3xTF32) product of length K is biased
# by about -(K/8) 2^-25 (the hi*hi accumulator takes K/8 truncating additions).
# At K = 10240 that is 3.8e-5, so the split path's bound on the full-size
# square root is 1e-4 (the 1e-5 target holds at n = 1024, where K/8 2^-25 =
# 3.8e-6).
TOL_3X_K10240 = 1e-4


@pytest.mark.parametrize("n,samples", [(1024, 2048), (10240, 20480)])
def test_config5_square_root(n, samples):
    """A = X X^T / samples + 1e-4 I (Marchenko-Pastur, ratio 1/2), A^(1/2) by
    d = 2, p = 16, split path, tol 1e-6.  At n = 1024 the whole result is
    compared with eigh (1e-5); at n = 10240 sampled entries of X X against A
    and the symmetry of X, within the bound the accumulation allows there."""
    P = prism()
    A = synth.mp_spd(n, samples, 1e-4, 105)
    S = synth.sketch_stack(40, n, 16, 1005)
    opts = P.make_opts(d=2, p=16, tol=1e-6, max_iter=40, prec="3xtf32")
    Xd, rep = P.matfn_inv_root(to_dev(torch, A[None]), "sqrt", opts, to_dev(torch, S))
    rep = {k: to_host(v) for k, v in rep.items()}
    assert rep["status"][0] in (o.OK, o.ESTALL), rep
    X = to_host(Xd)[0].astype(np.float64)
    if n <= 2048:
        assert relerr(X, o.spd_power_eigh(A, 0.5)) <= 1e-5
        Xo, infos = o.inv_root_ref(A, o.POW_SQRT, oracle_opts(opts), S,
                                   force_iters=rep["iters"][0][:1])
        assert relerr(X, Xo) <= 1e-5
        return
    rng = np.random.default_rng(0)
    I = rng.integers(0, n, 64)
    J = rng.integers(0, n, 64)
    A64 = A.astype(np.float64)
    XX = np.einsum("ik,ki->i", X[I, :], X[:, J])
    scale = np.einsum("ik,ki->i", np.abs(X[I, :]), np.abs(X[:, J]))
    # |X^2 - A| <= 2 delta |X||X| for a relative error delta of X
    assert np.all(np.abs(XX - A64[I, J]) <= 2 * TOL_3X_K10240 * scale + 1e-7)
    assert relerr(X[I], X[:, I].T) <= TOL_3X_K10240   # the true root is symmetric
