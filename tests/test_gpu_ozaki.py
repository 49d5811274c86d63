"""The fp64-grade path: Ozaki-scheme products on the int8 tensor cores and
the inverse-root passes with fp64 iterates built on them.

The product is checked element by element against float64 NumPy within the
scheme's error bound; the inverse roots against the float64 oracle run with
the GPU's iteration counts and against the eigendecomposition, at the
split-precision tolerance 1e-5, on spectra of condition 1e6 where fp32
storage cannot get there."""
import numpy as np
import pytest

from oracle import prism_ref as o
from second_order_optimizer_shampoo_b200 import synth

from helpers import relerr, to_dev, to_host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

POW = {"inv4": (o.POW_INV4, -0.25), "inv2": (o.POW_INV2, -0.5), "sqrt": (o.POW_SQRT, 0.5)}

# Error of one Ozaki product (five digit slices per operand, digit pairs of
# weight >= 2^-32 kept).  Row i of A is sigma_i sum_s D_s 2^-8s with
# sigma_i <= 2 max_k|A_ik| / 127 and a representation error of at most
# sigma_i 2^-33; the dropped pairs (weight <= 2^-40, |D| <= 128) add at most
# 4 sigma_i tau_j 2^14 2^-40 + ... per term.  Per term of the K-long sum
# that is below 2^-37 max|A_i.| max|B_.j|, so |C - AB|_ij <= K 2^-37
# max_k|A_ik| max_k|B_kj|, plus the fp64 rounding of the level combination.
def ozaki_bound(A, B):
    K = A.shape[-1]
    return K * 2.0 ** -37 * np.abs(A).max(axis=-1)[..., :, None] * np.abs(B).max(axis=-2)[..., None, :]


def prism():
    from second_order_optimizer_shampoo_b200 import prism as p
    return p


def oracle_opts(opts, **kw):
    base = dict(d=opts.d, p=opts.p, lo=opts.lo, hi=opts.hi, tol=opts.tol, max_iter=opts.max_iter,
                fixed_alpha=bool(opts.fixed_alpha), stall_below=opts.stall_below,
                stall_ratio=opts.stall_ratio, adaptive_degree=bool(opts.adaptive_degree),
                raise_above=opts.raise_above)
    base.update(kw)
    return o.PrismOpts(**base)


@pytest.mark.parametrize("M,N,K,batch", [(200, 292, 300, 2), (1024, 1024, 1024, 2),
                                         (96, 96, 64, 1), (300, 100, 1000, 3)])
def test_matmul_f64_elementwise_bound(M, N, K, batch):
    """Ragged shapes (tiles of 256 x 96, K steps of 64) and rows/columns whose
    magnitudes span 2.6 decades each: every element within the bound."""
    P = prism()
    rng = np.random.default_rng(M + N + K)
    A = rng.standard_normal((batch, M, K)) * np.exp(rng.uniform(-3, 3, (batch, M, 1)))
    B = rng.standard_normal((batch, K, N)) * np.exp(rng.uniform(-3, 3, (batch, 1, N)))
    C = to_host(P.shp_matmul_f64(to_dev(torch, A), to_dev(torch, B)))
    ref = A @ B
    bound = ozaki_bound(A, B) + 8 * 2.0 ** -53 * (np.abs(A) @ np.abs(B))
    assert np.all(np.abs(C - ref) <= bound), float((np.abs(C - ref) / bound).max())
    # typical error (random signs) sits far below the worst case
    assert relerr(C, ref) <= 1e-10


def test_matmul_f64_nan_and_zero_rows():
    """A NaN in row 3 of A reaches row 3 of C only; an all-zero row of A and
    column of B give exact zeros."""
    P = prism()
    rng = np.random.default_rng(7)
    M, N, K = 130, 100, 70
    A = rng.standard_normal((1, M, K))
    B = rng.standard_normal((1, K, N))
    A[0, 3, 5] = np.nan
    A[0, 10, :] = 0.0
    B[0, :, 20] = 0.0
    C = to_host(P.shp_matmul_f64(to_dev(torch, A), to_dev(torch, B)))[0]
    assert np.all(np.isnan(C[3]))
    mask = np.ones(M, bool)
    mask[3] = False
    assert np.all(np.isfinite(C[mask]))
    assert np.all(C[10] == 0.0) and np.all(C[mask, 20] == 0.0)
    ref = A[0] @ B[0]
    assert relerr(C[mask], ref[mask]) <= 1e-10


# Tolerances of the inverse roots.  The fp64 oracle itself ends within
# 5e-6 .. 1e-5 of the eigendecomposition on these spectra (its stopping
# residual), and the Ozaki iteration follows it to about 1e-7 (emulated:
# 7.1e-6 against eigh at n = 1024, cond 1e6, with the oracle's 6.8e-6), so
# the split-precision target 1e-5 applies against the same-recurrence oracle
# and, with the oracle's own distance added, against eigh.
TOL_SAME_RECURRENCE = 1e-5


@pytest.mark.parametrize("power", ["inv4", "inv2", "sqrt"])
@pytest.mark.parametrize("n", [256, 520])
def test_inv_root_ozaki_cond1e6(power, n):
    """cond 1e6 (lambda log-uniform on [1e-6, 1]), d = 2, p = 8, tol 1e-6:
    relative error within 1e-5 of the same-recurrence oracle and of eigh,
    alpha trajectories within 1e-4 of the oracle's."""
    P = prism()
    batch = 2
    A = synth.spd_batch(n, batch, 1e-6, 1.0, 111)
    S = synth.sketch_stack(60, n, 8, 1011)
    opts = P.make_opts(d=2, p=8, tol=1e-6, max_iter=30, prec="ozaki")
    X, rep = P.matfn_inv_root(to_dev(torch, A), power, opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    code, q = POW[power]
    for b in range(batch):
        assert rep["status"][b] in (o.OK, o.ESTALL), rep["status"]
        it = rep["iters"][b] if power == "inv4" else rep["iters"][b][:1]
        Xo, infos = o.inv_root_ref(A[b], code, oracle_opts(opts), S, force_iters=it)
        for ps, info in enumerate(infos):
            np.testing.assert_allclose(rep["alpha"][b, ps, :it[ps]], info.alpha, atol=1e-4)
        assert relerr(X[b], Xo) <= TOL_SAME_RECURRENCE
        ref = o.spd_power_eigh(A[b], q)
        assert relerr(X[b], ref) <= relerr(Xo, ref) + TOL_SAME_RECURRENCE


def test_inv_root_ozaki_d1_and_adaptive_degree():
    """The degree-1 update (Delta = alpha R elementwise) and the adaptive
    degree (masked degree-1 and degree-2 launches) on the fp64 path."""
    P = prism()
    n = 256
    A = synth.spd_batch(n, 2, 1e-4, 1.0, 112)
    S = synth.sketch_stack(80, n, 8, 1012)
    for kw in (dict(d=1), dict(d=2, adaptive_degree=True)):
        opts = P.make_opts(p=8, tol=1e-6, max_iter=40, prec="ozaki", **kw)
        X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
        X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
        for b in range(2):
            assert rep["status"][b] in (o.OK, o.ESTALL)
            it = rep["iters"][b]
            Xo, infos = o.inv_root_ref(A[b], o.POW_INV4, oracle_opts(opts), S, force_iters=it)
            for ps, info in enumerate(infos):
                np.testing.assert_allclose(rep["alpha"][b, ps, :it[ps]], info.alpha, atol=1e-4)
                if opts.adaptive_degree:
                    np.testing.assert_array_equal(rep["degree"][b, ps, :it[ps]], info.degree)
            assert relerr(X[b], Xo) <= TOL_SAME_RECURRENCE


@pytest.mark.parametrize("power", ["inv4", "sqrt"])
def test_inv_root_ozaki_nan_block_isolated(power):
    """A NaN in block 1 stops it with ENONFINITE at its first residual; the
    blocks beside it (and the shared launches) are unaffected."""
    P = prism()
    n = 128
    A = synth.spd_batch(n, 3, 1e-2, 1.0, 113)
    A[1, 5, 7] = np.nan
    S = synth.sketch_stack(60, n, 8, 1013)
    opts = P.make_opts(d=2, p=8, tol=1e-6, max_iter=30, prec="ozaki")
    X, rep = P.matfn_inv_root(to_dev(torch, A), power, opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    code, q = POW[power]
    assert rep["status"][1] == o.ENONFINITE and rep["iters"][1][0] == 0
    for b in (0, 2):
        assert rep["status"][b] in (o.OK, o.ESTALL)
        assert relerr(X[b], o.spd_power_eigh(A[b], q)) <= 1e-5


def test_matmul_f64_reuse_and_accumulate():
    """Slices of a fixed left operand reused against a new right operand, and
    C <- C + A B in place: both as the plain call gives them."""
    P = prism()
    rng = np.random.default_rng(11)
    batch, M, N, K = 2, 160, 96, 200
    A = to_dev(torch, rng.standard_normal((batch, M, K)))
    B1 = to_dev(torch, rng.standard_normal((batch, K, N)))
    B2 = to_dev(torch, rng.standard_normal((batch, K, N)))
    C0 = to_dev(torch, rng.standard_normal((batch, M, N)))
    ws = torch.empty(int(P.A.lib().shp_matmul_f64_workspace_bytes(M, N, K, batch)),
                     dtype=torch.uint8, device="cuda")
    ref1 = to_host(P.shp_matmul_f64(A, B1, ws=ws))
    ref2 = to_host(P.shp_matmul_f64(A, B2))
    got2 = to_host(P.shp_matmul_f64(A, B2, ws=ws, reuse_a=True))  # A's slices from the first call
    np.testing.assert_array_equal(got2, ref2)
    C = C0.clone()
    P.shp_matmul_f64(A, B1, out=C, ws=ws, accumulate=True)
    np.testing.assert_allclose(to_host(C), to_host(C0) + ref1, rtol=0, atol=1e-13 * np.abs(ref1).max())
