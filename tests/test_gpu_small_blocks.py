"""On-chip small-block path (n <= 64, p <= 16): one CTA per block runs the
whole iteration in shared memory with fp32 products.  Parity with the float64
oracle on the same sketch bytes and iteration counts, ragged sizes, both
degrees, every power, polar in both orientations, and the batched variant of
16384 independent 64 x 64 blocks (sampled blocks against the oracle)."""
import numpy as np
import pytest

from oracle import prism_ref as o
from second_order_optimizer_shampoo_b200 import synth

from helpers import relerr, to_dev, to_host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

POW = {"inv4": (o.POW_INV4, -0.25), "inv2": (o.POW_INV2, -0.5), "sqrt": (o.POW_SQRT, 0.5)}

# fp32 products: the iterate's relative error is a few u_fp32 = 6e-8 per step
# amplified by the conditioning of the root (cond(A)^(1/4) ~ 6 at cond 1e3),
# measured 1e-6 .. 3e-6 when emulated; the bound is 1e-5 as for the fp32-grade
# target of the split path.
TOL_FP32 = 1e-5


def prism():
    from second_order_optimizer_shampoo_b200 import prism as p
    return p


def oracle_opts(opts):
    return o.PrismOpts(d=opts.d, p=opts.p, lo=opts.lo, hi=opts.hi, tol=opts.tol,
                       max_iter=opts.max_iter, fixed_alpha=bool(opts.fixed_alpha),
                       stall_below=opts.stall_below, stall_ratio=opts.stall_ratio)


@pytest.mark.parametrize("n", [4, 36, 60, 64])
@pytest.mark.parametrize("d", [1, 2])
@pytest.mark.parametrize("power", ["inv4", "inv2", "sqrt"])
def test_small_inv_root_parity(n, d, power):
    P = prism()
    batch = 3
    A = synth.spd_batch(n, batch, 1e-3, 1.0, 201)
    p = 4 if d == 1 else 8
    S = synth.sketch_stack(80, n, p, 1201)
    lo = 0.5 if d == 1 else 0.375
    opts = P.make_opts(d=d, p=p, lo=lo, tol=1e-6, max_iter=40, prec="3xtf32")
    X, rep = P.matfn_inv_root(to_dev(torch, A), power, opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    code, q = POW[power]
    for b in range(batch):
        assert rep["status"][b] == o.OK, rep["status"]
        it = rep["iters"][b] if power == "inv4" else rep["iters"][b][:1]
        Xo, infos = o.inv_root_ref(A[b], code, oracle_opts(opts), S, force_iters=it)
        for ps, info in enumerate(infos):
            np.testing.assert_allclose(rep["alpha"][b, ps, :it[ps]], info.alpha, atol=1e-4)
            np.testing.assert_allclose(rep["resid"][b, ps, :it[ps] + 1], info.res, rtol=1e-3,
                                       atol=1e-6)
        assert relerr(X[b], Xo) <= TOL_FP32
        assert relerr(X[b], o.spd_power_eigh(A[b], q)) <= TOL_FP32


def test_small_nonsymmetric_input_takes_symmetric_part():
    """A block that is SPD plus a small antisymmetric part: the on-chip path
    starts from (A + A^T) / (2c) as the oracle does."""
    P = prism()
    n = 40
    A = synth.spd_batch(n, 1, 1e-2, 1.0, 205)
    K = synth.gaussian((n, n), 1e-2, 206)
    A[0] = A[0] + (K - K.T)
    S = synth.sketch_stack(80, n, 8, 1205)
    opts = P.make_opts(d=2, p=8, tol=1e-6, max_iter=40, prec="3xtf32")
    X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    assert rep["status"][0] == o.OK
    Xo, _ = o.inv_root_ref(A[0], o.POW_INV4, oracle_opts(opts), S, force_iters=rep["iters"][0])
    assert relerr(X[0], Xo) <= TOL_FP32
    As = 0.5 * (A[0].astype(np.float64) + A[0].astype(np.float64).T)
    assert relerr(X[0], o.spd_power_eigh(As, -0.25)) <= TOL_FP32


def test_small_sketch_width_16_degree_2():
    """p = 16, d = 2 fills the four sketch slots of one matrix buffer."""
    P = prism()
    n = 64
    # cond 1e3: at cond 1e4 the fp32 residual floor sits near 1e-6 and the
    # stall rule (correctly) ends the pass before tol 1e-6
    A = synth.spd_batch(n, 2, 1e-3, 1.0, 202)
    S = synth.sketch_stack(80, n, 16, 1202)
    opts = P.make_opts(d=2, p=16, tol=1e-6, max_iter=40, prec="3xtf32")
    X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    for b in range(2):
        assert rep["status"][b] == o.OK
        Xo, infos = o.inv_root_ref(A[b], o.POW_INV4, oracle_opts(opts), S,
                                   force_iters=rep["iters"][b])
        for ps, info in enumerate(infos):
            np.testing.assert_allclose(rep["alpha"][b, ps, :rep["iters"][b][ps]], info.alpha,
                                       atol=1e-4)
        assert relerr(X[b], Xo) <= TOL_FP32


def test_small_path_needs_no_workspace():
    P = prism()
    from second_order_optimizer_shampoo_b200 import _abi
    opts = P.make_opts(d=1, p=4)
    assert P.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, 64, 64, 16384, opts) <= 512
    assert P.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, 68, 68, 1, opts) > 512
    assert P.shp_workspace_bytes(_abi.SHP_OP_INV_ROOT, 64, 64, 1, P.make_opts(d=1, p=32)) > 512


@pytest.mark.parametrize("shape", [(64, 32), (32, 64), (48, 48), (64, 8)])
@pytest.mark.parametrize("d", [1, 2])
def test_small_polar_parity(shape, d):
    P = prism()
    m, n = shape
    G = synth.gaussian((2, m, n), 1.0, 203)
    S = synth.sketch_stack(40, min(m, n), 8, 1203)
    lo = 0.5 if d == 1 else 0.375
    opts = P.make_opts(d=d, p=8, lo=lo, tol=1e-6, max_iter=40, prec="3xtf32")
    X, rep = P.matfn_polar(to_dev(torch, G), opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    for b in range(2):
        assert rep["status"][b] == o.OK
        it = rep["iters"][b][0]
        Xo, infos = o.polar_ref(G[b], oracle_opts(opts), S, force_iters=it)
        np.testing.assert_allclose(rep["alpha"][b, 0, :it], infos[0].alpha, atol=1e-4)
        assert relerr(X[b], Xo) <= TOL_FP32
        assert relerr(X[b], o.polar_svd(G[b])) <= TOL_FP32


def test_small_edge_cases():
    """Identity (its root is I), a NaN block next to a good one, and
    max_iter reached: statuses, iteration counts and the last iterate."""
    P = prism()
    n = 32
    good = synth.spd_batch(n, 1, 1e-2, 1.0, 204)[0]
    bad = good.copy()
    bad[1, 2] = np.nan
    A = np.stack([np.eye(n, dtype=np.float32), bad, good])
    S = synth.sketch_stack(40, n, 4, 1204)
    opts = P.make_opts(d=1, p=4, lo=0.5, tol=1e-6, max_iter=20, prec="tf32")
    X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    # ||I||_F = sqrt(n): the iteration runs on B = I / sqrt(n) and the root is I
    assert rep["status"][0] == o.OK
    np.testing.assert_allclose(X[0], np.eye(n), atol=1e-5)
    assert rep["status"][1] == o.ENONFINITE
    assert list(rep["iters"][1]) == [0, 0]
    assert rep["status"][2] == o.OK
    assert relerr(X[2], o.spd_power_eigh(good, -0.25)) <= TOL_FP32
    opts2 = P.make_opts(d=1, p=4, lo=0.5, tol=1e-6, max_iter=3, prec="tf32")
    X2, rep2 = P.matfn_inv_root(to_dev(torch, A[2:]), "inv4", opts2, to_dev(torch, S))
    X2, rep2 = to_host(X2), {k: to_host(v) for k, v in rep2.items()}
    assert rep2["status"][0] == o.ENOCONV
    assert list(rep2["iters"][0]) == [3, 3]
    Xo, infos = o.inv_root_ref(good, o.POW_INV4, oracle_opts(opts2), S)
    assert [i.status for i in infos] == [o.ENOCONV, o.ENOCONV]
    assert relerr(X2[0], Xo) <= TOL_FP32


def test_small_batched_16384_blocks():
    """The batched small-block workload: 16384 independent 64 x 64 blocks
    (config-1 spectrum, d = 1, p = 4, tol 1e-6), every block OK, sampled
    blocks against the oracle with the same iteration counts."""
    P = prism()
    n, batch = 64, 16384
    A = synth.spd_batch(n, batch, 1e-3, 1.0, 101)
    S = synth.sketch_stack(100, n, 4, 1001)
    opts = P.make_opts(d=1, p=4, lo=0.5, tol=1e-6, max_iter=50, prec="3xtf32")
    X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    assert np.all(rep["status"] == o.OK)
    for b in (0, 1, 4095, 8192, batch - 1):
        Xo, _ = o.inv_root_ref(A[b], o.POW_INV4, oracle_opts(opts), S,
                               force_iters=rep["iters"][b])
        assert relerr(X[b], Xo) <= TOL_FP32
        assert relerr(X[b], o.spd_power_eigh(A[b], -0.25)) <= TOL_FP32


@pytest.mark.parametrize("n", [32, 128])
def test_zero_and_indefinite_blocks_are_isolated(n):
    """Faults injected on the host (on chip at n = 32, batched at n = 128): a
    zero block stops with ENONFINITE (0/0 in the normalisation, as the oracle),
    an indefinite block (R_0 has eigenvalues above 1) diverges and stops with
    ENONFINITE or ENOCONV, and the good block between them is unaffected."""
    P = prism()
    good = synth.spd_batch(n, 1, 1e-2, 1.0, 205)[0]
    Q, _ = np.linalg.qr(np.random.default_rng(206).standard_normal((n, n)))
    lam = np.linspace(-1.0, 1.0, n)
    lam[np.abs(lam) < 0.1] = 0.5
    indef = ((Q * lam) @ Q.T).astype(np.float32)
    A = np.stack([np.zeros((n, n), np.float32), good, indef])
    S = synth.sketch_stack(60, n, 4, 1206)
    opts = P.make_opts(d=2, p=4, tol=1e-6, max_iter=30, prec="3xtf32")
    X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    assert rep["status"][0] == o.ENONFINITE
    assert rep["status"][1] == o.OK
    assert rep["status"][2] in (o.ENONFINITE, o.ENOCONV)
    assert relerr(X[1], o.spd_power_eigh(good, -0.25)) <= 3e-5
    _, infos = o.inv_root_ref(A[0], o.POW_INV4, oracle_opts(opts), S)
    assert infos[0].status == o.ENONFINITE
    # polar of a zero block: the same status as the oracle's
    Gz = np.zeros((2, n, n // 2), np.float32)
    Gz[1] = synth.gaussian((n, n // 2), 1.0, 207)
    _, rp = P.matfn_polar(to_dev(torch, Gz), P.make_opts(d=2, p=4, tol=1e-6, max_iter=30,
                                                         prec="3xtf32"),
                          to_dev(torch, synth.sketch_stack(40, n // 2, 4, 1207)))
    assert list(to_host(rp["status"])) == [o.ENONFINITE, o.OK]


def test_polar_varsize_blocks():
    """Blocks of different shapes packed in one buffer, one CTA each: every
    block against the oracle (its sketch = the first min(m, n) rows of each
    64 x p slice) and the SVD; a block with out-of-range dims reports EINVAL
    and leaves its output untouched."""
    P = prism()
    shapes = [(64, 32), (48, 48), (40, 12), (16, 64), (8, 8), (60, 36), (68, 8)]
    blocks = [synth.gaussian(s, 1.0, 208, index=i) for i, s in enumerate(shapes)]
    offs = np.cumsum([0] + [m * n for m, n in shapes])[:-1].astype(np.int64)
    G = np.concatenate([b.ravel() for b in blocks]).astype(np.float32)
    S = synth.sketch_stack(40, 64, 8, 1208)
    opts = P.make_opts(d=2, p=8, tol=1e-6, max_iter=40, prec="3xtf32")
    dims = torch.tensor(shapes, dtype=torch.int32, device="cuda")
    out0 = torch.full((G.size,), 7.0, dtype=torch.float32, device="cuda")
    X, rep = P.matfn_polar_varsize(to_dev(torch, G), dims,
                                   torch.tensor(offs, device="cuda"), opts, to_dev(torch, S),
                                   out=out0)
    X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
    for i, (m, n) in enumerate(shapes):
        Xb = X[offs[i]: offs[i] + m * n].reshape(m, n)
        if m > 64:
            assert rep["status"][i] == 1  # SHP_EINVAL
            assert np.all(Xb == 7.0)
            continue
        assert rep["status"][i] == o.OK, (i, rep["status"])
        it = rep["iters"][i][0]
        k = min(m, n)
        Xo, infos = o.polar_ref(blocks[i], oracle_opts(opts), S[:, :k, :], force_iters=it)
        np.testing.assert_allclose(rep["alpha"][i, 0, :it], infos[0].alpha, atol=1e-4)
        assert relerr(Xb, Xo) <= TOL_FP32
        assert relerr(Xb, o.polar_svd(blocks[i])) <= TOL_FP32
