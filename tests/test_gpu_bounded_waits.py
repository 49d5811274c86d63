"""Failure detection without a GPU fault: every pipeline wait in the kernels
is bounded, and a wait that runs out must leave an error status the host can
read and a usable context.  shp_selftest_bounded_wait points one wait of a
real launch at a barrier that nothing completes (a short limit, about 10 ms);
the test reads SHP_ETIMEOUT and then checks that ordinary calls afterwards
are still correct: tensor memory was freed, no copy was left in flight, no
sticky CUDA error remains."""
import numpy as np
import pytest

from oracle import prism_ref as o
from second_order_optimizer_shampoo_b200 import synth

from helpers import relerr, to_dev, to_host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ETIMEOUT = 19


def prism():
    from second_order_optimizer_shampoo_b200 import prism as p
    return p


@pytest.mark.parametrize("which", ["gemm", "ozaki", "sketch", "sketch_alpha", "sketch_chain"])
def test_bounded_wait_runs_out_and_the_context_survives(which):
    P = prism()
    status, alpha = P.selftest_bounded_wait(which)
    assert status == ETIMEOUT
    if which.startswith("sketch"):
        assert np.isnan(alpha)  # no fit on the incomplete sketch vectors
    torch.cuda.synchronize()  # raises on a sticky error
    # ordinary work right after, on every kernel family involved
    n = 256
    A = synth.spd_batch(n, 2, 1e-3, 1.0, 141)
    S = synth.sketch_stack(60, n, 8, 1041)
    for prec in ("3xtf32", "ozaki"):
        opts = P.make_opts(d=2, p=8, tol=1e-6, max_iter=30, prec=prec)
        X, rep = P.matfn_inv_root(to_dev(torch, A), "inv4", opts, to_dev(torch, S))
        X, rep = to_host(X), {k: to_host(v) for k, v in rep.items()}
        oo = o.PrismOpts(d=2, p=8, lo=0.375, hi=1.0, tol=1e-6, max_iter=30)
        for b in range(2):
            assert rep["status"][b] in (o.OK, o.ESTALL)
            Xo, _ = o.inv_root_ref(A[b], o.POW_INV4, oo, S, force_iters=rep["iters"][b])
            assert relerr(X[b], Xo) <= (3e-5 if prec == "3xtf32" else 1e-5)


def test_alpha_fit_after_a_sketch_timeout():
    """An ordinary alpha fit right after the sketch's timed-out launch is
    correct (the copies the producer had in flight were drained)."""
    P = prism()
    status, alpha = P.selftest_bounded_wait("sketch")
    assert status == ETIMEOUT and np.isnan(alpha)
    n = 256
    R = synth.gaussian((1, n, n), 0.01, 142)
    R = (R + R.transpose(0, 2, 1)).astype(np.float32)
    S = synth.sketch_stack(1, n, 8, 1042)[0]
    a, _ = P.prism_alpha_fit(to_dev(torch, R), to_dev(torch, S), 2, 0.375, 1.0)
    ar, _ = o.prism_alpha_ref(R[0], S, 2, 0.375, 1.0)
    assert abs(float(to_host(a)[0]) - ar) <= 1e-4
