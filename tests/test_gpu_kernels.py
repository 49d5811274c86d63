"""GPU parity of the single-GEMM entry points and of the alpha fit, element by
element against the float64 oracle, within the forward-error bound of the
arithmetic (tests/helpers.py)."""
import numpy as np
import pytest

from oracle import prism_ref as o
from second_order_optimizer_shampoo_b200 import synth

from helpers import gemm_bound, relerr, to_dev, to_host, U_FP32

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [(128, 128, 1), (300, 196, 2), (64, 512, 1), (4, 4, 3), (516, 260, 1)]


def prism():
    from second_order_optimizer_shampoo_b200 import prism as p
    return p


@pytest.mark.parametrize("prec", ["tf32", "3xtf32"])
@pytest.mark.parametrize("m,n,batch", SHAPES)
def test_gram_ema(prec, m, n, batch):
    beta, eps = 0.95, 1e-3
    G = synth.gaussian((batch, m, n), 1.0, 11)
    L0 = synth.gaussian((batch, m, m), 0.1, 12)
    L0 = (L0 + L0.transpose(0, 2, 1)).astype(np.float32)
    R0 = synth.gaussian((batch, n, n), 0.1, 13)
    R0 = (R0 + R0.transpose(0, 2, 1)).astype(np.float32)
    Ld, Rd = to_dev(torch, L0), to_dev(torch, R0)
    prism().shampoo_gram_ema(to_dev(torch, G), Ld, Rd, beta, eps, prec)
    Lg, Rg = to_host(Ld), to_host(Rd)
    # from 256 on, the products are formed on the upper-triangle tiles and
    # mirrored: off the diagonal tiles the statistics are exactly symmetric,
    # on them to the rounding of the 3xTF32 cross terms
    for X, k in ((Lg, m), (Rg, n)):
        if k >= 256:
            asym = np.abs(X - X.transpose(0, 2, 1))
            assert asym.max() <= 4 * U_FP32 * np.abs(X).max()
            np.testing.assert_array_equal(asym[:, 256:, :256], 0)
    for b in range(batch):
        Lr, Rr = o.gram_ema_ref(G[b], L0[b], R0[b], beta, eps)
        aG = np.abs(G[b].astype(np.float64))
        bl = (1 - beta) * gemm_bound(aG, aG.T, n, prec) + 4 * U_FP32 * (np.abs(Lr) + beta * np.abs(L0[b]))
        br = (1 - beta) * gemm_bound(aG.T, aG, m, prec) + 4 * U_FP32 * (np.abs(Rr) + beta * np.abs(R0[b]))
        assert np.all(np.abs(Lg[b] - Lr) <= bl), np.max(np.abs(Lg[b] - Lr) / bl)
        assert np.all(np.abs(Rg[b] - Rr) <= br), np.max(np.abs(Rg[b] - Rr) / br)


@pytest.mark.parametrize("prec", ["tf32", "3xtf32"])
@pytest.mark.parametrize("m,n,batch,count", [(128, 128, 1, 10), (300, 196, 2, 3), (516, 260, 1, 1),
                                             (1024, 1024, 1, 10)])
def test_gram_ema_steps(prec, m, n, batch, count):
    """count EMA steps in one call against the oracle's one-step recurrence
    applied count times, element by element within the bound of the count
    products (each weighted (1-beta) beta^(count-t)) and of the fp32
    recurrence; and against count one-step GPU calls (same products, only the
    order of the fp32 sums differs)."""
    beta, eps = 0.95, 1e-3
    G = synth.gaussian((count, batch, m, n), 1.0, 31)
    L0 = synth.gaussian((batch, m, m), 0.1, 32)
    L0 = (L0 + L0.transpose(0, 2, 1)).astype(np.float32)
    R0 = synth.gaussian((batch, n, n), 0.1, 33)
    R0 = (R0 + R0.transpose(0, 2, 1)).astype(np.float32)
    P = prism()
    Ld, Rd = to_dev(torch, L0), to_dev(torch, R0)
    P.shampoo_gram_ema_steps(to_dev(torch, G), Ld, Rd, beta, eps, prec)
    Lg, Rg = to_host(Ld), to_host(Rd)
    L1, R1 = to_dev(torch, L0), to_dev(torch, R0)
    for t in range(count):
        P.shampoo_gram_ema(to_dev(torch, G[t]), L1, R1, beta, eps, prec)
    L1, R1 = to_host(L1), to_host(R1)
    for b in range(batch):
        Lr, Rr = L0[b].astype(np.float64), R0[b].astype(np.float64)
        bl = 4 * U_FP32 * count * np.abs(Lr)
        br = 4 * U_FP32 * count * np.abs(Rr)
        for t in range(count):
            Lr, Rr = o.gram_ema_ref(G[t, b], Lr, Rr, beta, eps)
            aG = np.abs(G[t, b].astype(np.float64))
            w = (1 - beta) * beta ** (count - 1 - t)
            bl = bl + w * gemm_bound(aG, aG.T, n, prec)
            br = br + w * gemm_bound(aG.T, aG, m, prec)
        bl = bl + 4 * U_FP32 * count * np.abs(Lr)
        br = br + 4 * U_FP32 * count * np.abs(Rr)
        assert np.all(np.abs(Lg[b] - Lr) <= bl), np.max(np.abs(Lg[b] - Lr) / bl)
        assert np.all(np.abs(Rg[b] - Rr) <= br), np.max(np.abs(Rg[b] - Rr) / br)
        # the one-step calls: identical products, recurrence in another order
        assert np.max(np.abs(Lg[b] - L1[b])) <= 8 * U_FP32 * count * np.abs(Lr).max()
        assert np.max(np.abs(Rg[b] - R1[b])) <= 8 * U_FP32 * count * np.abs(Rr).max()


@pytest.mark.parametrize("prec", ["tf32", "3xtf32"])
@pytest.mark.parametrize("m,n,batch", SHAPES)
def test_apply(prec, m, n, batch):
    lr = 0.1
    W = synth.gaussian((batch, m, n), 0.02, 21)
    G = synth.gaussian((batch, m, n), 0.02, 22)
    PL = synth.gaussian((batch, m, m), 1.0, 23)
    PR = synth.gaussian((batch, n, n), 1.0, 24)
    Wd = to_dev(torch, W)
    prism().shampoo_apply(Wd, to_dev(torch, G), to_dev(torch, PL), to_dev(torch, PR), lr, prec)
    Wg = to_host(Wd)
    for b in range(batch):
        Wr = o.apply_ref(W[b], G[b], PL[b], PR[b], lr)
        aL, aG, aR = (np.abs(x[b].astype(np.float64)) for x in (PL, G, PR))
        # two chained products: |T| <= |PL||G|, errors add through the second GEMM
        bound = lr * (gemm_bound(aL, aG, m, prec) @ aR + gemm_bound(aL @ aG, aR, n, prec))
        bound += 2 * U_FP32 * np.abs(Wr)
        assert np.all(np.abs(Wg[b] - Wr) <= bound), np.max(np.abs(Wg[b] - Wr) / bound)


@pytest.mark.parametrize("variant", ["momentum", "adaptive", "both"])
@pytest.mark.parametrize("prec", ["tf32", "3xtf32"])
@pytest.mark.parametrize("m,n,batch", [(256, 512, 2), (300, 196, 1)])
def test_apply_variants(variant, prec, m, n, batch):
    """Three steps of shampoo_apply_ex against the oracle's update variants
    ([Shampoo] 5.1-5.2): W, the momentum buffer and the running sum of squared
    gradient norms, each within the forward-error bound accumulated over the
    steps (the per-step bound of test_apply on P, carried through
    M = gamma M + P and W -= eta M)."""
    P = prism()
    lr, gamma = 0.05, 0.9
    use_m, use_acc = variant in ("momentum", "both"), variant in ("adaptive", "both")
    W = synth.gaussian((batch, m, n), 0.02, 61)
    PL = synth.gaussian((batch, m, m), 0.1, 62)
    PR = synth.gaussian((batch, n, n), 0.1, 63)
    Gs = [synth.gaussian((batch, m, n), 0.02, 64, index=t) for t in range(3)]
    Wd, PLd, PRd = to_dev(torch, W), to_dev(torch, PL), to_dev(torch, PR)
    Md = torch.zeros_like(Wd) if use_m else None
    accd = torch.full((batch,), 0.25, dtype=torch.float64, device="cuda") if use_acc else None
    for G in Gs:
        P.shampoo_apply_ex(Wd, to_dev(torch, G), PLd, PRd, lr, prec, M=Md, gamma=gamma,
                           gnorm2_acc=accd)
    Wg = to_host(Wd)
    for b in range(batch):
        Wr, Mr, accr = W[b].astype(np.float64), (np.zeros((m, n)) if use_m else None), \
            (0.25 if use_acc else None)
        aL, aR = np.abs(PL[b].astype(np.float64)), np.abs(PR[b].astype(np.float64))
        eW, eM = 2 * U_FP32 * np.abs(Wr), np.zeros((m, n))
        for G in Gs:
            Wr, Mr, accr = o.apply_variant_ref(Wr, G[b], PL[b], PR[b], lr, M=Mr, gamma=gamma,
                                               acc=accr)
            aG = np.abs(G[b].astype(np.float64))
            eP = gemm_bound(aL, aG, m, prec) @ aR + gemm_bound(aL @ aG, aR, n, prec)
            eta = lr / np.sqrt(1 + accr) if use_acc else lr
            step = np.abs(Mr) if use_m else np.abs(o.apply_ref(0 * Wr, G[b], PL[b], PR[b], -1.0))
            if use_m:
                eM = gamma * eM + eP + 2 * U_FP32 * np.abs(Mr)
                eW = eW + eta * (eM + 2 * U_FP32 * step) + 2 * U_FP32 * np.abs(Wr)
            else:
                eW = eW + eta * (eP + 2 * U_FP32 * step) + 2 * U_FP32 * np.abs(Wr)
        assert np.all(np.abs(Wg[b] - Wr) <= eW), np.max(np.abs(Wg[b] - Wr) / eW)
        if use_m:
            Mg = to_host(Md)[b]
            assert np.all(np.abs(Mg - Mr) <= eM), np.max(np.abs(Mg - Mr) / eM)
        if use_acc:
            assert to_host(accd)[b] == pytest.approx(accr, rel=1e-12)


def residual_like(n, batch, seed, lo=0.0, hi=0.8):
    """Symmetric matrices with spectrum in [lo, hi] (a residual R_k mid-iteration)."""
    out = np.empty((batch, n, n), dtype=np.float32)
    for b in range(batch):
        g = np.random.default_rng((seed, b))
        Q, _ = np.linalg.qr(g.standard_normal((n, n)))
        lam = g.uniform(lo, hi, n)
        out[b] = ((Q * lam) @ Q.T).astype(np.float32)
    return out


@pytest.mark.parametrize("d", [1, 2])
@pytest.mark.parametrize("p", [1, 4, 8, 16, 32])
@pytest.mark.parametrize("n", [64, 260])
def test_alpha_fit(d, p, n):
    batch = 3
    R = residual_like(n, batch, 31 + p + n)
    R[2] = (R[2] * -0.5).astype(np.float32)  # a residual with negative spectrum (overshoot)
    S = synth.sketch_stack(1, n, p, 41)[0]
    lo, hi = (0.5, 1.0) if d == 1 else (0.375, 1.0)
    a, J = prism().prism_alpha_fit(to_dev(torch, R), to_dev(torch, S), d, lo, hi)
    a, J = to_host(a), to_host(J)
    for b in range(batch):
        ar, Jr = o.prism_alpha_ref(R[b], S, d, lo, hi)
        assert abs(a[b] - ar) <= 1e-4, (b, a[b], ar)
        assert np.max(np.abs(J[b] - Jr)) <= 1e-4 * np.max(np.abs(Jr)), (J[b], Jr)


def test_alpha_fit_interior_values_and_clamps():
    # R = xi I gives the closed-form alpha; both an interior value and a clamp
    n, p = 128, 8
    S = synth.sketch_stack(1, n, p, 5)[0]
    R = np.stack([0.5 * np.eye(n), 0.75 * np.eye(n), -0.5 * np.eye(n)]).astype(np.float32)
    a, _ = prism().prism_alpha_fit(to_dev(torch, R), to_dev(torch, S), 1, 0.5, 1.0)
    a = to_host(a)
    assert a[0] == pytest.approx(2 * np.sqrt(2) - 2, abs=1e-5)
    assert a[1] == pytest.approx(1.0, abs=1e-6)
    assert a[2] == pytest.approx(0.5, abs=1e-6)
