"""prism_alpha_fit_noalloc: the alpha fit for callers that cannot allocate
device memory mid-step (their framework's caching allocator owns the free
memory, or they cannot take the device-wide synchronisation of
cudaMalloc/cudaFree).  It must give the same alphas and J coefficients as the
workspace-based prism_alpha_fit, call after call, although every call reuses
the same library-owned scratch array.  Called through the C ABI directly."""
import ctypes

import numpy as np
import pytest

from oracle import prism_ref as o
from second_order_optimizer_shampoo_b200 import _abi as A
from second_order_optimizer_shampoo_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def residuals(n, batch, seed):
    out = np.empty((batch, n, n), dtype=np.float32)
    for b in range(batch):
        g = np.random.default_rng((seed, b))
        Q, _ = np.linalg.qr(g.standard_normal((n, n)))
        out[b] = ((Q * g.uniform(0.0, 0.8, n)) @ Q.T).astype(np.float32)
    return out


def noalloc_fit(Rd, Sd, d, lo, hi):
    batch, n = Rd.shape[0], Rd.shape[-1]
    alpha = torch.full((batch,), float("nan"), dtype=torch.float32, device=Rd.device)
    J = torch.full((batch, 5), float("nan"), dtype=torch.float64, device=Rd.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = A.lib().prism_alpha_fit_noalloc(ctypes.c_void_p(Rd.data_ptr()), n, batch,
                                         ctypes.c_void_p(Sd.data_ptr()), Sd.shape[-1], d, lo, hi,
                                         ctypes.c_void_p(alpha.data_ptr()),
                                         ctypes.c_void_p(J.data_ptr()), stream)
    assert rc == A.SHP_OK, rc
    return alpha.cpu().numpy(), J.cpu().numpy()


@pytest.mark.parametrize("d,p,n,batch", [(2, 8, 1024, 3), (1, 4, 260, 5)])
def test_noalloc_matches_workspace_entry_point(d, p, n, batch):
    from second_order_optimizer_shampoo_b200 import prism
    lo, hi = (0.5, 1.0) if d == 1 else (0.375, 1.0)
    for call in range(2):  # two calls in a row share the scratch array
        R = residuals(n, batch, 70 + call)
        S = synth.sketch_stack(1, n, p, 80 + call)[0]
        Rd, Sd = torch.from_numpy(R).cuda(), torch.from_numpy(S).cuda()
        a_ws, J_ws = prism.prism_alpha_fit(Rd, Sd, d, lo, hi)
        a_na, J_na = noalloc_fit(Rd, Sd, d, lo, hi)
        a_ws, J_ws = a_ws.cpu().numpy(), J_ws.cpu().numpy()
        np.testing.assert_allclose(a_na, a_ws, atol=1e-4)
        np.testing.assert_allclose(J_na, J_ws, rtol=1e-4, atol=1e-4 * np.abs(J_ws).max())
        for b in range(batch):  # and both agree with the oracle
            ar, _ = o.prism_alpha_ref(R[b], S, d, lo, hi)
            assert abs(a_na[b] - ar) <= 1e-4


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """The scratch holds (2d+2) n p floats of sketch vectors and one timeout
    flag per block: the largest batch that fits runs, one more is refused
    before any launch."""
    n, p, d = 1024, 8, 2
    per_block = ((2 * d + 2) * n * p + 1) * 4
    fits = A.SHP_NOALLOC_SCRATCH_BYTES // per_block
    Rd = torch.zeros(fits + 1, n, n, device="cuda")
    Sd = torch.zeros(n, p, device="cuda")
    out = torch.zeros(fits + 1, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for batch, want in ((fits + 1, A.SHP_EUNSUPPORTED), (fits, A.SHP_OK)):
        rc = A.lib().prism_alpha_fit_noalloc(ctypes.c_void_p(Rd.data_ptr()), n, batch,
                                             ctypes.c_void_p(Sd.data_ptr()), p, d, 0.375, 1.0,
                                             ctypes.c_void_p(out.data_ptr()), None, stream)
        assert rc == want, (batch, rc)
    # R = 0 makes J constant: every block takes the lower end of the interval
    np.testing.assert_array_equal(out[:fits].cpu().numpy(), np.float32(0.375))
