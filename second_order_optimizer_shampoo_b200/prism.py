"""Python binding of the C ABI (argument marshalling only).

Each function takes CUDA tensors, allocates the scratch buffer the library
asks for through PyTorch's allocator, and calls the entry point of the same
name on the current stream.  Every arithmetic step runs in the library's
kernels; there is no CPU path.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi as A

_PREC = {"tf32": A.SHP_TF32, "3xtf32": A.SHP_3XTF32, "bf16": A.SHP_BF16, "ozaki": A.SHP_OZAKI}
_POW = {"inv4": A.SHP_POW_INV4, "inv2": A.SHP_POW_INV2, "sqrt": A.SHP_POW_SQRT}


def status_string(code: int) -> str:
    return A.lib().shp_status_string(int(code)).decode()


def version() -> str:
    return A.lib().shp_version().decode()


def _check(code: int, name: str):
    if code != A.SHP_OK:
        extra = ""
        if code == A.SHP_ECUDA:
            extra = f", {A.lib().shp_last_cuda_error().decode()}"
        raise RuntimeError(f"{name} failed: {status_string(code)} ({code}{extra})")


def _dev(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device (the library has no CPU path)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def make_opts(d=2, p=8, lo=None, hi=1.0, tol=1e-3, max_iter=40, prec="3xtf32",
              fixed_alpha=False, stall_below=0.05, stall_ratio=0.75, adaptive_degree=False,
              raise_above=0.9, host_loop=False) -> A.PrismOpts:
    if lo is None:
        lo = 0.5 if d == 1 else 0.375
    return A.PrismOpts(d, p, lo, hi, tol, max_iter, _PREC[prec] if isinstance(prec, str) else prec,
                       int(bool(fixed_alpha)), stall_below, stall_ratio,
                       int(bool(adaptive_degree)), raise_above, int(bool(host_loop)))


def shp_workspace_bytes(op: int, m: int, n: int, batch: int, opts: A.PrismOpts | None = None) -> int:
    return int(A.lib().shp_workspace_bytes(op, m, n, batch,
                                           ctypes.byref(opts) if opts is not None else None))


def _ws(nbytes: int, device):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def _as3(t, rows, cols):
    return t.reshape(-1, rows, cols)


def shampoo_gram_ema(G, L, R, beta: float, eps: float, prec: str = "tf32", ws=None):
    """L <- beta L + (1-beta) G G^T + eps I ; R <- beta R + (1-beta) G^T G + eps I (in place)."""
    _dev(G, L, R)
    m, n = G.shape[-2], G.shape[-1]
    batch = G.numel() // (m * n)
    o = make_opts(prec=prec)
    need = shp_workspace_bytes(A.SHP_OP_GRAM_EMA, m, n, batch, o)
    ws = _ws(need, G.device) if ws is None else ws
    _check(A.lib().shampoo_gram_ema(_p(G), m, n, batch, _p(L), _p(R), beta, eps, _PREC[prec],
                                    _p(ws), ws.numel(), _stream()), "shampoo_gram_ema")


def shampoo_gram_ema_steps(G, L, R, beta: float, eps: float, prec: str = "tf32", ws=None):
    """count successive EMA steps, one per gradient of G: [count][batch][m][n]
    (or [count][m][n]): L <- beta L + (1-beta) G_t G_t^T + eps I and
    R <- beta R + (1-beta) G_t^T G_t + eps I for t = 1..count (in place)."""
    _dev(G, L, R)
    m, n = G.shape[-2], G.shape[-1]
    count = G.shape[0]
    batch = G.numel() // (count * m * n)
    o = make_opts(prec=prec)
    need = shp_workspace_bytes(A.SHP_OP_GRAM_EMA_STEPS, m, n, count * batch, o)
    ws = _ws(need, G.device) if ws is None else ws
    _check(A.lib().shampoo_gram_ema_steps(_p(G), count, m, n, batch, _p(L), _p(R), beta, eps,
                                          _PREC[prec], _p(ws), ws.numel(), _stream()),
           "shampoo_gram_ema_steps")


def shampoo_apply(W, G, Lroot, Rroot, lr: float, prec: str = "tf32", ws=None):
    """W <- W - lr * Lroot G Rroot (in place)."""
    _dev(W, G, Lroot, Rroot)
    m, n = W.shape[-2], W.shape[-1]
    batch = W.numel() // (m * n)
    o = make_opts(prec=prec)
    need = shp_workspace_bytes(A.SHP_OP_APPLY, m, n, batch, o)
    ws = _ws(need, W.device) if ws is None else ws
    _check(A.lib().shampoo_apply(_p(W), _p(G), _p(Lroot), _p(Rroot), m, n, batch, lr, _PREC[prec],
                                 _p(ws), ws.numel(), _stream()), "shampoo_apply")


def shampoo_apply_ex(W, G, Lroot, Rroot, lr: float, prec: str = "tf32", M=None, gamma=0.0,
                     gnorm2_acc=None, ws=None):
    """Update variants (in place): with gnorm2_acc (float64 [batch]) the step is
    lr / sqrt(1 + acc) after acc += ||G||_F^2; with M (momentum buffer)
    M <- gamma M + P and W <- W - eta M; P = Lroot G Rroot."""
    _dev(W, G, Lroot, Rroot, M, gnorm2_acc)
    if gnorm2_acc is not None and gnorm2_acc.dtype != torch.float64:
        raise ValueError("gnorm2_acc must be float64")
    m, n = W.shape[-2], W.shape[-1]
    batch = W.numel() // (m * n)
    o = make_opts(prec=prec)
    need = shp_workspace_bytes(A.SHP_OP_APPLY, m, n, batch, o)
    ws = _ws(need, W.device) if ws is None else ws
    _check(A.lib().shampoo_apply_ex(_p(W), _p(M), _p(gnorm2_acc), _p(G), _p(Lroot), _p(Rroot),
                                    m, n, batch, lr, gamma, _PREC[prec], _p(ws), ws.numel(),
                                    _stream()), "shampoo_apply_ex")


def _report(batch, max_iter, device):
    return {
        "status": torch.full((batch,), -1, dtype=torch.int32, device=device),
        "iters": torch.full((batch, 2), -1, dtype=torch.int32, device=device),
        "resid": torch.full((batch, 2, max_iter + 1), float("nan"), dtype=torch.float32, device=device),
        "alpha": torch.full((batch, 2, max_iter), float("nan"), dtype=torch.float32, device=device),
        "degree": torch.full((batch, 2, max_iter), -1, dtype=torch.int32, device=device),
    }


def _report_struct(rep):
    if rep is None:
        return None
    deg = rep.get("degree")
    return ctypes.byref(A.PrismReport(rep["status"].data_ptr(), rep["iters"].data_ptr(),
                                      rep["resid"].data_ptr(), rep["alpha"].data_ptr(),
                                      deg.data_ptr() if deg is not None else None))


def make_report(batch, max_iter, device):
    """Device tensors for the per-block trajectory (status, iters, resid, alpha,
    degree)."""
    return _report(batch, max_iter, device)


def matfn_inv_root(Amat, power="inv4", opts: A.PrismOpts | None = None, S=None, out=None,
                   report=True, ws=None):
    """A^(-1/4) (or A^(-1/2), A^(1/2)) of a batch of SPD matrices.

    report: True (fresh tensors), False, or a dict from make_report() to reuse;
    the library caches one CUDA graph per distinct set of pointers and sizes,
    so reusing out/ws/report buffers keeps repeated calls on the cached graph."""
    opts = opts or make_opts()
    _dev(Amat, S, out)
    n = Amat.shape[-1]
    batch = Amat.numel() // (n * n)
    out = torch.empty_like(Amat) if out is None else out
    rep = report if isinstance(report, dict) else (
        _report(batch, opts.max_iter, Amat.device) if report else None)
    need = shp_workspace_bytes(A.SHP_OP_INV_ROOT, n, n, batch, opts)
    ws = _ws(need, Amat.device) if ws is None else ws
    s_count = 0 if S is None else S.shape[0]
    _check(A.lib().matfn_inv_root(_p(Amat), n, batch, _POW[power], ctypes.byref(opts), _p(S),
                                  s_count, _p(out), _report_struct(rep), _p(ws), ws.numel(),
                                  _stream()), "matfn_inv_root")
    return out, rep


def matfn_polar(G, opts: A.PrismOpts | None = None, S=None, out=None, report=True, ws=None):
    """Polar factor of a batch of m x n matrices; bf16 input keeps bf16 storage."""
    opts = opts or make_opts()
    _dev(G, S, out)
    m, n = G.shape[-2], G.shape[-1]
    batch = G.numel() // (m * n)
    if G.dtype == torch.bfloat16:
        storage = A.SHP_BF16
    elif G.dtype == torch.float32:
        storage = opts.prec if opts.prec in (A.SHP_TF32, A.SHP_3XTF32) else A.SHP_TF32
    else:
        raise ValueError("G must be float32 or bfloat16")
    out = torch.empty_like(G) if out is None else out
    rep = report if isinstance(report, dict) else (
        _report(batch, opts.max_iter, G.device) if report else None)
    o2 = A.PrismOpts.from_buffer_copy(opts)
    o2.prec = storage
    need = shp_workspace_bytes(A.SHP_OP_POLAR, m, n, batch, o2)
    ws = _ws(need, G.device) if ws is None else ws
    s_count = 0 if S is None else S.shape[0]
    _check(A.lib().matfn_polar(_p(G), storage, m, n, batch, ctypes.byref(opts), _p(S), s_count,
                               _p(out), _report_struct(rep), _p(ws), ws.numel(), _stream()),
           "matfn_polar")
    return out, rep


def matfn_polar_varsize(G, dims, offsets, opts: A.PrismOpts | None = None, S=None, out=None,
                        report=True):
    """Polar factors of small blocks of different shapes packed in the fp32
    tensor G: block b is dims[b] = (m_b, n_b) at element offsets[b] (dims int32
    [batch, 2], offsets int64 [batch], both on the device)."""
    opts = opts or make_opts()
    _dev(G, dims, offsets, S, out)
    if G.dtype != torch.float32 or dims.dtype != torch.int32 or offsets.dtype != torch.int64:
        raise ValueError("G float32, dims int32, offsets int64")
    batch = dims.shape[0]
    out = torch.empty_like(G) if out is None else out
    rep = report if isinstance(report, dict) else (
        _report(batch, opts.max_iter, G.device) if report else None)
    s_count = 0 if S is None else S.shape[0]
    _check(A.lib().matfn_polar_varsize(_p(G), _p(dims), _p(offsets), batch, ctypes.byref(opts),
                                       _p(S), s_count, _p(out), _report_struct(rep), _stream()),
           "matfn_polar_varsize")
    return out, rep


def matfn_sign(Amat, opts: A.PrismOpts | None = None, S=None, out=None, report=True, ws=None):
    """Matrix sign function of a batch of symmetric n x n matrices (bf16 input
    keeps bf16 storage)."""
    opts = opts or make_opts()
    _dev(Amat, S, out)
    n = Amat.shape[-1]
    if Amat.shape[-2] != n:
        raise ValueError("matfn_sign needs square matrices")
    batch = Amat.numel() // (n * n)
    if Amat.dtype == torch.bfloat16:
        storage = A.SHP_BF16
    elif Amat.dtype == torch.float32:
        storage = opts.prec if opts.prec in (A.SHP_TF32, A.SHP_3XTF32) else A.SHP_TF32
    else:
        raise ValueError("A must be float32 or bfloat16")
    out = torch.empty_like(Amat) if out is None else out
    rep = report if isinstance(report, dict) else (
        _report(batch, opts.max_iter, Amat.device) if report else None)
    o2 = A.PrismOpts.from_buffer_copy(opts)
    o2.prec = storage
    need = shp_workspace_bytes(A.SHP_OP_POLAR, n, n, batch, o2)
    ws = _ws(need, Amat.device) if ws is None else ws
    s_count = 0 if S is None else S.shape[0]
    _check(A.lib().matfn_sign(_p(Amat), storage, n, batch, ctypes.byref(opts), _p(S), s_count,
                              _p(out), _report_struct(rep), _p(ws), ws.numel(), _stream()),
           "matfn_sign")
    return out, rep


def prism_alpha_fit(R, S, d: int, lo: float, hi: float, ws=None):
    """alpha* on [lo, hi] for each residual in the batch, plus J's coefficients."""
    _dev(R, S)
    n = R.shape[-1]
    batch = R.numel() // (n * n)
    p = S.shape[-1]
    alpha = torch.empty(batch, dtype=torch.float32, device=R.device)
    J = torch.empty(batch, 5, dtype=torch.float64, device=R.device)
    need = shp_workspace_bytes(A.SHP_OP_ALPHA_FIT, n, n, batch, make_opts(d=d, p=p))
    ws = _ws(need, R.device) if ws is None else ws
    _check(A.lib().prism_alpha_fit(_p(R), n, batch, _p(S), p, d, lo, hi, _p(alpha), _p(J), _p(ws),
                                   ws.numel(), _stream()), "prism_alpha_fit")
    return alpha, J


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(A.lib().shp_kernel_launches())


def shp_split_tf32(X, hi=None, lo=None):
    """(hi, lo) with hi = TF32(X), lo = TF32(X - hi)."""
    _dev(X)
    hi = torch.empty_like(X) if hi is None else hi
    lo = torch.empty_like(X) if lo is None else lo
    _check(A.lib().shp_split_tf32(_p(X), X.numel(), _p(hi), _p(lo), _stream()), "shp_split_tf32")
    return hi, lo


def shp_matmul(Amat, B, prec="tf32", a_trans=False, b_trans=False, A_lo=None, B_lo=None, out=None):
    """Batched C = op(A) op(B) on the tensor cores (one kernel launch).

    A: [batch][M][K] (or [batch][K][M] with a_trans), B: [batch][K][N] (or
    [batch][N][K] with b_trans).  For prec='3xtf32' pass the high parts as
    A/B and the low parts as A_lo/B_lo (see shp_split_tf32)."""
    _dev(Amat, B, A_lo, B_lo, out)
    M, K = (Amat.shape[-1], Amat.shape[-2]) if a_trans else (Amat.shape[-2], Amat.shape[-1])
    N = B.shape[-2] if b_trans else B.shape[-1]
    batch = Amat.numel() // (M * K)
    dt = torch.bfloat16 if prec == "bf16" else torch.float32
    out = torch.empty(batch, M, N, dtype=dt, device=Amat.device) if out is None else out
    _check(A.lib().shp_matmul(_p(Amat), _p(A_lo), int(a_trans), _p(B), _p(B_lo), int(b_trans),
                              _p(out), M, N, K, batch, _PREC[prec], _stream()), "shp_matmul")
    return out


def shp_matmul_f64(Amat, B, out=None, ws=None, reuse_a=False, reuse_b=False, accumulate=False):
    """Batched C = A B in fp64-grade arithmetic on the int8 tensor cores (the
    Ozaki scheme); A [batch][M][K], B [batch][K][N] float64.  reuse_a /
    reuse_b take that operand's digit slices from `ws` as the previous call
    with the same operand and workspace left them; accumulate adds the
    product to `out` (which must then be given)."""
    _dev(Amat, B, out)
    if Amat.dtype != torch.float64 or B.dtype != torch.float64:
        raise ValueError("shp_matmul_f64 takes float64 tensors")
    M, K = Amat.shape[-2], Amat.shape[-1]
    N = B.shape[-1]
    batch = Amat.numel() // (M * K)
    if accumulate and out is None:
        raise ValueError("accumulate needs out")
    out = torch.empty(batch, M, N, dtype=torch.float64, device=Amat.device) if out is None else out
    need = int(A.lib().shp_matmul_f64_workspace_bytes(M, N, K, batch))
    if ws is None:
        if reuse_a or reuse_b:
            raise ValueError("reusing slices needs the workspace of the previous call")
        ws = _ws(need, Amat.device)
    flags = ((A.SHP_MATMUL_REUSE_A if reuse_a else 0) | (A.SHP_MATMUL_REUSE_B if reuse_b else 0)
             | (A.SHP_MATMUL_ACCUMULATE if accumulate else 0))
    _check(A.lib().shp_matmul_f64_ex(_p(Amat), _p(B), _p(out), M, N, K, batch, flags, _p(ws),
                                     ws.numel(), _stream()), "shp_matmul_f64")
    return out


def selftest_bounded_wait(which: str, device=None):
    """Make one bounded pipeline wait run out on purpose ("gemm", "ozaki",
    "sketch", "sketch_alpha" -- the last sketch pass with the fit folded in --
    or "sketch_chain", the few-block sketch's grid barrier); returns (status
    the kernel recorded, alpha of the sketch's fit) -- SHP_ETIMEOUT and, for
    the sketch cases, NaN are expected."""
    code = {"gemm": A.SHP_SELFTEST_GEMM, "ozaki": A.SHP_SELFTEST_OZAKI,
            "sketch": A.SHP_SELFTEST_SKETCH, "sketch_alpha": A.SHP_SELFTEST_SKETCH_ALPHA,
            "sketch_chain": A.SHP_SELFTEST_SKETCH_CHAIN}[which]
    device = device or torch.device("cuda", torch.cuda.current_device())
    status = torch.full((1,), -1, dtype=torch.int32, device=device)
    alpha = torch.zeros(1, dtype=torch.float32, device=device)
    ws = torch.empty(A.SHP_SELFTEST_WS_BYTES, dtype=torch.uint8, device=device)
    _check(A.lib().shp_selftest_bounded_wait(code, _p(status), _p(alpha), _p(ws), ws.numel(),
                                             _stream()), "shp_selftest_bounded_wait")
    return int(status.item()), float(alpha.item())
