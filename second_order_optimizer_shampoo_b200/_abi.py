"""ctypes view of the C ABI in include/shampoo_prism.h.

Only marshalling lives here: structure layouts, argument types and the
loader.  There is no fallback implementation; if the shared library is
missing the import of any entry point raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libshampoo_prism.so")

# status codes
SHP_OK, SHP_EINVAL, SHP_EUNSUPPORTED, SHP_ECUDA = 0, 1, 2, 3
SHP_ENOCONV, SHP_ESTALL, SHP_ENONFINITE, SHP_ETIMEOUT = 16, 17, 18, 19
# precisions / storage
SHP_TF32, SHP_3XTF32, SHP_BF16, SHP_OZAKI = 0, 1, 2, 3
# powers
SHP_POW_INV4, SHP_POW_INV2, SHP_POW_SQRT = 0, 1, 2
# workspace queries
SHP_OP_INV_ROOT, SHP_OP_POLAR, SHP_OP_ALPHA_FIT, SHP_OP_APPLY, SHP_OP_GRAM_EMA = 0, 1, 2, 3, 4
SHP_OP_GRAM_EMA_STEPS = 5
# shp_matmul_f64_ex flags
SHP_MATMUL_REUSE_A, SHP_MATMUL_REUSE_B, SHP_MATMUL_ACCUMULATE = 1, 2, 4
# bounded-wait self-test
SHP_SELFTEST_GEMM, SHP_SELFTEST_OZAKI, SHP_SELFTEST_SKETCH = 0, 1, 2
SHP_SELFTEST_SKETCH_ALPHA, SHP_SELFTEST_SKETCH_CHAIN = 3, 4
SHP_SELFTEST_WS_BYTES = 4 << 20
# fixed device scratch of prism_alpha_fit_noalloc
SHP_NOALLOC_SCRATCH_BYTES = 4 << 20

EXPORTS = ("shp_workspace_bytes", "shampoo_gram_ema", "shampoo_gram_ema_steps", "matfn_inv_root", "matfn_polar", "matfn_polar_varsize",
           "matfn_sign",
           "prism_alpha_fit", "shampoo_apply", "shampoo_apply_ex", "shp_matmul", "shp_split_tf32",
           "shp_matmul_f64_workspace_bytes", "shp_matmul_f64", "shp_matmul_f64_ex",
           "shp_kernel_launches", "prism_alpha_fit_noalloc", "shp_selftest_bounded_wait", "shp_status_string", "shp_last_cuda_error",
           "shp_version")


class PrismOpts(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("p", ctypes.c_int), ("lo", ctypes.c_float),
                ("hi", ctypes.c_float), ("tol", ctypes.c_float), ("max_iter", ctypes.c_int),
                ("prec", ctypes.c_int), ("fixed_alpha", ctypes.c_int),
                ("stall_below", ctypes.c_float), ("stall_ratio", ctypes.c_float),
                ("adaptive_degree", ctypes.c_int), ("raise_above", ctypes.c_float),
                ("host_loop", ctypes.c_int)]


class PrismReport(ctypes.Structure):
    _fields_ = [("status", ctypes.c_void_p), ("iters", ctypes.c_void_p),
                ("resid", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("degree", ctypes.c_void_p)]


_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float
_INT = ctypes.c_int

_SIGS = {
    "shp_workspace_bytes": (_SZ, [_INT, _I64, _I64, _I64, ctypes.POINTER(PrismOpts)]),
    "shampoo_gram_ema": (_INT, [_P, _I64, _I64, _I64, _P, _P, _F, _F, _INT, _P, _SZ, _P]),
    "shampoo_gram_ema_steps": (_INT, [_P, _I64, _I64, _I64, _I64, _P, _P, _F, _F, _INT, _P, _SZ,
                                      _P]),
    "matfn_inv_root": (_INT, [_P, _I64, _I64, _INT, ctypes.POINTER(PrismOpts), _P, _I64, _P,
                              ctypes.POINTER(PrismReport), _P, _SZ, _P]),
    "matfn_polar": (_INT, [_P, _INT, _I64, _I64, _I64, ctypes.POINTER(PrismOpts), _P, _I64, _P,
                           ctypes.POINTER(PrismReport), _P, _SZ, _P]),
    "matfn_polar_varsize": (_INT, [_P, _P, _P, _I64, ctypes.POINTER(PrismOpts), _P, _I64, _P,
                                   ctypes.POINTER(PrismReport), _P]),
    "matfn_sign": (_INT, [_P, _INT, _I64, _I64, ctypes.POINTER(PrismOpts), _P, _I64, _P,
                          ctypes.POINTER(PrismReport), _P, _SZ, _P]),
    "prism_alpha_fit": (_INT, [_P, _I64, _I64, _P, _INT, _INT, _F, _F, _P, _P, _P, _SZ, _P]),
    "shampoo_apply": (_INT, [_P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _P, _SZ, _P]),
    "shampoo_apply_ex": (_INT, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _F, _F, _INT, _P, _SZ,
                                _P]),
    "shp_matmul": (_INT, [_P, _P, _INT, _P, _P, _INT, _P, _I64, _I64, _I64, _I64, _INT, _P]),
    "shp_split_tf32": (_INT, [_P, _I64, _P, _P, _P]),
    "shp_matmul_f64_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I64]),
    "shp_matmul_f64": (_INT, [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "shp_matmul_f64_ex": (_INT, [_P, _P, _P, _I64, _I64, _I64, _I64, _INT, _P, _SZ, _P]),
    "shp_kernel_launches": (ctypes.c_uint64, []),
    "prism_alpha_fit_noalloc": (_INT, [_P, _I64, _I64, _P, _INT, _INT, _F, _F, _P, _P, _P]),
    "shp_selftest_bounded_wait": (_INT, [_INT, _P, _P, _P, _SZ, _P]),
    "shp_status_string": (ctypes.c_char_p, [_INT]),
    "shp_last_cuda_error": (ctypes.c_char_p, []),
    "shp_version": (ctypes.c_char_p, []),
}


def lib():
    """Load libshampoo_prism.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m second_order_optimizer_shampoo_b200.build_lib` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib
