"""Shared helpers for the GPU parity tests (upload/download, error measures,
the arithmetic error bounds the tolerances come from)."""
import numpy as np

# TF32 keeps 10 explicit mantissa bits and the B200 tensor cores truncate fp32
# operands to it: one operand carries a relative error below 2^-10.
U_TF32 = 2.0 ** -10
# fp32 accumulation over K terms: gamma_K = K * 2^-24 (standard bound).
U_FP32 = 2.0 ** -24
# 3xTF32: both parts are rounded to nearest TF32 (2^-11 each); the dropped
# lo*lo term and the rounding of lo leave about 2^-21 relative per product.
U_3XTF32 = 2.0 ** -21


def gemm_bound(absA, absB, K, prec):
    """Elementwise forward-error bound of C = A B computed on the tensor cores:
    (2 u_op + K u_fp32) (|A| |B|)_ij, with u_op the per-operand error."""
    u_op = U_TF32 if prec == "tf32" else U_3XTF32
    return (2 * u_op + K * U_FP32) * (absA @ absB)


def relerr(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def to_dev(torch, x, dev="cuda:0"):
    return torch.from_numpy(np.ascontiguousarray(x)).to(dev)


def bf16_to_dev(torch, bits, dev="cuda:0"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)


def to_host(t):
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()
