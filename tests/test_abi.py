"""Host-only checks of the C ABI: the library loads, exports every function
that include/shampoo_prism.h declares, sizes its workspace sensibly and
rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

from second_order_optimizer_shampoo_b200 import _abi as A

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "shampoo_prism.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, re.M)
    return sorted(set(n for n in names if not n.startswith(("if", "for", "while"))))


def test_header_parses():
    names = declared_functions()
    assert set(names) == set(A.EXPORTS), names


def test_header_constants_match_the_binding():
    """Every SHP_* enumerator and #define of the header has the same value in
    the Python binding (the binding restates them, so drift would go silent)."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    found = dict(re.findall(r"\b(SHP_[A-Z0-9_]+)\s*=\s*(\d+)", text))
    found.update(re.findall(r"#define\s+(SHP_[A-Z0-9_]+)\s+(\d+)\s*$", text, flags=re.M))
    m = re.search(r"#define\s+SHP_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m, "SHP_NOALLOC_SCRATCH_BYTES"
    found["SHP_NOALLOC_SCRATCH_BYTES"] = str(int(m.group(1)) << int(m.group(2)))
    assert len(found) >= 20, found
    for name, value in found.items():
        assert getattr(A, name) == int(value), name


def test_library_exports_every_declared_symbol():
    L = A.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.shp_version().decode().count(".") == 2
    assert L.shp_status_string(A.SHP_ESTALL).decode() == "residual stalled"
    # argument checks fail before any CUDA call, so no CUDA error is recorded
    assert L.shp_last_cuda_error().decode() == "none"


def opts(**kw):
    base = dict(d=2, p=8, lo=0.375, hi=1.0, tol=1e-3, max_iter=40, prec=A.SHP_3XTF32,
                fixed_alpha=0, stall_below=0.05, stall_ratio=0.75)
    base.update(kw)
    return A.PrismOpts(**base)


def test_workspace_sizes():
    L = A.lib()
    o = opts()
    n, batch = 1024, 64
    ws = L.shp_workspace_bytes(A.SHP_OP_INV_ROOT, n, n, batch, ctypes.byref(o))
    # 13 n x n fp32 buffers per block in split mode (Y, Z ping-pong and R, g as
    # hi/lo pairs, plus a plain R for the sketch passes), plus the sketch block
    assert ws >= 13 * n * n * 4 * batch
    assert ws < 14 * n * n * 4 * batch
    o1 = opts(prec=A.SHP_TF32)
    ws1 = L.shp_workspace_bytes(A.SHP_OP_INV_ROOT, n, n, batch, ctypes.byref(o1))
    assert 6 * n * n * 4 * batch <= ws1 < 7 * n * n * 4 * batch
    o2 = opts(prec=A.SHP_BF16)
    wp = L.shp_workspace_bytes(A.SHP_OP_POLAR, 4096, 1024, 96, ctypes.byref(o2))
    assert wp >= 2 * 4096 * 1024 * 2 * 96
    assert L.shp_workspace_bytes(A.SHP_OP_INV_ROOT, n, n, batch, ctypes.byref(opts(d=3))) == 0
    assert L.shp_workspace_bytes(A.SHP_OP_INV_ROOT, n, n, batch, ctypes.byref(opts(p=33))) == 0
    assert L.shp_workspace_bytes(99, n, n, batch, ctypes.byref(o)) == 0
    # several EMA steps at once: the products of both factors (plus split G)
    we = L.shp_workspace_bytes(A.SHP_OP_GRAM_EMA_STEPS, 512, 256, 10, ctypes.byref(o1))
    assert (512 * 512 + 256 * 256) * 4 * 10 <= we < (512 * 512 + 256 * 256) * 4 * 10 + (1 << 20)
    we3 = L.shp_workspace_bytes(A.SHP_OP_GRAM_EMA_STEPS, 512, 256, 10, ctypes.byref(o))
    assert we3 - we == 2 * 512 * 256 * 4 * 10


def test_invalid_arguments_rejected_before_launch():
    L = A.lib()
    o = opts()
    fake = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first
    # null input
    assert L.matfn_inv_root(None, 64, 1, 0, ctypes.byref(o), fake, 80, fake, None, fake, 1 << 40,
                            None) == A.SHP_EINVAL
    # n not a multiple of 4
    assert L.matfn_inv_root(fake, 66, 1, 0, ctypes.byref(o), fake, 80, fake, None, fake, 1 << 40,
                            None) == A.SHP_EINVAL
    # bad power
    assert L.matfn_inv_root(fake, 64, 1, 7, ctypes.byref(o), fake, 80, fake, None, fake, 1 << 40,
                            None) == A.SHP_EINVAL
    # too few sketch slices for two passes
    assert L.matfn_inv_root(fake, 64, 1, 0, ctypes.byref(o), fake, 79, fake, None, fake, 1 << 40,
                            None) == A.SHP_EINVAL
    # workspace too small
    assert L.matfn_inv_root(fake, 64, 1, 0, ctypes.byref(o), fake, 80, fake, None, fake, 16,
                            None) == A.SHP_EINVAL
    # bad degree / sketch width
    assert L.matfn_inv_root(fake, 64, 1, 0, ctypes.byref(opts(d=0)), fake, 80, fake, None, fake,
                            1 << 40, None) == A.SHP_EINVAL
    assert L.prism_alpha_fit(fake, 64, 1, fake, 0, 2, 0.375, 1.0, fake, None, fake, 1 << 30,
                             None) == A.SHP_EINVAL
    assert L.prism_alpha_fit(fake, 64, 1, fake, 8, 2, 1.0, 0.5, fake, None, fake, 1 << 30,
                             None) == A.SHP_EINVAL
    # bf16 polar with n not a multiple of 8
    assert L.matfn_polar(fake, A.SHP_BF16, 64, 36, 1, ctypes.byref(o), fake, 40, fake, None, fake,
                         1 << 40, None) == A.SHP_EINVAL
    # misaligned pointer
    mis = ctypes.c_void_p(0x10004)
    assert L.shampoo_gram_ema(mis, 64, 64, 1, fake, fake, 0.9, 1e-6, A.SHP_TF32, fake, 1 << 30,
                              None) == A.SHP_EINVAL
    assert L.shampoo_gram_ema_steps(fake, 0, 64, 64, 1, fake, fake, 0.9, 1e-6, A.SHP_TF32, fake,
                                    1 << 30, None) == A.SHP_EINVAL
    assert L.shampoo_gram_ema_steps(mis, 2, 64, 64, 1, fake, fake, 0.9, 1e-6, A.SHP_TF32, fake,
                                    1 << 30, None) == A.SHP_EINVAL
    assert L.shampoo_gram_ema_steps(fake, 2, 64, 64, 1, fake, fake, 0.9, 1e-6, A.SHP_TF32, fake,
                                    16, None) == A.SHP_EINVAL  # workspace too small
    assert L.shampoo_gram_ema_steps(fake, 300, 64, 64, 300, fake, fake, 0.9, 1e-6, A.SHP_TF32,
                                    fake, 1 << 40, None) == A.SHP_EUNSUPPORTED
    assert L.shampoo_apply(fake, fake, fake, fake, 64, 62, 1, 1e-3, A.SHP_TF32, fake, 1 << 30,
                           None) == A.SHP_EINVAL
    assert L.shampoo_apply(fake, fake, fake, fake, 64, 64, 1, 1e-3, 5, fake, 1 << 30,
                           None) == A.SHP_EINVAL


def test_adaptive_degree_validation():
    """Adaptive degree needs d = 2 (the degree it raises to), a fitted alpha
    and a threshold >= 0."""
    L = A.lib()
    fake = ctypes.c_void_p(0x10000)
    for bad in (opts(adaptive_degree=1, d=1), opts(adaptive_degree=1, fixed_alpha=1),
                opts(adaptive_degree=1, raise_above=-0.5)):
        assert L.shp_workspace_bytes(A.SHP_OP_INV_ROOT, 1024, 1024, 4, ctypes.byref(bad)) == 0
        assert L.matfn_inv_root(fake, 64, 1, 0, ctypes.byref(bad), fake, 80, fake, None, fake,
                                1 << 40, None) == A.SHP_EINVAL
    good = opts(adaptive_degree=1, raise_above=0.9)
    assert L.shp_workspace_bytes(A.SHP_OP_INV_ROOT, 1024, 1024, 4, ctypes.byref(good)) > 0


def test_apply_ex_validation():
    L = A.lib()
    fake = ctypes.c_void_p(0x10000)
    mis = ctypes.c_void_p(0x10004)
    # misaligned momentum buffer
    assert L.shampoo_apply_ex(fake, mis, None, fake, fake, fake, 64, 64, 1, 1e-3, 0.9,
                              A.SHP_TF32, fake, 1 << 30, None) == A.SHP_EINVAL
    # non-finite step or momentum factor
    assert L.shampoo_apply_ex(fake, None, None, fake, fake, fake, 64, 64, 1, float("nan"), 0.9,
                              A.SHP_TF32, fake, 1 << 30, None) == A.SHP_EINVAL
    assert L.shampoo_apply_ex(fake, fake, fake, fake, fake, fake, 64, 64, 1, 1e-3,
                              float("inf"), A.SHP_TF32, fake, 1 << 30, None) == A.SHP_EINVAL
    # workspace too small
    assert L.shampoo_apply_ex(fake, None, fake, fake, fake, fake, 64, 64, 1, 1e-3, 0.0,
                              A.SHP_TF32, fake, 8, None) == A.SHP_EINVAL


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    from second_order_optimizer_shampoo_b200 import prism
    x = torch.zeros(64, 64)
    with pytest.raises(ValueError):
        prism.matfn_inv_root(x)
