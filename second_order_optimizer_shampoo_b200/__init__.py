"""B200 (sm_100a) Shampoo preconditioner step with PRISM-accelerated
Newton-Schulz matrix functions.

The compute path is the C ABI in ``include/shampoo_prism.h`` implemented by
``libshampoo_prism.so`` (hand-written tcgen05/TMA kernels).  ``prism`` is its
thin Python binding; ``synth`` draws seeded synthetic inputs.
"""
import importlib

__all__ = ["prism", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
