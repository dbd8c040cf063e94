"""B200 (sm_100a) forward pass of VSA-style cube-based hierarchical sparse attention.

The computation runs in libvsa.so (hand-written CUDA, C ABI in include/vsa.h);
``vsa`` is its Python binding. Importing the package does not load the
library; the first call does, and raises if it is not built or no sm_100
GPU is present.
"""
__all__ = ["Plan", "forward", "VSAError", "lib_path"]


def __getattr__(name):
    if name in __all__:
        from . import vsa
        return getattr(vsa, name)
    raise AttributeError(name)
