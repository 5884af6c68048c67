"""SmolVLA action-chunk generation on B200 (sm_100a): prefix prefill into a
per-layer K/V cache and the Euler flow-matching denoise of the action expert,
as hand-written CUDA kernels behind the C ABI of include/svla.h.

``SmolVLA`` (runtime.py) is the Python face; ``_abi`` holds the ctypes
declarations; ``build`` compiles libsvla.so in-tree.
"""
from . import _abi  # noqa: F401

__all__ = ["SmolVLA", "_abi"]


def __getattr__(name):
    if name == "SmolVLA":
        from .runtime import SmolVLA
        return SmolVLA
    raise AttributeError(name)
