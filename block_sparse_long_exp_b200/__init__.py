"""MSA (MiniMax Sparse Attention) forward hot path for NVIDIA B200 (sm_100a).

The CUDA kernels live in libmsa.so (C ABI: include/msa.h); ``msa`` is the thin
Python binding (imported on first use).  ``workloads`` draws the seeded
synthetic inputs.
"""
import importlib

from . import workloads  # noqa: F401

__all__ = ["workloads", "msa", "build"]


def __getattr__(name):
    if name in ("msa", "build"):
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
