"""Grouped MXFP8 MoE expert MLP for NVIDIA B200 (sm_100a).

The CUDA library (libmoe_mxfp8.so, C ABI in include/moe_mxfp8.h) does all
the work; `lib` is its ctypes binding and `layer.GroupedMLP` holds the
device buffers of one layer.  `workloads` draws seeded synthetic inputs.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads", "lib", "layer"]


def __getattr__(name):
    # the CUDA binding is imported lazily so that the input generator works
    # on machines without the built library
    if name in ("lib", "layer"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
