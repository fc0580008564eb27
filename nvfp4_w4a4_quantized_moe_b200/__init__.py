"""NVFP4 W4A4 routed-expert MoE layer for B200 (sm_100a).

The compute lives in ``libnvfp4moe.so`` (hand-written CUDA behind a C ABI,
declared in ``include/nvfp4_moe.h``).  ``capi`` is the thin ctypes binding;
importing it loads the library and fails loudly if it is missing.
``workloads`` draws the seeded synthetic inputs.
"""
import importlib

__all__ = ["capi", "workloads"]


def __getattr__(name):
    if name in ("capi", "workloads"):
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
