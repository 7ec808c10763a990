"""B200-native (sm_100a) block self-attention for the Granite-Speech NAR encoder.

The compute lives in ``libnle.so`` (``csrc/``, C ABI declared in
``include/nle.h``); :mod:`chunked_block_self_b200.nle` is a thin ctypes
binding with the same function names.  The binding is imported lazily so
that :mod:`chunked_block_self_b200.workloads` can be used without the CUDA
library (for instance to draw inputs on a CPU-only host).
"""
__all__ = ["nle", "workloads"]

_SUBMODULES = ("nle", "workloads", "build", "dp")


def __getattr__(name):
    import importlib
    # submodules first: `build` and `workloads` must import without the
    # CUDA library (the build creates it)
    if name in _SUBMODULES:
        return importlib.import_module(f"{__name__}.{name}")
    if name.startswith("_"):
        raise AttributeError(name)
    _nle = importlib.import_module(f"{__name__}.nle")
    if hasattr(_nle, name):
        return getattr(_nle, name)
    raise AttributeError(name)
