"""H-BitLinear forward of BitNet v2 for B200 (sm_100a).

``hbl`` is the ctypes binding of libhbl.so (include/hbl.h); ``layer`` holds
small tensor-level helpers built on it; ``inputs`` draws the seeded synthetic
workloads.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs", "hbl", "layer"]


def __getattr__(name):
    if name in ("hbl", "layer"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
