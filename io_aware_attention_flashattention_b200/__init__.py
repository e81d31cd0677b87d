"""IO-aware exact attention (FlashAttention-style forward and recomputation
backward) for NVIDIA B200, sm_100a.

The compute lives in libfa_b200.so (C ABI: include/fa.h); ``api`` is the Python
binding and ``inputs`` the seeded synthetic workloads. Importing the package does
not load the library; the first call does, and fails loudly if it is missing.
"""
import importlib

__version__ = "0.1.0"

_SUBMODULES = ("api", "inputs", "build")


def __getattr__(name):
    # Lazy access to the binding, so that the input generators import on machines
    # where the library has not been built yet.
    if name in _SUBMODULES:
        return importlib.import_module(f"{__name__}.{name}")
    api = importlib.import_module(f"{__name__}.api")
    if hasattr(api, name):
        return getattr(api, name)
    raise AttributeError(name)
