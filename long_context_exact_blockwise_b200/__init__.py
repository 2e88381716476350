"""Exact blockwise (ring) attention for NVIDIA B200.

The Python binding lives in ``long_context_exact_blockwise_b200.ringattn``
(ctypes over ``libringattn.so``); its names are also reachable from this
package, loaded on first use.  ``build_lib`` builds the shared object with
nvcc and does not need it to exist.
"""
import importlib as _importlib

__all__ = ["ringattn", "build_lib"]


def __getattr__(name):
    if name in ("ringattn", "build_lib"):
        return _importlib.import_module(f"{__name__}.{name}")
    mod = _importlib.import_module(f"{__name__}.ringattn")
    try:
        return getattr(mod, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
