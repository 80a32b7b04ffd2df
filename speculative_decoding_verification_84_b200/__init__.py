"""B200-native batched speculative-sampling verification.

``verify`` / ``workspace_size`` come from the ctypes binding over the CUDA
C-ABI library (``binding.py``); ``workloads`` holds the seeded synthetic inputs.
The binding is imported lazily so that the input generators stay usable on a
machine without the built library.
"""
import importlib

__all__ = ["verify", "workspace_size"]


def __getattr__(name):
    if name in ("verify", "workspace_size"):
        return getattr(importlib.import_module(__name__ + ".binding"), name)
    raise AttributeError(name)
