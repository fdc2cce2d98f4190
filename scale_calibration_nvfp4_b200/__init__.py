"""NVFP4 scale calibration on B200 (sm_100a).

The compute path is the C-ABI library ``libnvfp4.so`` built from ``csrc/``;
``nvfp4`` is its thin ctypes binding (argument marshalling only).  Importing
the package itself loads nothing, so the seeded input module ``workloads``
can be used without the CUDA library.
"""
import importlib

__all__ = ["nvfp4", "workloads", "build"]
__version__ = "0.1.0"


def __getattr__(name):
    if name in __all__:
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
