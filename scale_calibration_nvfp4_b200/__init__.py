"""NVFP4 scale calibration on B200 (sm_100a).

The compute path is the C-ABI library ``libnvfp4.so`` built from ``csrc/``;
``nvfp4`` is its thin ctypes binding (argument marshalling only).  Importing
the package itself loads nothing, so the seeded input module ``workloads``
can be used without the CUDA library.
"""
__all__ = ["nvfp4", "workloads"]
__version__ = "0.1.0"


def __getattr__(name):
    if name == "nvfp4":
        from . import nvfp4 as _m
        return _m
    if name == "workloads":
        from . import workloads as _w
        return _w
    raise AttributeError(name)
