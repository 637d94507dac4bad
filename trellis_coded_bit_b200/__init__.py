"""EXL3 trellis-decoded matmul for NVIDIA B200 (sm_100a).

The compute path is the C-ABI CUDA library built from ``csrc/`` (declared in
``include/exl3.h``); ``exl3`` is its ctypes binding, ``inputs`` the seeded
synthetic-input generator and ``workloads`` the named layer shapes.  The
binding is imported lazily so that ``inputs``/``workloads`` work without CUDA.
"""

__all__ = ["exl3", "inputs", "workloads", "build"]


def __getattr__(name):
    if name in __all__:
        import importlib

        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
