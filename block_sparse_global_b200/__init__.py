"""Block-sparse global attention for VGGT-style 3D vision transformers on NVIDIA B200.

The computation lives in libress.so (C ABI, include/ress.h; CUDA kernels for sm_100a).
`ress` is its thin ctypes binding, `pipeline` orders the calls of one layer, `workload`
draws the seeded synthetic inputs.
"""
from . import workload  # noqa: F401  (no CUDA needed)

__all__ = ["workload", "ress", "pipeline"]


def __getattr__(name):
    if name in ("ress", "pipeline", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
