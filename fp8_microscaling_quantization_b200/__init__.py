"""Block-scaled microscaling quantization (NVFP4, MXFP4, FP8 power-of-two) for B200.

The compute lives in ``libbsq.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/bsq.h``).  ``fp8_microscaling_quantization_b200.bsq``
is the thin ctypes binding with the same entry-point names; it is imported on
first use of any of them, and raises if the library was not built.
"""
_BINDING_NAMES = None


def __getattr__(name):
    if name.startswith("bsq_") or name in ("BsqError", "lib_path", "Format", "DType", "Direction"):
        from . import bsq
        return getattr(bsq, name)
    raise AttributeError(name)
