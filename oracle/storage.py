"""Exact widening of stored cache elements to float64 (oracle; test infrastructure only).

The pages fix no storage precision; the cache may hold fp32, fp16 or bf16.  The
oracle reads the values exactly as stored and widens them without rounding:

* fp32: float32 -> float64 is exact.
* fp16: the 16-bit pattern is an IEEE binary16 value; NumPy's float16 decodes it,
        and float16 -> float64 is exact.
* bf16: a bfloat16 pattern is the upper half of a binary32 pattern, so shifting
        the 16 bits left by 16 and reading the word as float32 gives the value
        exactly; float32 -> float64 is exact.

16-bit types are passed as ``uint16`` arrays of bit patterns (fp16 may also be
passed as ``float16``); fp32 as ``float32``.
"""

import numpy as np

STORAGE_DTYPES = ("f32", "f16", "bf16")


def to_f64(raw, dtype):
    """Return ``raw`` (stored elements of ``dtype``) as a float64 array, exactly."""
    raw = np.asarray(raw)
    if dtype == "f32":
        if raw.dtype != np.float32:
            raise TypeError(f"f32 storage must be float32, got {raw.dtype}")
        return raw.astype(np.float64)
    if dtype == "f16":
        if raw.dtype == np.float16:
            return raw.astype(np.float64)
        if raw.dtype != np.uint16:
            raise TypeError(f"f16 storage must be uint16 bits or float16, got {raw.dtype}")
        return raw.view(np.float16).astype(np.float64)
    if dtype == "bf16":
        if raw.dtype != np.uint16:
            raise TypeError(f"bf16 storage must be uint16 bits, got {raw.dtype}")
        widened = raw.astype(np.uint32) << np.uint32(16)
        return widened.view(np.float32).astype(np.float64)
    raise ValueError(f"unknown storage dtype {dtype!r}; expected one of {STORAGE_DTYPES}")
