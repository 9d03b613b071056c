"""Decoding of 16-bit float bit patterns to fp64, for the oracle side.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py may use it.

The pages fix no precision for the kernel; the attention oracle works in fp64
on the exact fp16 / bf16 values the GPU reads. Inputs travel between the two
sides as raw ``uint16`` bit patterns, so both read identical bits.

* fp16: IEEE 754 binary16, decoded by NumPy's own float16 type.
* bf16: the upper 16 bits of an IEEE 754 binary32; decoding shifts the pattern
  into the high half of a 32-bit word.
"""

from __future__ import annotations

import numpy as np

F16 = "f16"
BF16 = "bf16"


def to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """uint16 bit patterns of ``dtype`` -> float64 values (exact)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float64)
    if dtype == BF16:
        return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


def half_ulp(x: np.ndarray, dtype: str) -> np.ndarray:
    """Half a unit in the last place of ``dtype`` at |x| (normal range)."""
    mant_bits = 10 if dtype == F16 else 7
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0**-14)
    return np.ldexp(1.0, np.floor(np.log2(ax)).astype(np.int64) - mant_bits - 1)
