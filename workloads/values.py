"""Seeded N(0,1) values as fp16 / bf16 bit patterns.

Values are drawn as float32 from NumPy's PCG64 generator and rounded to the
16-bit type: fp16 by NumPy's cast, bf16 by torch's CPU cast (round to nearest
even). The result is returned as ``uint16`` bits so that every consumer reads
exactly the same numbers. Each draw is keyed by a tuple of integers through
``numpy.random.SeedSequence``, so any op's values can be regenerated alone.
"""

from __future__ import annotations

import numpy as np

# Stream tags inside a workload's value seed.
K_STREAM, V_STREAM, Q_STREAM = 0, 1, 2


def value_seed_words(value_seed: int, stream: int, index: int) -> list[int]:
    return [int(value_seed), int(stream), int(index)]


def normal_bits(seed_words, shape, dtype: str) -> np.ndarray:
    """``shape`` draws of N(0,1), rounded to ``dtype`` ("f16" | "bf16"), as uint16 bits."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(seed_words))))
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        import torch

        t = torch.from_numpy(x).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16).reshape(shape)
    raise ValueError(f"unknown dtype {dtype!r}")
