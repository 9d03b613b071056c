"""Seeded N(0,1) values as fp16 / bf16 bit patterns.

Definition of the stream for seed words ``w`` and ``n`` values: the values are
cut into chunks of ``CHUNK`` (2^22); chunk ``c`` is
``Generator(PCG64(SeedSequence(w + [c]))).standard_normal(len, float32)``.
Chunks are independent, so they are drawn in parallel threads; the result
depends only on ``w`` and the shape. Values are rounded to the 16-bit type:
fp16 by NumPy's cast, bf16 by torch's CPU cast (round to nearest even), and
returned as ``uint16`` bits so every consumer reads exactly the same numbers.
"""

from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np

# Stream tags inside a workload's value seed.
K_STREAM, V_STREAM, Q_STREAM = 0, 1, 2
CHUNK = 1 << 22


def value_seed_words(value_seed: int, stream: int, index: int) -> list[int]:
    return [int(value_seed), int(stream), int(index)]


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(32, os.cpu_count() or 1))


def _draw(words, c, length, dtype):
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(words) + [c])))
    x = rng.standard_normal(size=length, dtype=np.float32)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    return x


def normal_bits(seed_words, shape, dtype: str) -> np.ndarray:
    """``shape`` draws of N(0,1), rounded to ``dtype`` ("f16" | "bf16"), as uint16 bits."""
    if dtype not in ("f16", "bf16"):
        raise ValueError(f"unknown dtype {dtype!r}")
    shape = tuple(int(s) for s in np.atleast_1d(shape)) if not isinstance(shape, tuple) else shape
    n = int(np.prod(shape)) if len(shape) else 1
    nchunks = max(1, -(-n // CHUNK))
    lengths = [min(CHUNK, n - c * CHUNK) for c in range(nchunks)]
    if nchunks == 1:
        parts = [_draw(seed_words, 0, lengths[0], dtype)]
    else:
        with cf.ThreadPoolExecutor(min(_threads(), nchunks)) as ex:
            parts = list(ex.map(lambda c: _draw(seed_words, c, lengths[c], dtype), range(nchunks)))
    x = parts[0] if len(parts) == 1 else np.concatenate(parts)
    if dtype == "bf16":
        import torch

        x = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return x.reshape(shape)
