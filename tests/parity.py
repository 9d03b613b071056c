"""Shared helpers of the GPU parity tests: seeded paged batches and the tolerance check.

Tolerance (stated for fp16/bf16 inputs with fp32 accumulation): every element
within 2e-3 of the fp64 oracle, and the whole output within 1e-2 in relative
2-norm. Small-context edge cases in bf16 may instead allow 2e-3 plus half a
bf16 unit in the last place of the reference, because an output near 1 or
above cannot be represented in bf16 to 2e-3.
"""

from __future__ import annotations

import numpy as np

from oracle.numerics import half_ulp, to_f64
import workloads

ATOL = 2e-3
RTOL_NORM = 1e-2


def to_bits(t) -> np.ndarray:
    import torch

    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(bits: np.ndarray, dtype: str, device="cuda"):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16).to(device)


def check_close(gpu_bits: np.ndarray, ref: np.ndarray, dtype: str, rows=None, allow_ulp=False):
    """Asserts the tolerance; returns (max abs error, relative 2-norm error)."""
    got = to_f64(gpu_bits, dtype)
    if rows is not None:
        got, ref = got[rows], ref[rows]
    err = np.abs(got - ref)
    bound = ATOL + (half_ulp(ref, dtype) if allow_ulp else 0.0)
    bad = err > bound
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / nref if nref > 0 else np.linalg.norm(got - ref)
    assert not np.isnan(got).any(), "NaN in output"
    assert not bad.any(), f"max abs err {err.max():.3e} at {np.argwhere(bad)[:5].tolist()}"
    assert rel <= RTOL_NORM, f"relative 2-norm err {rel:.3e}"
    return float(err.max()), float(rel)


def random_paged_batch(seed, S, Hq, Hkv, D, bs, lens, dtype, extra_blocks=7):
    """A paged cache holding ``lens`` tokens per sequence on shuffled physical blocks.

    Returns (q_bits [S,Hq,D], k_bits, v_bits [NB,Hkv,bs,D], tables int32 [S,MB], lens int32).
    Values are seeded N(0,1); slots past each sequence's length hold values too.
    """
    rng = np.random.default_rng(seed)
    need = [-(-L // bs) for L in lens]
    nb = sum(need) + extra_blocks
    perm = rng.permutation(nb).astype(np.int32)
    mb = max(1, max(need))
    tables = np.full((S, mb), -1, np.int32)
    i = 0
    for s, n in enumerate(need):
        tables[s, :n] = perm[i:i + n]
        i += n
    q = workloads.normal_bits([seed, 1], (S, Hq, D), dtype)
    k = workloads.normal_bits([seed, 2], (nb, Hkv, bs, D), dtype)
    v = workloads.normal_bits([seed, 3], (nb, Hkv, bs, D), dtype)
    return q, k, v, tables, np.asarray(lens, np.int32)


def random_e4m3_codes(seed, shape) -> np.ndarray:
    """Seeded uniform E4M3 codes (uint8) with the two NaN codes replaced by +-1.875
    (0x3F / 0xBF): a cache of every finite magnitude from 2^-9 to 448."""
    rng = np.random.default_rng(seed)
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    nan = (c & 0x7F) == 0x7F
    c[nan] = c[nan] & 0xBF
    return c
