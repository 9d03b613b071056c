"""Oracle of the FP8 KV cache: the E4M3 code, quantisation of new keys and
values into it, and attention over the dequantised cache, in fp64.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py may use it.

What the pages fix: KV-cache quantisation keeps the cached values in a
lower-precision representation, which cuts the bytes per cached token, and it
combines with paging, which only decides where the blocks live
("PagedAttention: KV cache memory management", section "PagedAttention vs
KV-cache quantization vs prefix caching"). They name no format. Readings:

1. Format: E4M3, the 8-bit float of 1 sign, 4 exponent and 3 mantissa bits,
   exponent bias 7, no infinities, S.1111.111 the only NaN codes; so the
   finite values are 0, +-m * 2^-9 (m = 1..7, subnormal) and
   +-(1 + m/8) * 2^(e-7) (e = 1..15, m = 0..7, except e = 15, m = 7), the
   largest being 448.
2. Scales: one fp32 scale per KV head for K and one for V; a cached code c of
   head g stands for ``decode(c) * scale[g]``.
3. Quantisation of a new value x (fp16 or bf16, exact in fp32): ``v = x / s``
   in fp32, correctly rounded; then v rounded to the nearest E4M3 value, ties
   to the even mantissa, with every |v| of 448 or more (infinities too)
   saturated to +-448; the sign is kept (-0 codes as 0x80); NaN codes as 0x7F.
"""

from __future__ import annotations

import numpy as np

from .attention import attend, gather

E4M3_MAX = 448.0
NAN_CODE = 0x7F


def decode(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> float64 values, exact (reading 1)."""
    b = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0**-9, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    val = np.where((b & 0x80) != 0, -mag, mag)
    return np.where((b & 0x7F) == NAN_CODE, np.nan, val)


def encode(v) -> np.ndarray:
    """fp32 values -> E4M3 codes: round to nearest, ties to even, saturating
    (reading 3). Works on exact float64 copies of the fp32 inputs."""
    x = np.asarray(v, dtype=np.float32).astype(np.float64)
    nan = np.isnan(x)
    sign = np.where(np.signbit(x), 0x80, 0)
    a = np.abs(x)
    sat = ~nan & (a >= E4M3_MAX)                  # infinities included
    a = np.where(nan | sat, 0.0, a)
    _, ex = np.frexp(a)                           # a = f * 2^ex, f in [0.5, 1) (0 for a = 0)
    e = np.maximum(ex - 1, -6)                    # binade of a; subnormals share the quantum of 2^-6
    quantum = np.ldexp(1.0, e - 3)                # 3 mantissa bits
    q = np.rint(a / quantum) * quantum            # a / quantum is exact; rint ties to even
    _, qe = np.frexp(q)
    E = qe - 1                                    # binade of the rounded value (may have moved up)
    normal = ((E + 7) << 3) | (q / np.ldexp(1.0, E) * 8 - 8).astype(np.int64)
    sub = (q / 2.0**-9).astype(np.int64)          # exponent field 0
    code = np.where(q == 0.0, 0, np.where(q < 2.0**-6, sub, normal))
    code = np.where(sat, 0x7E, code) | sign
    code = np.where(nan, NAN_CODE, code)
    return code.astype(np.uint8)


def quantize(x, scale) -> np.ndarray:
    """Values x (float, exact in fp32) with per-KV-head scales broadcast over
    the head axis by the caller -> codes of ``x / scale`` (the division in
    fp32)."""
    v = np.asarray(x, dtype=np.float32) / np.asarray(scale, dtype=np.float32)
    return encode(v.astype(np.float32))


def reshape_and_cache(k_cache: np.ndarray, v_cache: np.ndarray, k_new, v_new, slot_mapping,
                      block_size: int, k_scale, v_scale) -> None:
    """In place: the codes of token t's keys and values (``[T, Hkv, D]``
    floats) go to slot ``slot_mapping[t]`` of the uint8 caches
    ``[NB, Hkv, bs, D]``, each KV head quantised with its own scale; a
    negative slot is skipped."""
    k_scale = np.asarray(k_scale, dtype=np.float32)[:, None]
    v_scale = np.asarray(v_scale, dtype=np.float32)[:, None]
    num_blocks = k_cache.shape[0]
    for t, s in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if s < 0:
            continue
        b, o = divmod(s, block_size)
        if b >= num_blocks:
            raise IndexError(f"slot {s} outside the pool")
        k_cache[b, :, o, :] = quantize(k_new[t], k_scale)
        v_cache[b, :, o, :] = quantize(v_new[t], v_scale)


def paged_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables,
                 context_lens, scale: float, block_size: int, k_scale, v_scale) -> np.ndarray:
    """Decode attention over an E4M3 cache: the keys and values of KV head g
    are ``decode(code) * k_scale[g]`` and ``decode(code) * v_scale[g]``; then
    softmax(scale * q K^T) V as in the 16-bit case. ``q``: float64
    ``[S, Hq, D]``; returns float64 ``[S, Hq, D]``."""
    S, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    G = Hq // Hkv
    ks = np.asarray(k_scale, dtype=np.float32).astype(np.float64)
    vs = np.asarray(v_scale, dtype=np.float32).astype(np.float64)
    out = np.zeros((S, Hq, D), dtype=np.float64)
    for s in range(S):
        ctx = int(context_lens[s])
        for g in range(Hkv):
            K = decode(gather(k_cache, block_tables[s], ctx, g, block_size)) * ks[g]
            V = decode(gather(v_cache, block_tables[s], ctx, g, block_size)) * vs[g]
            out[s, g * G:(g + 1) * G] = attend(q[s, g * G:(g + 1) * G], K, V, scale)
    return out
