"""Oracle of decode attention over a paged KV cache, in fp64.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py may use it.

What it restates: the attention computation itself is unchanged by paging -
the same math as with a contiguous cache ("Your GPU was mostly empty", section
"The OS already solved this in the 1960s") - and the kernel only has to follow
the block table to find each token's keys and values ("vLLM and
PagedAttention", section "Architecture, step by step", step 3). So the oracle
is the plain definition written out:

1. gather: for token ``j < ctx`` of sequence ``s``, its key is
   ``k_cache[block_tables[s, j // bs], g, j % bs, :]`` (values likewise);
2. for each query head ``h`` of the sequence, with KV head ``g = h // G``
   (``G = num_q_heads // num_kv_heads``, contiguous groups - a reading, the
   pages do not discuss grouped heads):
   ``z = scale * K q_h``, ``p = exp(z - max z) / sum(exp(z - max z))``,
   ``out_h = p^T V``;
3. a sequence with ``ctx == 0`` attends to nothing; its output row is zero
   (a reading, the pages are silent).

For long contexts the token range is cut into partitions of ``partition_size``
tokens. :func:`partition_partials` gives each partition's running maximum
``m_p``, exponent sum ``l_p = sum exp(z - m_p)`` and unnormalised output
``acc_p = sum exp(z - m_p) v``; :func:`merge_partials` combines them by the
log-sum-exp identity ``M = max m_p``, ``L = sum l_p e^(m_p - M)``,
``out = sum e^(m_p - M) acc_p / L``, which equals the unsplit softmax exactly
in real arithmetic.
"""

from __future__ import annotations

import math

import numpy as np

from .numerics import to_f64


def gather(cache: np.ndarray, table, ctx: int, kv_head: int, block_size: int) -> np.ndarray:
    """Contiguous ``[ctx, head_dim]`` view of one sequence's tokens for one KV head."""
    j = np.arange(ctx)
    blocks = np.asarray(table, dtype=np.int64)[j // block_size]
    return cache[blocks, kv_head, j % block_size, :]


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q K^T) V for one or more query rows ``q[..., D]``; fp64."""
    q = np.asarray(q, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(q.shape[:-1] + (V.shape[1],), dtype=np.float64)
    z = scale * (q @ K.T)                       # [..., ctx]
    z = z - z.max(axis=-1, keepdims=True)
    p = np.exp(z)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ V


def _rows(cache, table, ctx, g, block_size, dtype):
    x = gather(cache, table, ctx, g, block_size)
    return x.astype(np.float64) if dtype is None else to_f64(x, dtype)


def paged_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables,
                 context_lens, scale: float, block_size: int, seqs=None, dtype=None) -> np.ndarray:
    """Decode attention for every sequence (or the subset ``seqs``).

    ``q``: float64 ``[S, Hq, D]``; caches ``[NB, Hkv, bs, D]``, either float
    values or, with ``dtype`` given ("f16" | "bf16"), uint16 bit patterns that
    are decoded to fp64 after the gather; returns float64 ``[S, Hq, D]`` (rows
    not in ``seqs`` stay zero).
    """
    S, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    G = Hq // Hkv
    out = np.zeros((S, Hq, D), dtype=np.float64)
    for s in (range(S) if seqs is None else seqs):
        ctx = int(context_lens[s])
        for g in range(Hkv):
            K = _rows(k_cache, block_tables[s], ctx, g, block_size, dtype)
            V = _rows(v_cache, block_tables[s], ctx, g, block_size, dtype)
            out[s, g * G:(g + 1) * G] = attend(q[s, g * G:(g + 1) * G], K, V, scale)
    return out


def paged_prefill(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables,
                  context_lens, scale: float, block_size: int, dtype=None) -> np.ndarray:
    """Attention of a chunk of ``T`` new tokens per sequence over the paged cache,
    causal within the chunk: the prefill of a prompt, or a chunk of it, whose keys
    and values are already in the sequence's blocks ("PagedAttention: KV cache
    memory management", section "A request lifecycle": prefill creates the
    cache state through the block table). Reading (the pages leave it open): query
    ``i`` of sequence ``s`` sits at position ``ctx_s - T + i`` and attends to the
    tokens ``j <= ctx_s - T + i``, where ``context_lens[s]`` counts the chunk; a
    query with no such token (``ctx_s < T - i``) gives a zero row.

    ``q``: float64 ``[S, T, Hq, D]``; caches and ``dtype`` as for
    :func:`paged_decode`; returns float64 ``[S, T, Hq, D]``.
    """
    S, T, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    G = Hq // Hkv
    out = np.zeros((S, T, Hq, D), dtype=np.float64)
    for s in range(S):
        ctx = int(context_lens[s])
        for g in range(Hkv):
            K = _rows(k_cache, block_tables[s], ctx, g, block_size, dtype)
            V = _rows(v_cache, block_tables[s], ctx, g, block_size, dtype)
            for i in range(T):
                vis = ctx - T + i + 1
                if vis > 0:
                    out[s, i, g * G:(g + 1) * G] = attend(q[s, i, g * G:(g + 1) * G], K[:vis], V[:vis],
                                                          scale)
    return out


def partition_partials(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float,
                       partition_size: int):
    """Per-partition ``(m_p, l_p, acc_p)`` for one query row over contiguous K/V."""
    ctx = K.shape[0]
    parts = []
    for start in range(0, ctx, partition_size):
        Kp, Vp = K[start:start + partition_size], V[start:start + partition_size]
        z = scale * (Kp @ q)
        m = float(z.max())
        w = np.exp(z - m)
        parts.append((m, float(w.sum()), w @ Vp))
    return parts


def merge_partials(parts) -> np.ndarray:
    """Log-sum-exp merge of ``[(m_p, l_p, acc_p), ...]`` into the normalised output."""
    M = max(m for m, _, _ in parts)
    L = sum(l * math.exp(m - M) for m, l, _ in parts)
    acc = sum(a * math.exp(m - M) for m, _, a in parts)
    return acc / L


def paged_decode_split(q, k_cache, v_cache, block_tables, context_lens, scale, block_size,
                       partition_size, seqs=None, dtype=None):
    """Same result as :func:`paged_decode`, computed partition by partition and merged."""
    S, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.zeros((S, Hq, D), dtype=np.float64)
    for s in (range(S) if seqs is None else seqs):
        ctx = int(context_lens[s])
        if ctx == 0:
            continue
        for g in range(Hkv):
            K = _rows(k_cache, block_tables[s], ctx, g, block_size, dtype)
            V = _rows(v_cache, block_tables[s], ctx, g, block_size, dtype)
            for h in range(g * G, (g + 1) * G):
                out[s, h] = merge_partials(partition_partials(q[s, h], K, V, scale, partition_size))
    return out
