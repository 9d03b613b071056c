"""Oracle of the two cache-content operations on the paged KV pool.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py may use it.

Layout (a reading: the pages fix none): ``k_cache`` and ``v_cache`` are
separate arrays of shape ``[num_blocks, num_kv_heads, block_size, head_dim]``;
the slot ``s`` of a token is physical block ``s // block_size``, offset
``s % block_size`` inside it. Both functions move bits and are dtype-agnostic;
callers pass ``uint16`` bit patterns.

* :func:`reshape_and_cache` - each new token's K and V (all KV heads) goes to
  its slot; decode appends new cache state to the sequence ("PagedAttention KV
  cache memory management", section "A request lifecycle: allocation, growth,
  sharing and release"). A negative slot marks a padding token and is skipped.
* :func:`copy_blocks` - the copy half of block-level copy-on-write: the whole
  physical block (K and V, every head, every slot) is duplicated ("Your GPU was
  mostly empty", section "Paging's second gift: copy-on-write").
"""

from __future__ import annotations

import numpy as np


def reshape_and_cache(k_cache: np.ndarray, v_cache: np.ndarray, k_new: np.ndarray,
                      v_new: np.ndarray, slot_mapping, block_size: int) -> None:
    """In place: ``k_cache[s // bs, :, s % bs, :] = k_new[t]`` for every t with s >= 0."""
    num_blocks = k_cache.shape[0]
    for t, s in enumerate(np.asarray(slot_mapping, dtype=np.int64).tolist()):
        if s < 0:
            continue
        b, o = divmod(s, block_size)
        if b >= num_blocks:
            raise IndexError(f"slot {s} outside the pool")
        k_cache[b, :, o, :] = k_new[t]
        v_cache[b, :, o, :] = v_new[t]


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, pairs) -> None:
    """In place: for each (src, dst) in order, block dst becomes a copy of block src."""
    for src, dst in pairs:
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]
