"""Capacity and waste model of a KV cache.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py may use it.

* Per token, one layer holds one key and one value vector of ``hidden``
  elements, so the cache costs ``2 * hidden * layers * elem_bytes`` bytes per
  token across the model ("Your GPU was mostly empty", section "Why the KV
  cache is an allocator problem", worked OPT-13B example; "vLLM and
  PagedAttention", section "Production takeaways" asks for exactly this model).
* A paged sequence can waste space only in its last, partly filled block:
  ``num_blocks * block_size - length`` slots, at most ``block_size - 1``
  ("Your GPU was mostly empty", section "The OS already solved this in the
  1960s").
* A contiguous reservation sized to the maximum length wastes
  ``max_len - length`` slots ("Your GPU was mostly empty", section "Why the KV
  cache is an allocator problem", the 50-of-2,048 example).
"""

from __future__ import annotations


def kv_bytes_per_token(hidden: int, layers: int, elem_bytes: int) -> int:
    return 2 * hidden * layers * elem_bytes


def kv_bytes_per_sequence(tokens: int, hidden: int, layers: int, elem_bytes: int) -> int:
    return tokens * kv_bytes_per_token(hidden, layers, elem_bytes)


def block_bytes(num_kv_heads: int, block_size: int, head_dim: int, elem_bytes: int) -> int:
    """Bytes of one physical block in one layer: K and V, every KV head."""
    return 2 * num_kv_heads * block_size * head_dim * elem_bytes


def blocks_for(length: int, block_size: int) -> int:
    return -(-length // block_size)


def paged_waste_slots(length: int, block_size: int) -> int:
    return blocks_for(length, block_size) * block_size - length


def slab_waste_fraction(length: int, max_len: int) -> float:
    return (max_len - length) / max_len


def max_resident_sequences(kv_budget_bytes: int, tokens_per_seq: int, block_size: int,
                           bytes_per_token: int) -> int:
    """How many sequences of a given length fit, each rounded up to whole blocks."""
    per_seq = blocks_for(tokens_per_seq, block_size) * block_size * bytes_per_token
    return kv_budget_bytes // per_seq
