"""Replays a workload's operation schedule through the oracle.

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py may use it.

Per decode step the order is: copy-on-write copies, then the new tokens'
K/V into their slots, then attention ("PagedAttention KV cache memory
management", section "A request lifecycle: allocation, growth, sharing and
release"; "Your GPU was mostly empty", section "Paging's second gift:
copy-on-write"). The copies go first because a token may land in a block
that was copied in the same step.

Inputs come from :mod:`workloads` (values keyed by the op's index); nothing
here reads a result of the CUDA library.
"""

from __future__ import annotations

import numpy as np

from workloads.values import K_STREAM, Q_STREAM, V_STREAM, normal_bits, value_seed_words

from . import attention, cache
from .block_manager import BlockManager
from .numerics import to_f64


class OracleReplay:
    """Oracle block manager + oracle cache + oracle attention over one workload."""

    def __init__(self, wl, with_cache: bool = True):
        g = wl.geometry
        self.wl = wl
        self.g = g
        self.bm = BlockManager(wl.num_blocks, g.block_size, wl.free_order)
        self.ids: dict[int, int] = {}
        self.with_cache = with_cache
        if with_cache:
            shape = (wl.num_blocks, g.num_kv_heads, g.block_size, g.head_dim)
            self.k_cache = np.zeros(shape, dtype=np.uint16)
            self.v_cache = np.zeros(shape, dtype=np.uint16)
        self._pending = []          # [(slots, op_index, n)]
        self.events = []            # [(op_index, kind, payload)]
        self.attends = []           # [(op_index, seq ids, block_tables, context_lens)]
        self.next_index = 0

    def kv_values(self, op_index: int, n: int):
        g = self.g
        shape = (n, g.num_kv_heads, g.head_dim)
        k = normal_bits(value_seed_words(self.wl.value_seed, K_STREAM, op_index), shape, g.dtype)
        v = normal_bits(value_seed_words(self.wl.value_seed, V_STREAM, op_index), shape, g.dtype)
        return k, v

    def q_values(self, op_index: int, num_seqs: int):
        g = self.g
        shape = (num_seqs, g.num_q_heads, g.head_dim)
        return normal_bits(value_seed_words(self.wl.value_seed, Q_STREAM, op_index), shape, g.dtype)

    def run(self, ops=None, attend=None, start_index=None):
        """Apply ``ops`` (default: the workload's own). ``attend(op_index, ids, tables, lens)``
        is called at every attend op; by default the batch metadata is recorded."""
        ops = self.wl.ops if ops is None else ops
        i = self.next_index if start_index is None else start_index
        for op in ops:
            self._apply(i, op, attend)
            i += 1
        self.next_index = i

    def _apply(self, i, op, attend):
        kind = op[0]
        bm = self.bm
        if kind == "create":
            self.ids[op[1]] = bm.create()
            self.events.append((i, "create", self.ids[op[1]]))
        elif kind == "append":
            slots = bm.append(self.ids[op[1]], op[2])
            self._pending.append((slots, i, op[2]))
            self.events.append((i, "append", slots))
        elif kind == "fork":
            self.ids[op[2]] = bm.fork(self.ids[op[1]])
            self.events.append((i, "fork", self.ids[op[2]]))
        elif kind == "release":
            bm.release(self.ids[op[1]])
            self.events.append((i, "release", None))
        elif kind == "sync":
            copies = bm.take_copies()
            self.events.append((i, "sync", copies))
            if self.with_cache:
                cache.copy_blocks(self.k_cache, self.v_cache, copies)
                for slots, j, n in self._pending:
                    if n:
                        k, v = self.kv_values(j, n)
                        cache.reshape_and_cache(self.k_cache, self.v_cache, k, v, slots,
                                                self.g.block_size)
            self._pending = []
        elif kind == "attend":
            seqs = [self.ids[h] for h in op[1]]
            max_blocks = max(1, max(len(bm.block_table(s)) for s in seqs))
            tables, lens = bm.build_batch(seqs, max_blocks)
            self.attends.append((i, seqs, tables, lens))
            if attend is not None:
                attend(i, seqs, np.asarray(tables, np.int32), np.asarray(lens, np.int32))
        else:
            raise ValueError(f"unknown op {op!r}")

    def decode(self, op_index, tables, lens, seqs=None, split=False):
        """fp64 attention output ``[S, Hq, D]`` of the attend op at ``op_index``."""
        q = to_f64(self.q_values(op_index, len(lens)), self.g.dtype)
        if split and self.wl.partition_size:
            return attention.paged_decode_split(q, self.k_cache, self.v_cache, tables, lens,
                                                self.wl.scale, self.g.block_size,
                                                self.wl.partition_size, seqs=seqs,
                                                dtype=self.g.dtype)
        return attention.paged_decode(q, self.k_cache, self.v_cache, tables, lens, self.wl.scale,
                                      self.g.block_size, seqs=seqs, dtype=self.g.dtype)
