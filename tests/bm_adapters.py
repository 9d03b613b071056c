"""Uniform driver interface over the two block managers, for trace tests.

The oracle adapter wraps :class:`oracle.block_manager.BlockManager`; the
library adapter wraps the C-ABI host allocator in ``libkvp.so``. Errors are
reported as the strings "oom", "no_seq", "invalid", "capacity".
"""

from oracle import block_manager as obm


class OracleBM:
    def __init__(self, num_blocks, block_size, free_order):
        self.bm = obm.BlockManager(num_blocks, block_size, free_order)

    def call(self, name, *args):
        try:
            return None, getattr(self.bm, name)(*args)
        except obm.OracleError as e:
            return e.code, None

    def free_list(self):
        return self.bm.free_list()

    def refcounts(self):
        return list(self.bm.rc)

    def table(self, seq):
        return self.bm.block_table(seq)

    def seq_len(self, seq):
        return self.bm.seq_len(seq)

    def pending(self):
        return self.bm.pending_copies()

    def stats(self):
        s = self.bm.stats()
        return (s.num_free, s.num_used, s.num_shared, s.waste_slots, s.cow_copies_total, s.num_seqs)


class LibBM:
    def __init__(self, num_blocks, block_size, free_order, num_kv_heads=1, head_dim=8, dtype="f16"):
        from paged_kv_cache_319_b200 import BlockPool

        self.bm = BlockPool(num_blocks, block_size, num_kv_heads, head_dim, dtype, free_order)

    def call(self, name, *args):
        from paged_kv_cache_319_b200 import KvpError

        try:
            return None, getattr(self.bm, name)(*args)
        except KvpError as e:
            return e.kind, None

    def free_list(self):
        return self.bm.free_list()

    def refcounts(self):
        return self.bm.refcounts()

    def table(self, seq):
        return self.bm.block_table(seq)

    def seq_len(self, seq):
        return self.bm.seq_len(seq)

    def pending(self):
        return self.bm.pending_copies()

    def stats(self):
        s = self.bm.stats()
        return (s["num_free"], s["num_used"], s["num_shared"], s["waste_slots"],
                s["cow_copies_total"], s["num_seqs"])
