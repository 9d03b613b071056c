"""Oracle of the host-side KV block manager (fp-free, integer bookkeeping).

TEST INFRASTRUCTURE: only tests/, __graft_entry__.smoke() and bench.py may use it.

What it restates:

* Fixed-size physical blocks, a per-sequence block table mapping logical block
  numbers to physical ones, and allocation only when a sequence grows into a
  new block - "Your GPU was mostly empty", section "The OS already solved this
  in the 1960s"; "vLLM and PagedAttention", section "Architecture, step by
  step" (steps 1 and 2); "PagedAttention KV cache memory management", section
  "How logical blocks, physical blocks and the block table work".
* Sharing by reference count and block-level copy-on-write when a sequence
  writes into a block that another sequence also references - "Your GPU was
  mostly empty", section "Paging's second gift: copy-on-write".
* Release: a block that no live sequence references goes back to the shared
  pool - "PagedAttention KV cache memory management", sections "How logical
  blocks, physical blocks and the block table work" and "A request lifecycle:
  allocation, growth, sharing and release".

The pages leave the allocation *policy* open. This oracle pins one reading so
that the CUDA library's host code can be compared with it bit for bit:

1. The free pool is a stack. At creation it holds a caller-given permutation
   of ``0..num_blocks-1`` arranged so that the first block handed out is
   ``free_order[0]`` (identity order when none is given).
2. ``append(seq, n)`` writes ``n`` tokens one after another. A token at
   position ``pos`` with ``pos % block_size == 0`` takes a new block from the
   pool. Otherwise, if the last block is shared (reference count > 1), the
   writer takes a new block, a copy (old -> new) is queued, the old block's
   count drops by one and the writer's table points to the new block. Its
   slot is ``table[pos // block_size] * block_size + pos % block_size``.
   The whole call fails, with nothing changed, if the pool cannot supply every
   block it needs.
3. ``fork(parent)`` gives the child the parent's table and length and adds one
   reference to every block in it.
4. ``release(seq)`` drops one reference from each block in logical order and
   pushes every block that reaches zero onto the pool stack.
5. ``take_copies()`` returns the queued copy pairs in creation order and
   clears the queue.
6. Sequence ids are handed out as 0, 1, 2, ... and never reused.
"""

from __future__ import annotations

from dataclasses import dataclass


class OracleError(Exception):
    """Base class; ``code`` mirrors the status a C caller would see."""

    code = "invalid"


class InvalidArgument(OracleError):
    code = "invalid"


class OutOfBlocks(OracleError):
    code = "oom"


class NoSuchSequence(OracleError):
    code = "no_seq"


class CapacityTooSmall(OracleError):
    code = "capacity"


@dataclass
class PoolStats:
    num_free: int
    num_used: int
    num_shared: int
    waste_slots: int
    cow_copies_total: int
    num_seqs: int


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


class BlockManager:
    """Refcounted paged-KV block allocator (pinned policy in the module doc)."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise InvalidArgument("num_blocks and block_size must be positive")
        if free_order is None:
            order = list(range(num_blocks))
        else:
            order = [int(b) for b in free_order]
            if sorted(order) != list(range(num_blocks)):
                raise InvalidArgument("free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.block_size = block_size
        # Stack: the end of the list is the top, i.e. the next block handed out.
        self._free = order[::-1]
        self.rc = [0] * num_blocks
        self._tables: dict[int, list[int]] = {}
        self._lens: dict[int, int] = {}
        self._pending: list[tuple[int, int]] = []
        self._next_seq = 0
        self._cow_total = 0

    # ---- queries -----------------------------------------------------------
    def num_free(self) -> int:
        return len(self._free)

    def free_list(self) -> list[int]:
        """Free blocks in the order they would be handed out."""
        return self._free[::-1]

    def refcount(self, block: int) -> int:
        if not 0 <= block < self.num_blocks:
            raise InvalidArgument("block id out of range")
        return self.rc[block]

    def seq_len(self, seq: int) -> int:
        self._check(seq)
        return self._lens[seq]

    def block_table(self, seq: int) -> list[int]:
        self._check(seq)
        return list(self._tables[seq])

    def live_seqs(self) -> list[int]:
        return sorted(self._tables)

    def pending_copies(self) -> list[tuple[int, int]]:
        return list(self._pending)

    def stats(self) -> PoolStats:
        used = sum(1 for c in self.rc if c > 0)
        shared = sum(1 for c in self.rc if c > 1)
        waste = sum(len(t) * self.block_size - self._lens[s] for s, t in self._tables.items())
        return PoolStats(len(self._free), used, shared, waste, self._cow_total, len(self._tables))

    # ---- mutations ---------------------------------------------------------
    def create(self) -> int:
        seq = self._next_seq
        self._next_seq += 1
        self._tables[seq] = []
        self._lens[seq] = 0
        return seq

    def blocks_needed(self, seq: int, n: int) -> int:
        """Blocks ``append(seq, n)`` would take from the pool."""
        self._check(seq)
        table, length = self._tables[seq], self._lens[seq]
        bs = self.block_size
        need = _ceil_div(length + n, bs) - _ceil_div(length, bs)
        if n > 0 and length % bs != 0 and self.rc[table[-1]] > 1:
            need += 1  # the first token lands in a shared, partly filled block
        return need

    def append(self, seq: int, n: int) -> list[int]:
        self._check(seq)
        if n < 0:
            raise InvalidArgument("n must be >= 0")
        if self.blocks_needed(seq, n) > len(self._free):
            raise OutOfBlocks("not enough free blocks")
        table = self._tables[seq]
        bs = self.block_size
        slots = []
        for _ in range(n):
            pos = self._lens[seq]
            if pos % bs == 0:
                b = self._free.pop()
                self.rc[b] = 1
                table.append(b)
            elif self.rc[table[-1]] > 1:
                src = table[-1]
                dst = self._free.pop()
                self._pending.append((src, dst))
                self._cow_total += 1
                self.rc[src] -= 1
                self.rc[dst] = 1
                table[-1] = dst
            slots.append(table[pos // bs] * bs + pos % bs)
            self._lens[seq] = pos + 1
        return slots

    def fork(self, parent: int) -> int:
        self._check(parent)
        child = self._next_seq
        self._next_seq += 1
        self._tables[child] = list(self._tables[parent])
        self._lens[child] = self._lens[parent]
        for b in self._tables[child]:
            self.rc[b] += 1
        return child

    def release(self, seq: int) -> None:
        self._check(seq)
        for b in self._tables.pop(seq):
            self.rc[b] -= 1
            if self.rc[b] == 0:
                self._free.append(b)
        del self._lens[seq]

    def take_copies(self) -> list[tuple[int, int]]:
        out, self._pending = self._pending, []
        return out

    def build_batch(self, seqs, max_blocks: int):
        """Block tables padded with -1 to ``max_blocks`` columns, and lengths."""
        tables, lens = [], []
        for s in seqs:
            self._check(s)
            t = self._tables[s]
            if len(t) > max_blocks:
                raise CapacityTooSmall("max_blocks smaller than a block table")
            tables.append(t + [-1] * (max_blocks - len(t)))
            lens.append(self._lens[s])
        return tables, lens

    def _check(self, seq: int) -> None:
        if seq not in self._tables:
            raise NoSuchSequence(f"no live sequence {seq}")


class PrefixCachingBlockManager(BlockManager):
    """The block manager with prefix caching across requests: full blocks keep the
    keys and values of a token prefix that a later request with the same prefix
    reuses instead of recomputing ("PagedAttention: KV cache memory management",
    section "PagedAttention vs KV-cache quantization vs prefix caching"; sharing
    across requests: "vLLM and PagedAttention", section "Key claims from the
    paper"). The pages give no policy; this oracle pins one (readings 7-13, on top
    of 1-6 of the module doc):

    7. A full block is cached under the key (parent, tokens): ``tokens`` are its
       ``block_size`` token ids and ``parent`` is the registration number of the
       block before it in the table that filled it (-1 for a first block).
       Registrations are numbered 0, 1, 2, ... and numbers are never reused, so
       a key names one exact token prefix: a match means the whole prefix up to
       that block is equal (by induction over the parents), even after a parent
       block was evicted and its physical block reused.
    8. ``append_tokens(seq, tokens)`` is ``append`` with the token ids given;
       whenever a token fills a block, that block is registered under its key
       unless the key is taken (another request computed the same prefix: the
       first registration stays), the block is registered already, or the block
       before it is not registered (then no lookup can reach it). A plain
       ``append`` on a sequence stops its registration for good (its later
       tokens are unknown).
    9. ``create_prefixed(tokens)`` creates a sequence holding the longest run of
       leading cached blocks of ``tokens`` whose tokens end before the prompt's
       last one (the last prompt token is always computed): each matched block
       gains a reference. It returns (sequence, cached tokens); the caller
       appends ``tokens[cached:]`` with ``append_tokens``.
    10. ``release`` drops references in logical order; a block reaching zero goes
        to the free stack if it is not registered, else it becomes evictable.
        The blocks of one release become evictable from the last logical block
        to the first, so the deepest blocks of a prefix are evicted first.
    11. A new block comes from the free stack; when it is empty, the evictable
        block released longest ago is evicted (its key dropped) and used.
        Capacity checks count free and evictable blocks.
    12. A lookup that matches an evictable block takes it back (it leaves the
        evictable list).
    13. ``fork`` copies the parent's tokens and registration state.
    """

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        super().__init__(num_blocks, block_size, free_order)
        self._key_of: dict[int, tuple] = {}     # registered block -> key
        self._block_of: dict[tuple, int] = {}   # key -> registered block
        self._reg_of: dict[int, int] = {}       # registered block -> registration number
        self._next_reg = 0
        self._evictable: list[int] = []         # front = evicted next
        self._tokens: dict[int, list[int]] = {}  # tracked sequences' token ids
        self.hit_tokens = 0

    # ---- queries -----------------------------------------------------------
    def evictable(self) -> list[int]:
        return list(self._evictable)

    def cached_blocks(self) -> int:
        return len(self._key_of)

    def available(self) -> int:
        return len(self._free) + len(self._evictable)

    # ---- mutations ---------------------------------------------------------
    def _take(self) -> int:
        if self._free:
            return self._free.pop()
        b = self._evictable.pop(0)
        del self._block_of[self._key_of.pop(b)]
        del self._reg_of[b]
        return b

    def create(self) -> int:
        seq = super().create()
        self._tokens[seq] = []
        return seq

    def create_prefixed(self, tokens) -> tuple[int, int]:
        tokens = [int(t) for t in tokens]
        seq = self.create()
        bs = self.block_size
        table = self._tables[seq]
        parent = -1
        i = 0
        while (i + 1) * bs <= len(tokens) - 1:
            b = self._block_of.get((parent, tuple(tokens[i * bs:(i + 1) * bs])))
            if b is None:
                break
            if self.rc[b] == 0:
                self._evictable.remove(b)
            self.rc[b] += 1
            table.append(b)
            parent = self._reg_of[b]
            i += 1
        self._lens[seq] = i * bs
        self._tokens[seq] = tokens[:i * bs]
        self.hit_tokens += i * bs
        return seq, i * bs

    def blocks_needed(self, seq: int, n: int) -> int:
        return super().blocks_needed(seq, n)

    def append_tokens(self, seq: int, tokens) -> list[int]:
        tokens = [int(t) for t in tokens]
        return self._append(seq, len(tokens), tokens)

    def append(self, seq: int, n: int) -> list[int]:
        return self._append(seq, n, None)

    def _append(self, seq, n, tokens):
        self._check(seq)
        if n < 0:
            raise InvalidArgument("n must be >= 0")
        if self.blocks_needed(seq, n) > self.available():
            raise OutOfBlocks("not enough free blocks")
        if tokens is None:
            self._tokens.pop(seq, None)  # reading 8: registration stops
        table = self._tables[seq]
        bs = self.block_size
        slots = []
        for k in range(n):
            pos = self._lens[seq]
            if pos % bs == 0:
                b = self._take()
                self.rc[b] = 1
                table.append(b)
            elif self.rc[table[-1]] > 1:
                src = table[-1]
                dst = self._take()
                self._pending.append((src, dst))
                self._cow_total += 1
                self.rc[src] -= 1
                self.rc[dst] = 1
                table[-1] = dst
            slots.append(table[pos // bs] * bs + pos % bs)
            self._lens[seq] = pos + 1
            if seq in self._tokens:
                self._tokens[seq].append(tokens[k])
                if (pos + 1) % bs == 0:
                    blk = table[pos // bs]
                    prev = table[pos // bs - 1] if pos // bs > 0 else None
                    parent = -1 if prev is None else self._reg_of.get(prev)
                    key = (parent, tuple(self._tokens[seq][pos + 1 - bs:pos + 1]))
                    if parent is not None and key not in self._block_of and blk not in self._key_of:
                        self._block_of[key] = blk
                        self._key_of[blk] = key
                        self._reg_of[blk] = self._next_reg
                        self._next_reg += 1
        return slots

    def fork(self, parent: int) -> int:
        child = super().fork(parent)
        if parent in self._tokens:
            self._tokens[child] = list(self._tokens[parent])
        return child

    def release(self, seq: int) -> None:
        self._check(seq)
        newly = []
        for b in self._tables.pop(seq):
            self.rc[b] -= 1
            if self.rc[b] == 0:
                if b in self._key_of:
                    newly.append(b)
                else:
                    self._free.append(b)
        self._evictable.extend(reversed(newly))
        del self._lens[seq]
        self._tokens.pop(seq, None)
