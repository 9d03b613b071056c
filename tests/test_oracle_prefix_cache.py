"""Pins of the prefix-caching block manager (oracle/block_manager.py,
PrefixCachingBlockManager): a hand-derived trace, and on random request streams the
property prefix caching exists for - every slot a sequence's table points at holds
that sequence's own token at that position, whether the block was computed by this
request or reused from another - plus the bookkeeping invariants."""

import numpy as np
import pytest

from oracle.block_manager import OutOfBlocks, PrefixCachingBlockManager


def test_hand_derived_trace():
    m = PrefixCachingBlockManager(8, 4)
    s0, c0 = m.create_prefixed(range(10))
    assert (s0, c0) == (0, 0)
    assert m.append_tokens(s0, range(10)) == list(range(10))  # blocks 0, 1, 2 in order
    assert m.block_table(s0) == [0, 1, 2] and m.cached_blocks() == 2  # the two full blocks
    # a second request with the same first 9 tokens reuses blocks 0 and 1 while s0 lives
    s1, c1 = m.create_prefixed(list(range(9)) + [99])
    assert (s1, c1) == (1, 8) and m.block_table(s1) == [0, 1] and m.refcount(0) == 2
    assert m.append_tokens(s1, [8, 99]) == [12, 13]  # block 3 (next on the stack)
    m.release(s0)
    assert m.free_list() == [2, 4, 5, 6, 7] and m.evictable() == []  # 0, 1 still held by s1
    m.release(s1)
    # s1's blocks: 3 is unregistered (partial) -> free; 1 then 0 become evictable
    assert m.free_list() == [3, 2, 4, 5, 6, 7] and m.evictable() == [1, 0]
    # a prompt of exactly 8 tokens reuses only block 0: its last token must be computed
    s2, c2 = m.create_prefixed(range(8))
    assert c2 == 4 and m.block_table(s2) == [0] and m.evictable() == [1]
    assert m.hit_tokens == 12


def test_eviction_takes_the_deepest_block_released_longest_ago():
    m = PrefixCachingBlockManager(4, 2)
    a, _ = m.create_prefixed([1, 2, 3, 4, 5])
    m.append_tokens(a, [1, 2, 3, 4, 5])  # blocks 0, 1 registered, 2 partial
    m.release(a)
    assert m.evictable() == [1, 0] and m.free_list() == [2, 3]
    b = m.create()
    m.append_tokens(b, [7, 7, 7, 7, 7])  # takes 2, 3, then evicts 1
    assert m.block_table(b) == [2, 3, 1] and m.evictable() == [0]
    # the prefix [1, 2] is still found; [1, 2, 3, 4] no longer
    c, hit = m.create_prefixed([1, 2, 3, 4, 9])
    assert hit == 2 and m.block_table(c) == [0]
    with pytest.raises(OutOfBlocks):
        m.append_tokens(c, [3, 4, 9, 9, 9])  # needs 3 blocks, none free or evictable


def test_a_block_after_an_unregistered_one_is_not_registered():
    """Two requests fill the same prefix at once: the first keeps the cache entry, the
    second's copy stays private, and so does every block after it."""
    m = PrefixCachingBlockManager(8, 2)
    a, b = m.create(), m.create()
    m.append_tokens(a, [1, 2])
    m.append_tokens(b, [1, 2, 3, 4])  # b's first block duplicates a's: not registered
    m.append_tokens(a, [3, 4])
    assert m.cached_blocks() == 2 and set(m._key_of) == set(m.block_table(a))
    m.release(b)  # b's blocks were private: straight to the free stack
    assert m.evictable() == [] and m.num_free() == 6
    c, hit = m.create_prefixed([1, 2, 3, 4, 5])
    assert hit == 4 and m.block_table(c) == m.block_table(a)


def test_plain_append_stops_registration():
    m = PrefixCachingBlockManager(6, 2)
    s = m.create()
    m.append_tokens(s, [1, 2, 3])
    m.append(s, 3)  # unknown tokens from here on
    assert m.cached_blocks() == 1
    m.release(s)
    assert m.evictable() == [0] and sorted(m.free_list()) == [1, 2, 3, 4, 5]


def _random_stream(seed, steps=400, NB=48, bs=4):
    """Requests over a small vocabulary with shared system prompts, forks, decode
    appends, releases; yields the manager and a shadow of every slot's token."""
    rng = np.random.default_rng(seed)
    m = PrefixCachingBlockManager(NB, bs, rng.permutation(NB).tolist())
    content = np.full(NB * bs, -1, np.int64)
    hist = {}
    systems = [rng.integers(0, 5, size=int(rng.integers(3, 14))).tolist() for _ in range(3)]
    for _ in range(steps):
        op = rng.random()
        live = m.live_seqs()
        try:
            if op < 0.35 or not live:
                prompt = list(systems[int(rng.integers(0, 3))]) + \
                    rng.integers(0, 5, size=int(rng.integers(1, 6))).tolist()
                if rng.random() < 0.2:
                    prompt = rng.integers(0, 5, size=int(rng.integers(1, 12))).tolist()
                need = -(-len(prompt) // bs)
                if need > m.available():
                    continue
                s, cached = m.create_prefixed(prompt)
                hist[s] = list(prompt[:cached])
                slots = m.append_tokens(s, prompt[cached:])
                content[slots] = prompt[cached:]
                hist[s] += prompt[cached:]
            elif op < 0.75:
                s = live[int(rng.integers(0, len(live)))]
                tok = rng.integers(0, 5, size=int(rng.integers(1, 4))).tolist()
                slots = m.append_tokens(s, tok)
                for src, dst in m.take_copies():  # copy-on-write: the copy happens before the write
                    content[dst * bs:(dst + 1) * bs] = content[src * bs:(src + 1) * bs]
                content[slots] = tok
                hist[s] += tok
            elif op < 0.82:
                s = live[int(rng.integers(0, len(live)))]
                c = m.fork(s)
                hist[c] = list(hist[s])
            else:
                s = live[int(rng.integers(0, len(live)))]
                m.release(s)
                del hist[s]
        except OutOfBlocks:
            m.take_copies()
            continue
        yield m, content, hist


@pytest.mark.parametrize("seed", [1, 2, 3, 4])
def test_every_table_slot_holds_the_sequence_own_tokens(seed):
    hits = 0
    for m, content, hist in _random_stream(seed):
        bs = m.block_size
        for s in m.live_seqs():
            t = m.block_table(s)
            L = m.seq_len(s)
            got = [int(content[t[p // bs] * bs + p % bs]) for p in range(L)]
            assert got == hist[s], f"sequence {s}"
        hits = m.hit_tokens
    assert hits > 0  # the stream did reuse cached prefixes


@pytest.mark.parametrize("seed", [5, 6])
def test_bookkeeping_invariants(seed):
    for m, content, hist in _random_stream(seed):
        NB, bs = m.num_blocks, m.block_size
        refs = [0] * NB
        for s in m.live_seqs():
            for b in m.block_table(s):
                refs[b] += 1
        assert refs == [m.refcount(b) for b in range(NB)]
        free, ev = set(m.free_list()), set(m.evictable())
        used = {b for b in range(NB) if refs[b] > 0}
        assert not (free & ev) and not (free & used) and not (ev & used)
        assert len(free) + len(ev) + len(used) == NB
        for b in ev:
            assert b in m._key_of  # only registered blocks wait for reuse
        for b, (parent, toks) in m._key_of.items():
            assert [int(x) for x in content[b * bs:(b + 1) * bs]] == list(toks)
            assert parent == -1 or parent < m._reg_of[b]  # parents were registered first
