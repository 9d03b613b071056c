"""The library's prefix caching (kv_pool_set_prefix_caching, kv_seq_create_prefixed,
kv_seq_append_tokens and its batch form, evictable blocks) against the oracle's PrefixCachingBlockManager,
operation by operation on random request streams: block tables, slots, reference
counts, the free stack, the evictable list, copy-on-write pairs and the cached-token
counts must agree exactly. Also: the switch's rules, and that a pool without prefix
caching behaves as before."""

import copy

import numpy as np
import pytest

import paged_kv_cache_319_b200 as kvp
from oracle.block_manager import OutOfBlocks, PrefixCachingBlockManager


def _pair(NB, bs, seed):
    order = np.random.default_rng(seed).permutation(NB).tolist()
    lib = kvp.BlockPool(NB, bs, 2, 64, free_order=order)
    lib.set_prefix_caching(True)
    return lib, PrefixCachingBlockManager(NB, bs, order)


def _same(lib, ora):
    assert lib.free_list() == ora.free_list()
    assert lib.evictable() == ora.evictable()
    assert lib.refcounts() == [ora.refcount(b) for b in range(ora.num_blocks)]
    assert lib.pending_copies() == ora.pending_copies()
    st = lib.prefix_stats()
    assert (st["registered"], st["evictable"], st["hit_tokens"]) == \
        (ora.cached_blocks(), len(ora.evictable()), ora.hit_tokens)
    for s in ora.live_seqs():
        assert lib.block_table(s) == ora.block_table(s) and lib.seq_len(s) == ora.seq_len(s)


@pytest.mark.parametrize("seed,NB,bs", [(1, 40, 4), (2, 24, 2), (3, 64, 8), (4, 16, 4)])
def test_random_streams_match_the_oracle(seed, NB, bs):
    rng = np.random.default_rng(100 + seed)
    lib, ora = _pair(NB, bs, seed)
    systems = [rng.integers(0, 4, size=int(rng.integers(2, 3 * bs))).tolist() for _ in range(3)]
    hits = 0
    for _ in range(500):
        op = rng.random()
        live = ora.live_seqs()
        if op < 0.3 or not live:
            prompt = list(systems[int(rng.integers(0, 3))]) + \
                rng.integers(0, 4, size=int(rng.integers(1, bs + 2))).tolist()
            s1, c1 = ora.create_prefixed(prompt)
            s2, c2 = lib.create_prefixed(prompt)
            assert (s1, c1) == (s2, c2)
            try:
                sl1 = ora.append_tokens(s1, prompt[c1:])
            except OutOfBlocks:
                with pytest.raises(kvp.KvpError):
                    lib.append_tokens(s2, prompt[c2:])
                ora.release(s1)
                lib.release(s2)
            else:
                assert lib.append_tokens(s2, prompt[c2:]) == sl1
        elif op < 0.6:
            s = live[int(rng.integers(0, len(live)))]
            tok = rng.integers(0, 4, size=int(rng.integers(1, bs + 1))).tolist()
            plain = rng.random() < 0.05
            try:
                sl1 = ora.append(s, len(tok)) if plain else ora.append_tokens(s, tok)
            except OutOfBlocks:
                with pytest.raises(kvp.KvpError):
                    lib.append(s, len(tok)) if plain else lib.append_tokens(s, tok)
            else:
                assert (lib.append(s, len(tok)) if plain else lib.append_tokens(s, tok)) == sl1
        elif op < 0.64:  # a decode step of several sequences at once
            pick = sorted(rng.choice(live, size=min(len(live), int(rng.integers(1, 5))),
                                     replace=False).tolist())
            n_each = int(rng.integers(1, 3))
            tok = rng.integers(0, 4, size=(len(pick), n_each))
            trial = copy.deepcopy(ora)
            try:
                want = [x for s, t in zip(pick, tok) for x in trial.append_tokens(s, t.tolist())]
            except OutOfBlocks:
                with pytest.raises(kvp.KvpError):
                    lib.append_tokens_batch(pick, tok)
            else:
                assert lib.append_tokens_batch(pick, tok).tolist() == want
                ora = trial
        elif op < 0.68:
            s = live[int(rng.integers(0, len(live)))]
            assert lib.fork(s) == ora.fork(s)
        elif op < 0.75:
            assert lib.take_copies() == ora.take_copies()
        else:
            s = live[int(rng.integers(0, len(live)))]
            ora.release(s)
            lib.release(s)
        _same(lib, ora)
        hits = ora.hit_tokens
    assert hits > 0


def test_switch_rules():
    lib = kvp.BlockPool(8, 2, 1, 64)
    s = lib.create()
    with pytest.raises(kvp.KvpError):
        lib.set_prefix_caching(True)  # a live sequence
    with pytest.raises(kvp.KvpError):
        lib.create_prefixed([1, 2, 3])  # still off
    lib.release(s)
    lib.set_prefix_caching(True)
    a, _ = lib.create_prefixed([1, 2, 3, 4, 5])
    lib.append_tokens(a, [1, 2, 3, 4, 5])
    lib.release(a)
    assert sorted(lib.evictable()) == [0, 1]
    lib.set_prefix_caching(False)  # evictable blocks become free, registrations go
    assert lib.evictable() == [] and lib.num_free() == 8
    assert lib.prefix_stats()["registered"] == 0


def test_without_prefix_caching_release_frees_every_block():
    lib = kvp.BlockPool(6, 2, 1, 64)
    s = lib.create()
    lib.append_tokens(s, [1, 2, 3, 4])
    lib.release(s)
    assert lib.evictable() == [] and lib.free_list() == [1, 0, 2, 3, 4, 5]
