"""Driver of tests/test_host_sanitized.py (run in a child process whose host library
was built with AddressSanitizer and UndefinedBehaviorSanitizer): random pool and
prefix-cache streams through the library's C API, checked step by step against the
oracle (slots, block tables, free and evictable lists, copy-on-write pairs).

Usage: python host_sanitizer_driver.py <path of the sanitized host library>
"""
import copy
import ctypes as C
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
from oracle.block_manager import BlockManager, OutOfBlocks, PrefixCachingBlockManager  # noqa: E402

L = C.CDLL(sys.argv[1])
P32, P64 = C.POINTER(C.c_int32), C.POINTER(C.c_int64)
def arr32(x): a = np.ascontiguousarray(np.asarray(x, np.int32)); return a, a.ctypes.data_as(P32)
def run(seed, NB, bs, caching):
    rng = np.random.default_rng(seed)
    order = rng.permutation(NB).astype(np.int32)
    pool = C.c_void_p()
    assert L.kv_pool_create(NB, bs, 2, 64, 0, order.ctypes.data_as(P32), C.byref(pool)) == 0
    if caching: assert L.kv_pool_set_prefix_caching(pool, 1) == 0
    ora = (PrefixCachingBlockManager if caching else BlockManager)(NB, bs, order.tolist())
    systems = [rng.integers(0, 4, size=int(rng.integers(2, 3 * bs))).tolist() for _ in range(3)]
    def table(s):
        n = C.c_int32(); buf = np.zeros(NB, np.int32)
        assert L.kv_seq_block_table(pool, C.c_int64(s), buf.ctypes.data_as(P32), NB, C.byref(n)) == 0
        return buf[:n.value].tolist()
    def lists():
        n = C.c_int32(); buf = np.zeros(NB, np.int32)
        assert L.kv_pool_free_list(pool, buf.ctypes.data_as(P32), NB, C.byref(n)) == 0
        free = buf[:n.value].tolist()
        ev = []
        if caching:
            assert L.kv_pool_evictable_list(pool, buf.ctypes.data_as(P32), NB, C.byref(n)) == 0
            ev = buf[:n.value].tolist()
        return free, ev
    for step in range(600):
        live = ora.live_seqs(); op = rng.random()
        if op < 0.3 or not live:
            prompt = list(systems[int(rng.integers(0, 3))]) + rng.integers(0, 4, size=int(rng.integers(1, bs + 2))).tolist()
            if caching:
                s1, c1 = ora.create_prefixed(prompt)
                t, tp = arr32(prompt); sid, cached = C.c_int64(), C.c_int32()
                assert L.kv_seq_create_prefixed(pool, tp, len(prompt), C.byref(sid), C.byref(cached)) == 0
                assert (sid.value, cached.value) == (s1, c1)
            else:
                s1 = ora.create(); c1 = 0; sid = C.c_int64()
                assert L.kv_seq_create(pool, C.byref(sid)) == 0 and sid.value == s1
            rest = prompt[c1:]; t, tp = arr32(rest); out = np.zeros(len(rest), np.int64)
            try:
                want = ora.append_tokens(s1, rest) if caching else ora.append(s1, len(rest))
            except OutOfBlocks:
                rc = L.kv_seq_append_tokens(pool, C.c_int64(s1), tp, len(rest), out.ctypes.data_as(P64))
                assert rc == -2
                ora.release(s1); assert L.kv_seq_release(pool, C.c_int64(s1)) == 0
            else:
                rc = L.kv_seq_append_tokens(pool, C.c_int64(s1), tp, len(rest), out.ctypes.data_as(P64))
                assert rc == 0 and out.tolist() == want
        elif op < 0.55:
            pick = sorted(rng.choice(live, size=min(len(live), int(rng.integers(1, 5))), replace=False).tolist())
            n_each = int(rng.integers(1, 3)); tok = rng.integers(0, 4, size=(len(pick), n_each))
            trial = copy.deepcopy(ora)
            seqs = np.asarray(pick, np.int64); t, tp = arr32(tok.reshape(-1)); out = np.zeros(len(pick) * n_each, np.int64)
            try:
                want = [x for s, tt in zip(pick, tok) for x in (trial.append_tokens(s, tt.tolist()) if caching else trial.append(s, n_each))]
            except OutOfBlocks:
                rc = L.kv_seq_append_tokens_batch(pool, seqs.ctypes.data_as(P64), len(pick), n_each, tp, out.ctypes.data_as(P64))
                assert rc == -2
            else:
                rc = L.kv_seq_append_tokens_batch(pool, seqs.ctypes.data_as(P64), len(pick), n_each, tp, out.ctypes.data_as(P64))
                assert rc == 0 and out.tolist() == want; ora = trial
        elif op < 0.62:
            s = live[int(rng.integers(0, len(live)))]; cid = C.c_int64()
            assert L.kv_seq_fork(pool, C.c_int64(s), C.byref(cid)) == 0 and cid.value == ora.fork(s)
        elif op < 0.7:
            n = C.c_int32(); buf = np.zeros(2 * NB + 2, np.int32)
            assert L.kv_pool_take_copies(pool, buf.ctypes.data_as(P32), NB + 1, C.byref(n)) == 0
            got = [(int(buf[2 * i]), int(buf[2 * i + 1])) for i in range(n.value)]
            assert got == ora.take_copies()
        else:
            s = live[int(rng.integers(0, len(live)))]
            ora.release(s); assert L.kv_seq_release(pool, C.c_int64(s)) == 0
        free, ev = lists()
        assert free == ora.free_list(), (step, free, ora.free_list())
        if caching: assert ev == ora.evictable()
        for s in ora.live_seqs(): assert table(s) == ora.block_table(s)
    # the grouping planner over the live batch (forks and cached prefixes share first blocks)
    live = ora.live_seqs()
    if live:
        S, MB = len(live), max(1, max(len(ora.block_table(s)) for s in live))
        seqs = np.asarray(live, np.int64)
        tables = np.zeros((S, MB), np.int32)
        lens = np.zeros(S, np.int32)
        assert L.kv_build_batch(pool, seqs.ctypes.data_as(P64), S, MB, tables.ctypes.data_as(P32),
                                lens.ctypes.data_as(P32)) == 0
        L.kvp_decode_group_plan_words.restype = C.c_size_t
        words = L.kvp_decode_group_plan_words(S)
        plan = np.zeros(words, np.int32)
        rc = L.kv_decode_group_plan(tables.ctypes.data_as(P32), lens.ctypes.data_as(P32), S, MB,
                                    MB * bs, bs, 4 * bs, 8, 8, NB, plan.ctypes.data_as(P32),
                                    C.c_size_t(words))
        assert rc == 0
        assert plan[0] <= S // 2 + 1  # subgroups of two or more members
    if caching:
        assert L.kv_pool_set_prefix_caching(pool, 0) == 0
    assert L.kv_pool_destroy(pool) == 0
    return ora
if __name__ == "__main__":
    for seed in range(12):
        for caching in (True, False):
            NB, bs = [(40, 4), (24, 2), (64, 8), (16, 4)][seed % 4]
            run(seed, NB, bs, caching)
    print("sanitized host streams ok")
