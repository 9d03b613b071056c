"""The C++ host allocator of libkvp against the oracle: bit-exact bookkeeping (CPU only)."""

import random

import numpy as np
import pytest

from bm_adapters import LibBM, OracleBM
from test_oracle_block_manager import run_trace
import workloads


def test_hand_trace_library():
    run_trace(LibBM)


def state(bm, live):
    return (bm.free_list(), bm.refcounts(), [(s, bm.table(s), bm.seq_len(s)) for s in live],
            bm.pending(), bm.stats())


@pytest.mark.parametrize("seed", range(8))
def test_random_schedules_bit_exact(seed):
    rnd = random.Random(100 + seed)
    nb, bs = rnd.choice([(16, 2), (64, 4), (200, 16)])
    order = rnd.sample(range(nb), nb)
    a, b = OracleBM(nb, bs, order), LibBM(nb, bs, order)
    live = []
    for _ in range(500):
        r = rnd.random()
        if r < 0.15 or not live:
            op = ("create",)
        elif r < 0.55:
            op = ("append", rnd.choice(live), rnd.randint(0, 3 * bs))
        elif r < 0.7:
            op = ("fork", rnd.choice(live))
        elif r < 0.85:
            op = ("release", rnd.choice(live + [10**6]))
        elif r < 0.95:
            op = ("take_copies",)
        else:
            op = ("append", rnd.choice(live), -1)
        ra, rb = a.call(op[0], *op[1:]), b.call(op[0], *op[1:])
        assert ra[0] == rb[0], (op, ra, rb)
        if ra[0] is None:
            if op[0] == "take_copies":
                assert [tuple(p) for p in ra[1]] == [tuple(p) for p in rb[1]]
            else:
                assert ra[1] == rb[1], op
            if op[0] in ("create", "fork"):
                live.append(ra[1])
            if op[0] == "release":
                live.remove(op[1])
        assert state(a, live) == state(b, live), op


def test_batch_append_equals_sequential_and_is_atomic():
    import paged_kv_cache_319_b200 as kvp

    p1 = kvp.BlockPool(40, 4, 1, 8, "f16", list(range(40)))
    p2 = kvp.BlockPool(40, 4, 1, 8, "f16", list(range(40)))
    seqs = []
    for p in (p1, p2):
        s = p.create()
        p.append(s, 6)
        c1, c2 = p.fork(s), p.fork(s)      # three sharers of a partial block
        seqs = [s, c1, c2]
    got = p1.append_batch(seqs, 3)
    want = np.concatenate([np.asarray(p2.append(s, 3)) for s in seqs])
    assert got.tolist() == want.tolist()
    # s copies block 1 into 2 and grows into 3; c1 copies into 4; c2 writes in place
    assert p1.pending_copies() == p2.pending_copies() == [(1, 2), (1, 4)]
    assert p1.refcounts() == p2.refcounts() and p1.free_list() == p2.free_list()
    # a batch that cannot be satisfied in full changes nothing
    before = (p1.free_list(), p1.refcounts(), [p1.block_table(s) for s in seqs])
    with pytest.raises(kvp.KvpError) as e:
        p1.append_batch(seqs, 4 * 40)
    assert e.value.kind == "oom"
    assert (p1.free_list(), p1.refcounts(), [p1.block_table(s) for s in seqs]) == before
    with pytest.raises(kvp.KvpError) as e:
        p1.append_batch([seqs[0], seqs[0]], 1)
    assert e.value.kind == "invalid"


def test_rejected_duplicate_batch_leaves_no_trace():
    # The batch check lowers a shared last block's count for each earlier sharer
    # it has seen; a batch rejected part-way (a duplicate) must leave later
    # batches computing the same need as sequential appends.
    import paged_kv_cache_319_b200 as kvp

    pools = [kvp.BlockPool(16, 4, 1, 8, "f16", list(range(16))) for _ in range(2)]
    seqs = []
    for p in pools:
        s = p.create()
        p.append(s, 5)                     # block 1 partial
        seqs = [s, p.fork(s), p.fork(s)]   # three sharers of it
    p1, p2 = pools
    with pytest.raises(kvp.KvpError) as e:
        p1.append_batch([seqs[1], seqs[2], seqs[1]], 1)
    assert e.value.kind == "invalid"
    assert p1.refcounts() == p2.refcounts() and p1.free_list() == p2.free_list()
    got = p1.append_batch([seqs[1], seqs[2], seqs[0]], 1)
    want = [p2.append(s, 1)[0] for s in (seqs[1], seqs[2], seqs[0])]
    assert got.tolist() == want
    assert p1.pending_copies() == p2.pending_copies() == [(1, 2), (1, 3)]
    # exactly enough blocks for a batch whose sharers copy in turn
    q1, q2 = (kvp.BlockPool(6, 4, 1, 8, "f16", list(range(6))) for _ in range(2))
    for q in (q1, q2):
        a = q.create()
        q.append(a, 2)
        b, c = q.fork(a), q.fork(a)
    assert q1.num_free() == 5
    q1.append_batch([a, b, c], 3)          # two copies (a, b) + c in place, 3 more for growth
    for s in (a, b, c):
        q2.append(s, 3)
    assert q1.refcounts() == q2.refcounts() and q1.free_list() == q2.free_list()


def test_errors_and_capacity():
    import paged_kv_cache_319_b200 as kvp

    with pytest.raises(kvp.KvpError) as e:
        kvp.BlockPool(4, 4, 1, 8, "f16", [0, 1, 1, 3])
    assert e.value.kind == "invalid"
    p = kvp.BlockPool(8, 4, 1, 8, "f16")
    s = p.create()
    p.append(s, 9)
    with pytest.raises(kvp.KvpError) as e:
        p.build_batch([s], 2)
    assert e.value.kind == "capacity"
    t, l = p.build_batch([s], 5)
    assert t.tolist() == [[0, 1, 2, -1, -1]] and l.tolist() == [9]
    with pytest.raises(kvp.KvpError) as e:
        p.refcount(8)
    assert e.value.kind == "invalid"
    p.release(s)
    with pytest.raises(kvp.KvpError) as e:
        p.seq_len(s)
    assert e.value.kind == "no_seq"
    assert p.num_free() == 8


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("opt13b", {}), ("sharing_A", {}),
                                     ("sharing_B", {}), ("beam", {"steps": 12}),
                                     ("llama13b_churn", {"steps": 6})])
def test_workload_schedules_bit_exact(name, kw):
    """Every op of the workload schedules: same slots, tables, copies, counts."""
    wl = workloads.by_name(name, **kw)
    a = OracleBM(wl.num_blocks, wl.geometry.block_size, wl.free_order)
    b = LibBM(wl.num_blocks, wl.geometry.block_size, wl.free_order)
    ida, idb = {}, {}
    for op in wl.ops:
        k = op[0]
        if k == "create":
            ida[op[1]] = a.call("create")[1]
            idb[op[1]] = b.call("create")[1]
        elif k == "append":
            ra, rb = a.call("append", ida[op[1]], op[2]), b.call("append", idb[op[1]], op[2])
            assert ra == rb
        elif k == "fork":
            ida[op[2]] = a.call("fork", ida[op[1]])[1]
            idb[op[2]] = b.call("fork", idb[op[1]])[1]
        elif k == "release":
            assert a.call("release", ida[op[1]]) == b.call("release", idb[op[1]])
        elif k == "sync":
            ca, cb = a.call("take_copies")[1], b.call("take_copies")[1]
            assert [tuple(x) for x in ca] == [tuple(x) for x in cb]
        elif k == "attend":
            assert a.refcounts() == b.refcounts()
            assert a.free_list() == b.free_list()
            for h in op[1]:
                assert a.table(ida[h]) == b.table(idb[h])
    assert a.stats() == b.stats()
