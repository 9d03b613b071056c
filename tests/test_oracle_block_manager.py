"""Pins of the block-manager oracle: a hand-derived trace, invariants, sharing counts."""

import json
import math
import os
import random

import pytest

from bm_adapters import OracleBM
from oracle.replay import OracleReplay
import workloads

TRACE = os.path.join(os.path.dirname(__file__), "golden", "block_manager_trace.json")


def run_trace(make):
    with open(TRACE) as f:
        tr = json.load(f)
    bm = make(tr["num_blocks"], tr["block_size"], tr["free_order"])
    for step in tr["steps"]:
        op, exp = step["op"], step["expect"]
        name, args = op[0], op[1:]
        err, res = bm.call(name, *args)
        assert err == exp.get("error"), (op, err)
        if "seq" in exp:
            assert res == exp["seq"], op
        if "slots" in exp:
            assert list(res) == exp["slots"], op
        if "copies" in exp:
            assert [list(p) for p in res] == exp["copies"], op
        for s, t in exp.get("table", {}).items():
            assert bm.table(int(s)) == t, (op, s)
        for s, n in exp.get("len", {}).items():
            assert bm.seq_len(int(s)) == n, (op, s)
        if "free" in exp:
            assert bm.free_list() == exp["free"], op
        for b, c in exp.get("rc", {}).items():
            assert bm.refcounts()[int(b)] == c, (op, b)
        if "pending" in exp:
            assert [list(p) for p in bm.pending()] == exp["pending"], op
        for s, w in exp.get("waste", {}).items():
            assert len(bm.table(int(s))) * tr["block_size"] - bm.seq_len(int(s)) == w
    assert all(c == 0 for c in bm.refcounts())
    assert sorted(bm.free_list()) == list(range(tr["num_blocks"]))


def test_hand_trace_oracle():
    run_trace(OracleBM)


def random_ops(seed, n_ops=400, num_blocks=64, bs=4):
    rnd = random.Random(seed)
    bm = OracleBM(num_blocks, bs, rnd.sample(range(num_blocks), num_blocks))
    live = []
    for _ in range(n_ops):
        r = rnd.random()
        if r < 0.15 or not live:
            _, s = bm.call("create")
            live.append(s)
        elif r < 0.6:
            s = rnd.choice(live)
            err, _ = bm.call("append", s, rnd.randint(0, 9))
            assert err in (None, "oom")
        elif r < 0.75:
            _, c = bm.call("fork", rnd.choice(live))
            live.append(c)
        elif r < 0.9:
            s = live.pop(rnd.randrange(len(live)))
            assert bm.call("release", s)[0] is None
        else:
            bm.call("take_copies")
        yield bm, live, bs, num_blocks


@pytest.mark.parametrize("seed", range(6))
def test_invariants_on_random_schedules(seed):
    for bm, live, bs, nb in random_ops(seed):
        rc = bm.refcounts()
        refs = [0] * nb
        for s in live:
            t = bm.table(s)
            L = bm.seq_len(s)
            # allocation on growth only: exactly ceil(len / bs) blocks
            assert len(t) == math.ceil(L / bs)
            # waste only in the last, partly filled block
            assert 0 <= len(t) * bs - L <= bs - 1
            for b in t:
                refs[b] += 1
        # refcount == number of table references
        assert rc == refs
        free = bm.free_list()
        assert len(set(free)) == len(free)
        assert all(rc[b] == 0 for b in free)
        # conservation: free + referenced == pool
        assert len(free) + sum(1 for c in rc if c > 0) == nb


def test_oom_leaves_state_unchanged():
    bm = OracleBM(4, 4, [0, 1, 2, 3])
    _, s = bm.call("create")
    assert bm.call("append", s, 10)[0] is None     # 3 blocks
    _, c = bm.call("fork", s)
    before = (bm.free_list(), bm.refcounts(), bm.table(s), bm.table(c), bm.pending())
    # needs 1 CoW block + 2 growth blocks, only 1 free
    assert bm.call("append", c, 7)[0] == "oom"
    assert (bm.free_list(), bm.refcounts(), bm.table(s), bm.table(c), bm.pending()) == before
    # exactly one block is still enough for the copy-on-write of one token
    err, slots = bm.call("append", c, 1)
    assert err is None and bm.pending() == [(2, 3)] and slots == [3 * 4 + 2]


def test_release_everything_restores_pool():
    wl = workloads.beam_search(steps=5)
    rp = OracleReplay(wl, with_cache=False)
    rp.run()
    for s in rp.bm.live_seqs():
        rp.bm.release(s)
    assert rp.bm.num_free() == wl.num_blocks
    assert all(c == 0 for c in rp.bm.rc)


def test_sharing_variant_a_has_no_copies_and_full_sharing():
    wl = workloads.sharing_sampling("A")
    rp = OracleReplay(wl, with_cache=False)
    forks_done = None
    for i, op in enumerate(wl.ops):
        rp._apply(i, op, None)
        if op[0] == "fork":
            forks_done = i
        elif forks_done is not None:
            break
    # after the 7 forks of each 512-token prompt: 32 blocks per prompt with rc 8
    shared = [b for b, c in enumerate(rp.bm.rc) if c == 8]
    assert len(shared) == 8 * 32
    rp2 = OracleReplay(wl, with_cache=False)
    rp2.run()
    copies = [p for (_, kind, payload) in rp2.events if kind == "sync" for p in payload]
    assert copies == []


def test_sharing_variant_b_has_seven_copies_per_prompt():
    wl = workloads.sharing_sampling("B")
    rp = OracleReplay(wl, with_cache=False)
    rp.run()
    copies = [p for (_, kind, payload) in rp.events if kind == "sync" for p in payload]
    assert len(copies) == 8 * 7
    # every copy's source is one of the prompts' shared partial last blocks
    assert len({src for src, _ in copies}) == 8
    st = rp.bm.stats()
    assert st.cow_copies_total == 56
    # full prompt blocks stay shared by all 8 samples: 31 per prompt
    assert sum(1 for c in rp.bm.rc if c == 8) == 8 * 31


def test_beam_copies_match_parent_multiplicity():
    wl = workloads.beam_search(steps=3)
    rp = OracleReplay(wl, with_cache=False)
    rp.run()
    # with width 4, at most 3 copies per prompt per step, and only of partial blocks
    per_sync = [len(payload) for (_, kind, payload) in rp.events if kind == "sync"]
    assert all(n <= 8 * 3 for n in per_sync)
    assert sum(per_sync) > 0
