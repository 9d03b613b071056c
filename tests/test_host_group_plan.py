"""kv_decode_group_plan: the host planner of the grouped decode.

The plan decides only which sequences read a shared prefix together; the
decode's result does not depend on it (the GPU tests check that). Here the
plan is checked against the rule it states (sorted keys, subgroups cut in
order, the longest common prefix of full blocks), against a plain Python
restatement of that rule, and on the fork workloads, whose sharing is known
from their construction.
"""

import numpy as np
import pytest

import paged_kv_cache_319_b200 as kvp
from paged_kv_cache_319_b200._lib import KvpError
import workloads

HDR, SUBW = 8, 20


def batch(seed, groups, bs, extra=3):
    """groups: (shared_blocks, member lengths); members hold the group's blocks first."""
    rng = np.random.default_rng(seed)
    members = [(gi, L) for gi, (_, lens) in enumerate(groups) for L in lens]
    need = [-(-L // bs) for _, L in members]
    ids = iter(rng.permutation(10_000).tolist())
    shared = [[next(ids) for _ in range(sb)] for sb, _ in groups]
    order = rng.permutation(len(members))
    mb = max(1, max(need))
    t = np.full((len(members), mb), -1, np.int32)
    lens = np.zeros(len(members), np.int32)
    for row, mi in enumerate(order):
        gi, L = members[mi]
        n = need[mi]
        k = min(n, len(shared[gi]))
        t[row, :k] = shared[gi][:k]
        t[row, k:n] = [next(ids) for _ in range(n - k)]
        lens[row] = L
    return t, lens


def reference_plan(t, lens, bs, part, G, nb, mcl):
    """The rule, restated plainly."""
    mmax = max(1, (8 if G == 1 else 16) // G)
    S = len(lens)
    ctx = np.clip(lens, 0, mcl)
    keyed = sorted((int(t[s, 0]), s) for s in range(S) if ctx[s] >= bs and 0 <= t[s, 0] < nb)
    runs = {}
    for k, s in keyed:
        runs.setdefault(k, []).append(s)
    subs = []
    for k in sorted(runs):
        r = runs[k]
        for i in range(0, len(r), mmax):
            m = r[i:i + mmax]
            if len(m) < 2:
                continue
            cap = min(ctx[x] // bs for x in m)
            c = 0
            while c < cap and all(t[x, c] == t[m[0], c] for x in m):
                c += 1
            subs.append((c, m))
    cb = np.zeros(S, np.int64)
    for c, m in subs:
        cb[m] = c
    own = ctx - cb * bs
    plan = np.zeros(HDR + S + (S // 2 + 1) * SUBW, np.int64)
    plan[0] = len(subs)
    plan[1] = max([-(-c * bs // part) for c, _ in subs], default=0)
    plan[2] = max([-(-int(o) // part) for o in own if o > 0], default=0)
    plan[3] = sum(c for c, _ in subs)
    plan[4] = sum(-(-int(o) // bs) for o in own if o > 0)
    plan[HDR:HDR + S] = cb
    for i, (c, m) in enumerate(subs):
        e = HDR + S + i * SUBW
        plan[e], plan[e + 1] = c, len(m)
        plan[e + 4:e + 4 + len(m)] = m
    return plan


GROUPS = [
    (31, [600, 700, 511, 767, 520, 530, 540, 550]),
    (40, [700] * 9),
    (4, [50, 100, 64]),
    (2, [16, 16]),
    (3, [40, 40]),
    (1, [300, 900]),
    (0, [0]), (0, [5]), (0, [1500]),
    (20, [272] * 17),
]


@pytest.mark.parametrize("G,bs,part", [(1, 16, 512), (1, 32, 128), (4, 16, 256), (2, 16, 512),
                                       (5, 32, 256), (8, 16, 128), (16, 16, 512)])
def test_plan_matches_the_rule(G, bs, part):
    t, lens = batch(G * 100 + bs, GROUPS, bs)
    mcl = int(lens.max())
    got = kvp.group_plan(t, lens, block_size=bs, partition_size=part, num_q_heads=8 * G,
                         num_kv_heads=8, num_blocks=10_000, max_context_len=mcl)
    ref = reference_plan(t, lens, bs, part, G, 10_000, mcl)
    assert np.array_equal(got, ref.astype(np.int32))


def test_plan_invariants_on_random_batches():
    rng = np.random.default_rng(7)
    for trial in range(40):
        bs = int(rng.choice([16, 32]))
        part = bs * int(rng.choice([4, 8, 32]))
        G = int(rng.choice([1, 2, 4]))
        mmax = (8 if G == 1 else 16) // G
        groups = [(int(rng.integers(0, 12)), rng.integers(0, 400, size=int(rng.integers(1, 20))).tolist())
                  for _ in range(int(rng.integers(1, 8)))]
        t, lens = batch(trial, groups, bs)
        S = len(lens)
        mcl = int(max(lens.max(), 1))
        p = kvp.group_plan(t, lens, block_size=bs, partition_size=part, num_q_heads=4 * G,
                           num_kv_heads=4, num_blocks=10_000, max_context_len=mcl)
        n_sub = p[0]
        seen = set()
        for i in range(n_sub):
            e = HDR + S + i * SUBW
            c, nm = p[e], p[e + 1]
            m = p[e + 4:e + 4 + nm].tolist()
            assert 2 <= nm <= mmax and m == sorted(m) and not (set(m) & seen)
            seen |= set(m)
            cap = min(lens[x] // bs for x in m)
            assert 1 <= c <= cap
            assert all(np.array_equal(t[x, :c], t[m[0], :c]) for x in m)
            assert c == cap or len({int(t[x, c]) for x in m}) > 1  # longest common prefix
            assert all(p[HDR + x] == c for x in m)
        assert all(p[HDR + s] == 0 for s in range(S) if s not in seen)
        # a run of >= 2 groupable sequences with one first block leaves at most one out
        keys = {}
        for s in range(S):
            if lens[s] >= bs:
                keys.setdefault(int(t[s, 0]), []).append(s)
        for k, r in keys.items():
            left = [s for s in r if s not in seen]
            assert len(left) <= 1 and (not left or len(r) % mmax == 1)


def test_fork_workloads_group_as_built():
    """Sampling B: 8 prompts of 511..504 tokens x 8 samples; every sample copies the
    prompt's partial last block on its first write, so each prompt's 8 samples
    share exactly its 31 full blocks. Sampling A: 512-token prompts, 32 shared blocks."""
    from oracle.replay import OracleReplay

    for name, c_expect in (("sharing_B", 31), ("sharing_A", 32)):
        wl = workloads.by_name(name)
        got = []
        OracleReplay(wl).run(attend=lambda i, seqs, tables, lens: got.append((tables, lens)))
        (t, lens), = got
        p = kvp.group_plan(t, lens, block_size=16, partition_size=512, num_q_heads=40,
                           num_kv_heads=40, num_blocks=wl.num_blocks, max_context_len=int(lens.max()))
        S = len(lens)
        assert p[0] == 8 and p[3] == 8 * c_expect
        for i in range(8):
            e = HDR + S + i * SUBW
            assert p[e] == c_expect and p[e + 1] == 8
        assert (p[HDR:HDR + S] == c_expect).all()
        assert p[4] == sum(-(-(int(L) - c_expect * 16) // 16) for L in lens)


def test_plan_rejects_bad_arguments():
    t, lens = batch(1, [(2, [40, 40])], 16)
    with pytest.raises(KvpError) as e:
        kvp.group_plan(t, lens, block_size=16, partition_size=100, num_q_heads=8, num_kv_heads=8,
                       num_blocks=100)
    assert e.value.kind == "invalid"
    with pytest.raises(KvpError):
        kvp.group_plan(t, lens, block_size=16, partition_size=0, num_q_heads=8, num_kv_heads=8,
                       num_blocks=100)
    with pytest.raises(KvpError):
        kvp.group_plan(t, lens, block_size=16, partition_size=512, num_q_heads=6, num_kv_heads=4,
                       num_blocks=100)
