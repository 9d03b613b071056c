"""The packed plan of the packed grouped decode (host planner, CPU only).

The plan's promise, checked on random batches with shared prefixes: for every
sequence, the entries of its group's block stream that carry its member's
columns are exactly its block table, in order, with each block's valid
tokens; the shared prefix comes first and carries every member's columns;
every chunk of every group is one unit record, with its entries, and units run
longest first. The groups are the subgroups of kv_decode_group_plan's rule
(and a group of one for every other sequence).
"""

import numpy as np
import pytest


def shared_batch(rng, groups, bs, extra=5):
    """groups: list of (shared blocks, member lengths) -> (tables [S, MB], lens [S], NB)."""
    members = [(gi, L) for gi, (_, ls) in enumerate(groups) for L in ls]
    need = [-(-L // bs) for _, L in members]
    nb = sum(sb for sb, _ in groups) + sum(need) + extra
    perm = rng.permutation(nb).astype(np.int32)
    pos = 0
    shared = []
    for sb, _ in groups:
        shared.append(perm[pos:pos + sb])
        pos += sb
    order = rng.permutation(len(members))
    tables = np.full((len(members), max(1, max(need))), -1, np.int32)
    lens = np.zeros(len(members), np.int32)
    for row, mi in enumerate(order):
        gi, L = members[mi]
        n = need[mi]
        k = min(n, len(shared[gi]))
        tables[row, :k] = shared[gi][:k]
        tables[row, k:n] = perm[pos:pos + n - k]
        pos += n - k
        lens[row] = L
    return tables, lens, nb


def decode_plan(plan, S):
    ngr, nu, ne, mc, bs, bpc, uoff, eoff = (int(x) for x in plan[:8])
    seq_group = plan[8:8 + S]
    groups = []
    for g in range(ngr):
        e = plan[8 + S + 20 * g: 8 + S + 20 * (g + 1)]
        groups.append(dict(first=int(e[0]), nm=int(e[1]), n=int(e[2]), chunks=int(e[3]),
                           seqs=[int(x) for x in e[4:4 + e[1]]]))
    units = [tuple(int(x) for x in plan[uoff + 4 * i: uoff + 4 * i + 4]) for i in range(nu)]
    ents = plan[eoff:eoff + 2 * ne].reshape(ne, 2)
    return dict(ngr=ngr, mc=mc, bs=bs, bpc=bpc, seq_group=seq_group, groups=groups, units=units,
                ents=ents)


CASES = [
    # (Hq, Hkv, bs, groups)
    (8, 8, 16, [(31, [600, 700, 511, 767, 520, 530, 540, 550]), (40, [700] * 9), (4, [50, 100, 64]),
                (2, [16, 16]), (0, [0]), (0, [5]), (0, [1500]), (20, [272] * 17)]),
    (4, 4, 32, [(15, [480, 481, 482, 500]), (9, [288, 300]), (0, [40])]),
    (16, 4, 16, [(31, [600, 700, 511, 767, 520]), (8, [128, 300, 129]), (0, [0]), (0, [2000])]),
    (16, 2, 16, [(20, [400, 500, 600]), (30, [480, 480]), (0, [64])]),
    (16, 1, 32, [(10, [200, 300]), (0, [50])]),
]


@pytest.mark.parametrize("Hq,Hkv,bs,groups", CASES)
@pytest.mark.parametrize("seed", [0, 1])
def test_pack_plan_streams_cover_every_table(Hq, Hkv, bs, groups, seed):
    import paged_kv_cache_319_b200 as kvp

    rng = np.random.default_rng(seed)
    tables, lens, nb = shared_batch(rng, groups, bs)
    S = len(lens)
    G = Hq // Hkv
    plan = kvp.pack_plan(tables, lens, block_size=bs, num_q_heads=Hq, num_kv_heads=Hkv,
                         num_blocks=nb, max_context_len=int(lens.max()))
    p = decode_plan(plan, S)
    assert p["bs"] == bs and p["bpc"] == 512 // bs
    seen = np.zeros(S, int)
    for gi, gr in enumerate(p["groups"]):
        assert 1 <= gr["nm"] <= max(1, 16 // G if G > 1 else 8)
        assert gr["chunks"] == -(-gr["n"] // p["bpc"])
        stream = p["ents"][gr["first"]:gr["first"] + gr["n"]]
        cols_all = (1 << (gr["nm"] * G)) - 1
        for m, s in enumerate(gr["seqs"]):
            seen[s] += 1
            assert p["seq_group"][s] == gi
            mine = (1 << G) - 1 << (m * G)
            ids, valid = [], []
            for bid, w in stream:
                mask = int(w) >> 8
                assert mask & ~cols_all == 0
                assert mask & mine in (0, mine)  # a member takes all or none of a block
                if mask & mine:
                    ids.append(int(bid))
                    valid.append(int(w) & 0xFF)
            nblk = -(-int(lens[s]) // bs)
            assert ids == tables[s, :nblk].tolist()
            assert valid == [min(bs, int(lens[s]) - b * bs) for b in range(nblk)]
        # the shared prefix leads the stream and every member takes it
        k = 0
        while k < len(stream) and (int(stream[k][1]) >> 8) == cols_all and gr["nm"] > 1:
            k += 1
        if gr["nm"] > 1:
            assert all(int(w) >> 8 != cols_all for _, w in stream[k:])
    assert (seen == 1).all()
    assert p["mc"] == max(g["chunks"] for g in p["groups"])
    # units: every (group, chunk) once, with its entries, longest first
    got = sorted((u[0], u[3]) for u in p["units"])
    want = sorted((gi, c) for gi, g in enumerate(p["groups"]) for c in range(g["chunks"]))
    assert got == want
    for g, first, n, c in p["units"]:
        gr = p["groups"][g]
        assert first == gr["first"] + c * p["bpc"] and n == min(p["bpc"], gr["n"] - c * p["bpc"])
    ns = [u[2] for u in p["units"]]
    assert ns == sorted(ns, reverse=True)


@pytest.mark.parametrize("Hq,Hkv,bs,groups", CASES)
def test_pack_plan_groups_are_the_grouping_rule(Hq, Hkv, bs, groups):
    import paged_kv_cache_319_b200 as kvp

    tables, lens, nb = shared_batch(np.random.default_rng(7), groups, bs)
    S = len(lens)
    plan = kvp.pack_plan(tables, lens, block_size=bs, num_q_heads=Hq, num_kv_heads=Hkv,
                         num_blocks=nb, max_context_len=int(lens.max()))
    p = decode_plan(plan, S)
    gp = kvp.group_plan(tables, lens, block_size=bs, partition_size=512, num_q_heads=Hq,
                        num_kv_heads=Hkv, num_blocks=nb, max_context_len=int(lens.max()))
    subs = {tuple(int(x) for x in gp[8 + S + 20 * i + 4: 8 + S + 20 * i + 4 + gp[8 + S + 20 * i + 1]])
            for i in range(int(gp[0]))}
    multi = {tuple(g["seqs"]) for g in p["groups"] if g["nm"] > 1}
    assert multi == subs
    for g in p["groups"]:
        if g["nm"] > 1:
            c = int(gp[8 + g["seqs"][0]])  # the shared prefix of the grouped plan
            stream = p["ents"][g["first"]:g["first"] + c]
            cols_all = (1 << (g["nm"] * (Hq // Hkv))) - 1
            assert all(int(w) >> 8 == cols_all for _, w in stream)


def test_pack_plan_refuses_bad_arguments():
    import paged_kv_cache_319_b200 as kvp

    t = np.zeros((2, 4), np.int32)
    l = np.array([16, 16], np.int32)
    for kw in (dict(block_size=8), dict(num_q_heads=6, num_kv_heads=4), dict(max_context_len=65)):
        args = dict(block_size=16, num_q_heads=4, num_kv_heads=4, num_blocks=8, max_context_len=32)
        args.update(kw)
        with pytest.raises(kvp.KvpError):
            kvp.pack_plan(t, l, **args)
