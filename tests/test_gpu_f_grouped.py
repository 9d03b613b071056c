"""paged_attention_decode_grouped against the oracle and against paged_attention_decode.

The grouped entry point reads blocks held by several sequences once per
subgroup of them; the oracle decodes every sequence on its own, so agreement
shows the sharing changes nothing but the traffic. Batches are built with
explicit sharing: the members of a group hold the same physical blocks for a
leading run, then blocks of their own, in a shuffled batch order. The cases
cover groups larger than one subgroup (with a leftover member of one), a
member whose partial last block another member holds in full (the shared
prefix stops at full blocks), whole-sequence duplicates, sequences that share
only their first block, sequences shorter than a block, empty sequences,
shared prefixes that end inside a partition, own ranges of a block or two
(per-head warps), grouped-query heads, and
batches the entry point hands to paged_attention_decode (unsplit, a query
group too wide for two members, a head size the tensor cores do not take,
more sequences than the plan takes).
"""

import math

import numpy as np
import pytest

from oracle import attention
from oracle.numerics import to_f64
from parity import ATOL, check_close, from_bits, to_bits
import workloads

pytestmark = pytest.mark.gpu


def shared_batch(seed, groups, Hq, Hkv, D, bs, dtype, extra_blocks=5):
    """groups: list of (shared_blocks, member lengths). Each member's first
    min(shared_blocks, its own blocks) blocks are the group's; the rest are its own.
    Returns (q, k, v bits, tables int32 [S, MB], lens int32 [S])."""
    rng = np.random.default_rng(seed)
    members = [(gi, L) for gi, (_, lens) in enumerate(groups) for L in lens]
    need = [-(-L // bs) for _, L in members]
    n_shared = [sb for sb, _ in groups]
    nb = sum(n_shared) + sum(max(0, n - n_shared[gi]) for (gi, _), n in zip(members, need))
    nb += extra_blocks
    perm = rng.permutation(nb).astype(np.int32)
    pos = 0
    shared_ids = []
    for sb in n_shared:
        shared_ids.append(perm[pos:pos + sb])
        pos += sb
    order = rng.permutation(len(members))
    S = len(members)
    mb = max(1, max(need))
    tables = np.full((S, mb), -1, np.int32)
    lens = np.zeros(S, np.int32)
    for row, mi in enumerate(order):
        gi, L = members[mi]
        n = need[mi]
        k = min(n, n_shared[gi])
        tables[row, :k] = shared_ids[gi][:k]
        tables[row, k:n] = perm[pos:pos + n - k]
        pos += n - k
        lens[row] = L
    q = workloads.normal_bits([seed, 11], (S, Hq, D), dtype)
    k = workloads.normal_bits([seed, 12], (nb, Hkv, bs, D), dtype)
    v = workloads.normal_bits([seed, 13], (nb, Hkv, bs, D), dtype)
    return q, k, v, tables, lens


def host_plan(tables, lens, Hq, Hkv, bs, partition, num_blocks):
    import paged_kv_cache_319_b200 as kvp

    return kvp.group_plan(tables, lens, block_size=bs, partition_size=partition, num_q_heads=Hq,
                          num_kv_heads=Hkv, num_blocks=num_blocks,
                          max_context_len=int(max(lens.max(), 1)))


def run(q, k, v, tables, lens, dtype, scale, partition, grouped, workspace=None, plan=None,
        upload=False):
    """upload: also pass a device copy of the host plan (the call then copies nothing)."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    dplan = torch.from_numpy(plan).cuda() if upload and plan is not None else None
    out = kvp.paged_attention_decode(
        from_bits(q, dtype), from_bits(k, dtype), from_bits(v, dtype),
        torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(), scale,
        max_context_len=int(max(lens.max(), 1)), partition_size=partition, grouped=grouped,
        workspace=workspace, host_plan=plan, device_plan=dplan)
    kvp.check_device_error()
    return to_bits(out)


def oracle(q, k, v, tables, lens, dtype, scale, bs):
    return attention.paged_decode(to_f64(q, dtype), k, v, tables, lens, scale, bs, dtype=dtype)


# One query head per KV head: subgroups of up to 8.
GROUPS_MHA = [
    (31, [600, 700, 511, 767, 520, 530, 540, 550]),  # one subgroup of 8, prefix 31 blocks
    (40, [700] * 9),          # identical lengths: a subgroup of 8 and a leftover decoded alone
    (4, [50, 100, 64]),       # the 50-token member holds block 3 partly: prefix 3 blocks
    (2, [16, 16]),            # one full block each, nothing of their own
    (3, [40, 40]),            # duplicates whose last block is partial: prefix 2 blocks
    (1, [300, 900]),          # only the first block in common
    (0, [0]), (0, [5]), (0, [1500]),
    (20, [272] * 17),         # 17 members: 8 + 8 + a leftover
]

CASES = [
    # (name, Hq, Hkv, bs, dtype, partition, groups)
    ("mha_f16_bs16_p512", 8, 8, 16, "f16", 512, GROUPS_MHA),
    ("mha_bf16_bs32_p128", 4, 4, 32, "bf16", 128, GROUPS_MHA),
    ("mha_f16_bs16_p256", 2, 2, 16, "f16", 256, GROUPS_MHA),
    # own ranges of a block or two (beams): per-head warps on the CUDA cores
    ("mha_short_own_f16_bs16", 8, 8, 16, "f16", 512,
     [(30, [480, 481, 482, 490, 500, 495]), (20, [320, 321, 322]), (2, [33, 40]), (0, [9])]),
    ("mha_short_own_bf16_bs32", 6, 6, 32, "bf16", 256,
     [(15, [480, 481, 482, 500]), (9, [288, 300]), (0, [40])]),
    ("gqa4_bf16_bs16_p512", 16, 4, 16, "bf16", 512,
     [(31, [600, 700, 511, 767, 520]), (8, [128, 300, 129]), (0, [0]), (0, [7]), (0, [2000])]),
    ("gqa2_f16_bs32_p256", 8, 4, 32, "f16", 256,
     [(12, [400, 390, 500, 385, 1000, 386, 387, 388, 389]), (1, [33, 64]), (0, [1])]),
    ("gqa5_f16_bs16_p128", 10, 2, 16, "f16", 128,
     [(9, [150, 160, 170, 180]), (2, [20, 40]), (0, [300])]),
    ("gqa8_bf16_bs16_p512", 16, 2, 16, "bf16", 512,
     [(20, [400, 500, 600]), (30, [480, 480]), (0, [64])]),
    # handed to paged_attention_decode: a 16-wide query group, unsplit, 64-dim heads
    ("gqa16_fallback", 16, 1, 16, "bf16", 512, [(10, [200, 300]), (0, [50])]),
    ("unsplit_fallback", 4, 4, 16, "f16", 0, [(5, [100, 120]), (0, [30])]),
]


@pytest.mark.parametrize("plan_on", ["device", "host", "host+upload"])
@pytest.mark.parametrize("name,Hq,Hkv,bs,dtype,partition,groups", CASES, ids=[c[0] for c in CASES])
def test_grouped_matches_oracle(name, Hq, Hkv, bs, dtype, partition, groups, plan_on):
    seed = sum(map(ord, name))
    q, k, v, t, l = shared_batch(seed, groups, Hq, Hkv, 128, bs, dtype)
    scale = 1 / math.sqrt(128)
    plan = None
    if plan_on.startswith("host") and partition:
        plan = host_plan(t, l, Hq, Hkv, bs, partition, k.shape[0])
    got = run(q, k, v, t, l, dtype, scale, partition, grouped=True, plan=plan,
              upload=plan_on.endswith("upload"))
    ref = oracle(q, k, v, t, l, dtype, scale, bs)
    check_close(got, ref, dtype, allow_ulp=(dtype == "bf16"))


@pytest.mark.parametrize("name,Hq,Hkv,bs,dtype,partition,groups",
                         [c for c in CASES if c[5] and c[1] // c[2] < 16],
                         ids=[c[0] for c in CASES if c[5] and c[1] // c[2] < 16])
def test_device_plan_equals_host_plan(name, Hq, Hkv, bs, dtype, partition, groups):
    """The GPU plan kernel and the host planner build the same plan, word for word."""
    import torch

    q, k, v, t, l = shared_batch(sum(map(ord, name)), groups, Hq, Hkv, 128, bs, dtype)
    S, mcl = len(l), int(l.max())
    import paged_kv_cache_319_b200 as kvp

    need = kvp.decode_grouped_workspace_bytes(S, Hq, 128, mcl, partition)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device="cuda")
    run(q, k, v, t, l, dtype, 0.09, partition, grouped=True, workspace=ws)
    pmax = -(-mcl // partition)
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    off = up(S * Hq * (pmax + 1) * 8) + up(S * Hq * (pmax + 1) * 128 * 4)
    ref = host_plan(t, l, Hq, Hkv, bs, partition, k.shape[0])
    dev = ws[off:off + 4 * len(ref)].cpu().numpy().view(np.int32)
    # member slots past a subgroup's size are not written by the GPU kernel
    n_sub = int(ref[0])
    mask = np.ones(len(ref), bool)
    for i in range(n_sub):
        e = 8 + S + i * 20
        mask[e + 4 + ref[e + 1]:e + 20] = False
    mask[8 + S + n_sub * 20:] = False
    assert np.array_equal(dev[mask], ref[mask])


def run_packed(q, k, v, tables, lens, dtype, scale, Hq, Hkv, bs, upload=False):
    import torch
    import paged_kv_cache_319_b200 as kvp

    plan = kvp.pack_plan(tables, lens, block_size=bs, num_q_heads=Hq, num_kv_heads=Hkv,
                         num_blocks=k.shape[0], max_context_len=int(max(lens.max(), 1)))
    dplan = torch.from_numpy(plan).cuda() if upload else None
    out = kvp.paged_attention_decode_packed(
        from_bits(q, dtype), from_bits(k, dtype), from_bits(v, dtype),
        torch.from_numpy(lens).cuda(), scale, plan, max_context_len=int(max(lens.max(), 1)),
        device_plan=dplan)
    kvp.check_device_error()
    return to_bits(out)


# the packed decode takes 128-dim heads, blocks of 16 or 32, up to 16 query heads per KV head
PACKED_CASES = [c for c in CASES if c[0] not in ("unsplit_fallback",)]


@pytest.mark.parametrize("upload", [False, True])
@pytest.mark.parametrize("name,Hq,Hkv,bs,dtype,partition,groups", PACKED_CASES,
                         ids=[c[0] for c in PACKED_CASES])
def test_packed_matches_oracle(name, Hq, Hkv, bs, dtype, partition, groups, upload):
    seed = sum(map(ord, name)) + 7
    q, k, v, t, l = shared_batch(seed, groups, Hq, Hkv, 128, bs, dtype)
    scale = 1 / math.sqrt(128)
    got = run_packed(q, k, v, t, l, dtype, scale, Hq, Hkv, bs, upload=upload)
    ref = oracle(q, k, v, t, l, dtype, scale, bs)
    check_close(got, ref, dtype, allow_ulp=(dtype == "bf16"))


def test_packed_rejects_a_plan_of_another_shape():
    import torch
    import paged_kv_cache_319_b200 as kvp

    q, k, v, t, l = shared_batch(3, [(31, [600, 700, 520]), (0, [40])], 8, 8, 128, 16, "f16")
    plan = kvp.pack_plan(t, l, block_size=16, num_q_heads=8, num_kv_heads=8, num_blocks=k.shape[0])
    args = (from_bits(q, "f16"), from_bits(k, "f16"), from_bits(v, "f16"),
            torch.from_numpy(l).cuda(), 0.09)
    bad = plan.copy()
    bad[int(plan[6]) + 2] += 1                         # a unit with one entry too many
    with pytest.raises(kvp.KvpError):
        kvp.paged_attention_decode_packed(*args, bad)
    bad = plan.copy()
    bad[8] = (bad[8] + 1) % int(plan[0])               # a sequence's group word
    with pytest.raises(kvp.KvpError):
        kvp.paged_attention_decode_packed(*args, bad)
    bad = plan.copy()
    bad[int(plan[7]) + 1] |= 1 << 30                   # an entry's columns past its group
    with pytest.raises(kvp.KvpError):
        kvp.paged_attention_decode_packed(*args, bad)


def test_head_dim_64_is_handed_on():
    q, k, v, t, l = shared_batch(5, [(6, [100, 130, 140]), (0, [20])], 4, 4, 64, 16, "f16")
    got = run(q, k, v, t, l, "f16", 0.125, 512, grouped=True)
    check_close(got, oracle(q, k, v, t, l, "f16", 0.125, 16), "f16")


def test_grouped_agrees_with_the_ungrouped_entry():
    q, k, v, t, l = shared_batch(21, GROUPS_MHA, 8, 8, 128, 16, "f16")
    a = to_f64(run(q, k, v, t, l, "f16", 0.088, 512, grouped=True), "f16")
    b = to_f64(run(q, k, v, t, l, "f16", 0.088, 512, grouped=False), "f16")
    assert np.abs(a - b).max() <= ATOL


def test_reused_workspace_two_batches_in_a_row():
    """The plan and partial slots left in the workspace by one call must not leak into the next."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    ws = torch.empty(kvp.decode_grouped_workspace_bytes(64, 8, 128, 2048, 512), dtype=torch.uint8,
                     device="cuda")
    ws.fill_(0xFF)  # NaN bit patterns everywhere
    for seed, groups in ((1, GROUPS_MHA), (2, [(2, [40, 2000, 700]), (0, [900]), (9, [150] * 5)])):
        q, k, v, t, l = shared_batch(seed, groups, 8, 8, 128, 16, "f16")
        assert l.max() <= 2048 and len(l) <= 64
        for plan in (None, host_plan(t, l, 8, 8, 16, 512, k.shape[0])):
            got = run(q, k, v, t, l, "f16", 0.09, 512, grouped=True, workspace=ws, plan=plan)
            check_close(got, oracle(q, k, v, t, l, "f16", 0.09, 16), "f16")


def test_malformed_host_plans_are_rejected():
    """Every index and count of a caller's plan is checked on the host before a kernel reads it."""
    import torch
    import paged_kv_cache_319_b200 as kvp
    from paged_kv_cache_319_b200._lib import KvpError

    q, k, v, t, l = shared_batch(3, [(4, [100, 120]), (0, [30])], 8, 8, 128, 16, "f16")
    plan = host_plan(t, l, 8, 8, 16, 512, k.shape[0])
    S = len(l)
    sub0 = 8 + S  # first subgroup entry
    assert plan[0] == 1 and plan[sub0 + 1] == 2
    members = plan[sub0 + 4:sub0 + 6].tolist()
    other = next(x for x in range(S) if x not in members)

    def corrupt(fn):
        bad = plan.copy()
        fn(bad)
        return bad

    malformed = [
        corrupt(lambda b: b.__setitem__(0, 99)),                 # more subgroups than the batch holds
        corrupt(lambda b: b.__setitem__(sub0 + 4, S)),           # member index outside the batch
        corrupt(lambda b: b.__setitem__(sub0 + 5, members[0])),  # a member twice
        corrupt(lambda b: b.__setitem__(sub0, 500)),             # prefix past every table
        corrupt(lambda b: b.__setitem__(8 + other, 3)),          # a prefix for a sequence in no subgroup
        corrupt(lambda b: b.__setitem__(sub0 + 1, 17)),          # more members than columns
        corrupt(lambda b: b.__setitem__(1, 2)),                  # shared partition count off
    ]
    for bad in malformed:
        with pytest.raises(KvpError) as e:
            run(q, k, v, t, l, "f16", 0.09, 512, grouped=True, plan=bad)
        assert e.value.kind == "invalid"
    # a device copy without the host plan it copies is rejected too
    with pytest.raises(KvpError) as e:
        kvp.paged_attention_decode(
            from_bits(q, "f16"), from_bits(k, "f16"), from_bits(v, "f16"),
            torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(), 0.09,
            max_context_len=int(l.max()), partition_size=512, grouped=True,
            device_plan=torch.from_numpy(plan).cuda())
    assert e.value.kind == "invalid"
    torch.cuda.synchronize()


@pytest.mark.parametrize("plan_on", ["device", "host"])
@pytest.mark.parametrize("S", [4096, 4100])
def test_batch_size_limit_of_the_plan(S, plan_on):
    """4096 sequences are grouped (the plan's limit); 4100 go through paged_attention_decode."""
    rng = np.random.default_rng(S)
    groups, n = [], 0
    while n < S:
        m = int(min(S - n, rng.integers(1, 12)))
        groups.append((int(rng.integers(1, 4)), rng.integers(1, 60, size=m).tolist()))
        n += m
    q, k, v, t, l = shared_batch(S, groups, 1, 1, 128, 16, "f16")
    plan = host_plan(t, l, 1, 1, 16, 128, k.shape[0]) if plan_on == "host" and S <= 4096 else None
    got = run(q, k, v, t, l, "f16", 0.09, 128, grouped=True, plan=plan)
    check_close(got, oracle(q, k, v, t, l, "f16", 0.09, 16), "f16")


@pytest.mark.parametrize("plan_on", ["device", "host"])
@pytest.mark.parametrize("name,kw", [("sharing_A", {}), ("sharing_B", {}), ("beam", {"steps": 16})])
def test_fork_workloads_grouped_every_output(name, kw, plan_on):
    """The sampling and beam workloads (blocks shared through fork and copy-on-write),
    decoded through the grouped entry point at every attend op."""
    from oracle.replay import OracleReplay
    from paged_kv_cache_319_b200.replay import DeviceReplay
    import paged_kv_cache_319_b200 as kvp

    wl = workloads.by_name(name, **kw)
    dev = DeviceReplay(wl, "cuda", grouped=True, plan_on=plan_on)
    dev.run()
    kvp.check_device_error()
    ora = OracleReplay(wl)
    refs = {}
    ora.run(attend=lambda i, seqs, tables, lens: refs.__setitem__(i, ora.decode(i, tables, lens.tolist())))
    assert refs
    for i, ref in refs.items():
        check_close(to_bits(dev.outputs[i]), ref, wl.geometry.dtype)
