"""Pins of the attention oracle: closed forms, a library routine, brute force, paging invariance."""

import math

import numpy as np
import pytest
import torch

from oracle import attention, cache
from oracle.block_manager import BlockManager
from oracle.numerics import to_f64
from oracle.replay import OracleReplay
import workloads


def sdpa64(q, K, V, scale):
    """torch fp64 scaled_dot_product_attention for one sequence; q [H, D], K/V [H, ctx, D]."""
    qt = torch.from_numpy(q)[:, None, :]
    out = torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(K), torch.from_numpy(V), scale=scale)
    return out[:, 0, :].numpy()


def paged_random(rng, S, Hq, Hkv, D, bs, lens, extra_blocks=3):
    """Random fp64 paged cache with sequences placed on a shuffled set of blocks."""
    nblk = sum(-(-L // bs) for L in lens) + extra_blocks
    perm = rng.permutation(nblk)
    k = rng.standard_normal((nblk, Hkv, bs, D))
    v = rng.standard_normal((nblk, Hkv, bs, D))
    mb = max(1, max(-(-L // bs) for L in lens))
    tables = np.full((S, mb), -1, np.int64)
    i = 0
    for s, L in enumerate(lens):
        for j in range(-(-L // bs)):
            tables[s, j] = perm[i]
            i += 1
    q = rng.standard_normal((S, Hq, D))
    return q, k, v, tables


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (32, 8)])
def test_matches_torch_sdpa(Hq, Hkv):
    rng = np.random.default_rng(7)
    bs, D = 16, 32
    lens = [1, 15, 16, 37, 100]
    q, k, v, bt = paged_random(rng, len(lens), Hq, Hkv, D, bs, lens)
    scale = 1 / math.sqrt(D)
    out = attention.paged_decode(q, k, v, bt, lens, scale, bs)
    G = Hq // Hkv
    for s, L in enumerate(lens):
        K = np.stack([attention.gather(k, bt[s], L, g, bs) for g in range(Hkv)])
        V = np.stack([attention.gather(v, bt[s], L, g, bs) for g in range(Hkv)])
        # torch's grouped-query convention: query head h reads KV head h // G
        K = np.repeat(K, G, axis=0)
        V = np.repeat(V, G, axis=0)
        ref = sdpa64(q[s], K, V, scale)
        np.testing.assert_allclose(out[s], ref, rtol=1e-12, atol=1e-12)


def test_identity_block_table_equals_plain_attention():
    rng = np.random.default_rng(3)
    S, H, D, bs, L = 3, 2, 16, 8, 40
    mb = L // bs
    k = rng.standard_normal((S * mb, H, bs, D))
    v = rng.standard_normal((S * mb, H, bs, D))
    bt = np.arange(S * mb).reshape(S, mb)       # contiguous, in order
    q = rng.standard_normal((S, H, D))
    out = attention.paged_decode(q, k, v, bt, [L] * S, 0.3, bs)
    # the same buffers read as one contiguous [S, H, L, D] tensor
    Kc = k.reshape(S, mb, H, bs, D).transpose(0, 2, 1, 3, 4).reshape(S, H, L, D)
    Vc = v.reshape(S, mb, H, bs, D).transpose(0, 2, 1, 3, 4).reshape(S, H, L, D)
    for s in range(S):
        np.testing.assert_allclose(out[s], sdpa64(q[s], Kc[s], Vc[s], 0.3), rtol=1e-12, atol=1e-12)


def test_permutation_of_physical_blocks_gives_identical_output():
    rng = np.random.default_rng(11)
    S, H, D, bs = 4, 3, 8, 4
    lens = [5, 17, 1, 30]
    q, k, v, bt = paged_random(rng, S, H, H, D, bs, lens, extra_blocks=0)
    out1 = attention.paged_decode(q, k, v, bt, lens, 0.5, bs)
    # move every physical block to a new place and rewrite the tables
    perm = rng.permutation(k.shape[0])
    k2 = np.empty_like(k)
    v2 = np.empty_like(v)
    k2[perm] = k
    v2[perm] = v
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1)
    out2 = attention.paged_decode(q, k2, v2, bt2, lens, 0.5, bs)
    assert np.array_equal(out1, out2)


def brute_force(q, k, v, tables, lens, scale, bs):
    """Scalar loops, no NumPy arithmetic: the textbook softmax-weighted average."""
    S, H, D = len(q), len(q[0]), len(q[0][0])
    Hkv = len(k[0])
    G = H // Hkv
    out = [[[0.0] * D for _ in range(H)] for _ in range(S)]
    for s in range(S):
        for h in range(H):
            g = h // G
            scores = []
            for j in range(lens[s]):
                blk = tables[s][j // bs]
                dot = 0.0
                for d in range(D):
                    dot += q[s][h][d] * k[blk][g][j % bs][d]
                scores.append(dot * scale)
            if not scores:
                continue
            mx = max(scores)
            w = [math.exp(x - mx) for x in scores]
            tot = sum(w)
            for j in range(lens[s]):
                blk = tables[s][j // bs]
                for d in range(D):
                    out[s][h][d] += w[j] / tot * v[blk][g][j % bs][d]
    return out


def test_brute_force_on_tiny_workload():
    wl = workloads.tiny()
    rp = OracleReplay(wl)
    rp.run()
    (i, seqs, tables, lens), = rp.attends
    out = rp.decode(i, tables, lens)
    qf = to_f64(rp.q_values(i, len(lens)), "f16")
    kf = to_f64(rp.k_cache, "f16")
    vf = to_f64(rp.v_cache, "f16")
    ref = brute_force(qf.tolist(), kf.tolist(), vf.tolist(), tables, lens, wl.scale, 16)
    np.testing.assert_allclose(out, np.array(ref), rtol=1e-12, atol=1e-13)
    assert lens == [1, 15, 16, 37]


def test_closed_forms():
    bs = 2
    # weights 1:3 -> out = v0/4 + 3 v1/4 (z = [0, ln 3])
    k = np.zeros((4, 1, bs, 2))
    v = np.zeros((4, 1, bs, 2))
    k[2, 0, 1] = [math.log(3.0), 0.0]     # token 1 lives in block 2, slot 1
    v[2, 0, 0] = [1.0, 0.0]
    v[2, 0, 1] = [0.0, 1.0]
    q = np.array([[[1.0, 0.0]]])
    out = attention.paged_decode(q, k, v, [[2]], [2], 1.0, bs)
    np.testing.assert_allclose(out[0, 0], [0.25, 0.75], rtol=0, atol=1e-15)
    # ctx = 1 -> the single value vector, exactly
    rng = np.random.default_rng(5)
    k = rng.standard_normal((3, 2, 4, 8))
    v = rng.standard_normal((3, 2, 4, 8))
    q = rng.standard_normal((1, 2, 8))
    out = attention.paged_decode(q, k, v, [[1]], [1], 0.7, 4)
    assert np.array_equal(out[0], v[1, :, 0, :])
    # q = 0 -> uniform weights -> mean of the values
    out = attention.paged_decode(np.zeros((1, 2, 8)), k, v, [[2, 0]], [7], 0.7, 4)
    Vg = np.concatenate([v[2], v[0]], axis=1)[:, :7, :]
    np.testing.assert_allclose(out[0], Vg.mean(axis=1), rtol=1e-13, atol=1e-14)
    # all keys equal -> mean of the values whatever q is
    k_eq = np.broadcast_to(k[0, :, :1, :], k.shape).copy()
    out = attention.paged_decode(q, k_eq, v, [[2, 0]], [7], 0.7, 4)
    np.testing.assert_allclose(out[0], Vg.mean(axis=1), rtol=1e-13, atol=1e-14)
    # ctx = 0 -> zeros, no NaN
    out = attention.paged_decode(q, k, v, [[-1]], [0], 0.7, 4)
    assert np.array_equal(out, np.zeros_like(out))


@pytest.mark.parametrize("part", [1, 4, 16, 17, 64, 1000])
def test_split_merge_equals_unsplit(part):
    rng = np.random.default_rng(part)
    lens = [1, 33, 64, 200]
    q, k, v, bt = paged_random(rng, 4, 4, 2, 16, 16, lens)
    # large logits make the per-partition maxima differ by a lot
    q *= 4.0
    a = attention.paged_decode(q, k, v, bt, lens, 0.5, 16)
    b = attention.paged_decode_split(q, k, v, bt, lens, 0.5, 16, part)
    np.testing.assert_allclose(b, a, rtol=0, atol=1e-12)


def test_merge_of_one_partition_is_the_partition():
    rng = np.random.default_rng(9)
    K = rng.standard_normal((10, 4))
    V = rng.standard_normal((10, 4))
    q = rng.standard_normal(4)
    parts = attention.partition_partials(q, K, V, 1.0, 10)
    m, l, acc = parts[0]
    np.testing.assert_allclose(attention.merge_partials(parts), acc / l, rtol=0, atol=0)
    np.testing.assert_allclose(acc / l, attention.attend(q, K, V, 1.0), rtol=1e-14, atol=1e-15)


def test_cache_scatter_round_trips_through_block_tables():
    rng = np.random.default_rng(2)
    bm = BlockManager(8, 4, rng.permutation(8))
    s0, s1 = bm.create(), bm.create()
    kc = np.zeros((8, 2, 4, 3), np.uint16)
    vc = np.zeros_like(kc)
    toks = {s0: [], s1: []}
    for s, n in [(s0, 5), (s1, 3), (s0, 2), (s1, 6)]:
        slots = bm.append(s, n)
        k = rng.integers(0, 2**16, (n, 2, 3), dtype=np.uint16)
        v = rng.integers(0, 2**16, (n, 2, 3), dtype=np.uint16)
        cache.reshape_and_cache(kc, vc, k, v, slots, 4)
        toks[s].append((k, v))
    for s in (s0, s1):
        K = np.concatenate([k for k, _ in toks[s]])
        V = np.concatenate([v for _, v in toks[s]])
        for g in range(2):
            assert np.array_equal(attention.gather(kc, bm.block_table(s), len(K), g, 4), K[:, g])
            assert np.array_equal(attention.gather(vc, bm.block_table(s), len(V), g, 4), V[:, g])


def test_cache_padding_slots_skipped_and_last_write_wins():
    kc = np.zeros((2, 1, 2, 2), np.uint16)
    vc = np.zeros_like(kc)
    k = np.arange(8, dtype=np.uint16).reshape(4, 1, 2) + 1
    v = k + 100
    cache.reshape_and_cache(kc, vc, k, v, [3, -1, 0, 3], 2)
    assert kc[1, 0, 1].tolist() == k[3, 0].tolist()     # slot 3 written twice: last wins
    assert kc[0, 0, 0].tolist() == k[2, 0].tolist()
    assert int(kc.astype(np.int64).sum()) == int(k[3].sum() + k[2].sum())
    k1, v1 = kc[1].copy(), vc[1].copy()
    cache.copy_blocks(kc, vc, [(1, 0)])
    # dst receives src's contents; src is untouched
    assert np.array_equal(kc[0], k1) and np.array_equal(vc[0], v1)
    assert np.array_equal(kc[1], k1) and np.array_equal(vc[1], v1)
    assert not np.array_equal(k1, np.zeros_like(k1))


def test_bf16_decoding():
    # 1.0, -2.0, 0.5 and the smallest normal in bf16
    bits = np.array([0x3F80, 0xC000, 0x3F00, 0x0080], np.uint16)
    assert to_f64(bits, "bf16").tolist() == [1.0, -2.0, 0.5, 2.0**-126]
    bits = np.array([0x3C00, 0xC000, 0x3800, 0x0400], np.uint16)
    assert to_f64(bits, "f16").tolist() == [1.0, -2.0, 0.5, 2.0**-14]


# ---- paged prefill (a chunk of T new tokens per sequence, causal within the chunk)

def _prefill_batch(seed, lens, T, Hq=4, Hkv=2, D=16, bs=4):
    rng = np.random.default_rng(seed)
    need = [-(-L // bs) for L in lens]
    nb = sum(need) + 3
    perm = rng.permutation(nb)
    tables = np.full((len(lens), max(need)), -1, np.int64)
    i = 0
    for s, n in enumerate(need):
        tables[s, :n] = perm[i:i + n]
        i += n
    k = rng.standard_normal((nb, Hkv, bs, D))
    v = rng.standard_normal((nb, Hkv, bs, D))
    q = rng.standard_normal((len(lens), T, Hq, D))
    return q, k, v, tables, np.asarray(lens)


def test_prefill_of_one_token_is_decode():
    q, k, v, t, l = _prefill_batch(1, [5, 17, 9], T=1)
    a = attention.paged_prefill(q, k, v, t, l, 0.3, 4)
    b = attention.paged_decode(q[:, 0], k, v, t, l, 0.3, 4)
    assert np.array_equal(a[:, 0], b)


def test_prefill_rows_are_the_decodes_of_their_prefixes():
    """Query i of a chunk attends exactly what a decode step at length ctx - T + i + 1 would."""
    T = 6
    q, k, v, t, l = _prefill_batch(2, [6, 11, 23], T=T)
    out = attention.paged_prefill(q, k, v, t, l, 0.25, 4)
    for i in range(T):
        lens_i = l - T + i + 1
        ref = attention.paged_decode(q[:, i], k, v, t, lens_i, 0.25, 4)
        assert np.allclose(out[:, i], ref, atol=1e-12, rtol=0)


def test_prefill_matches_sdpa_with_an_explicit_causal_mask():
    """torch fp64 scaled_dot_product_attention on the gathered contiguous K/V, with the
    bottom-right causal mask (query i at position L - T + i) built as a boolean matrix."""
    torch = pytest.importorskip("torch")
    T, Hq, Hkv = 5, 4, 2
    q, k, v, t, l = _prefill_batch(3, [5, 9, 20], T=T, Hq=Hq, Hkv=Hkv)
    out = attention.paged_prefill(q, k, v, t, l, 0.2, 4)
    for s, L in enumerate(l):
        for g in range(Hkv):
            K = torch.from_numpy(attention.gather(k, t[s], L, g, 4))
            V = torch.from_numpy(attention.gather(v, t[s], L, g, 4))
            mask = torch.arange(L)[None, :] <= (L - T + torch.arange(T))[:, None]
            for hh in range(g * (Hq // Hkv), (g + 1) * (Hq // Hkv)):
                Q = torch.from_numpy(q[s, :, hh])
                ref = torch.nn.functional.scaled_dot_product_attention(
                    Q[None], K[None], V[None], attn_mask=mask[None], scale=0.2)[0].numpy()
                assert np.allclose(out[s, :, hh], ref, atol=1e-12, rtol=0)


def test_prefill_closed_forms():
    """A whole prompt (ctx = T): row 0 is v_0 exactly; zero queries give the mean of the
    visible values, a different mean for every row; queries with no visible token give 0."""
    T = 7
    q, k, v, t, l = _prefill_batch(4, [7, 3], T=T, Hq=2, Hkv=2)
    out = attention.paged_prefill(q, k, v, t, l, 0.5, 4)
    V0 = attention.gather(v, t[0], 7, 0, 4)
    assert np.array_equal(out[0, 0, 0], V0[0])
    qz = np.zeros_like(q)
    outz = attention.paged_prefill(qz, k, v, t, l, 0.5, 4)
    for i in range(T):
        assert np.allclose(outz[0, i, 0], V0[:i + 1].mean(axis=0), atol=1e-13)
    # sequence 1 holds 3 tokens but the chunk has 7: queries 0..3 see nothing
    assert not outz[1, :4].any()
    V1 = attention.gather(v, t[1], 3, 1, 4)
    assert np.allclose(outz[1, 6, 1], V1.mean(axis=0), atol=1e-13)
