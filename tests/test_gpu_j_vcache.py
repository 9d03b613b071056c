"""Virtually contiguous KV cache (CUDA virtual memory management) on the GPU.

The alternative to block tables that the pages name: each sequence's keys and
values stay contiguous in virtual memory and physical chunks are mapped on
demand ("Your GPU was mostly empty", section "The tradeoff: you just wrote a
virtual memory subsystem in userspace"). Checked here:

* writes land bit for bit where the token-major layout says (read back through
  views of the mapped ranges);
* decode over the contiguous cache equals the fp64 oracle run through an
  identity block table (block size 1, table entry j of sequence s = the flat
  token index of its slot's token j), element by element within the parity
  tolerance, on the CUDA cores and on the tensor cores;
* with the same data, the CUDA-core decode reads the same tiles in the same
  order as the paged decode over a block-16 pool, so the two outputs are
  identical bit for bit (only the address translation differs);
* contexts beyond a slot's capacity are clamped (and reported), a slot out of
  range reads nothing, and trimmed chunks are reused by later growth.
"""

import numpy as np
import pytest

from oracle import attention
from oracle.numerics import to_f64
from parity import check_close, from_bits, to_bits
import workloads

pytestmark = pytest.mark.gpu

D = 128


def _fill(vc, lens, Hkv, dtype, seed):
    """Reserves each slot to its length and writes seeded K/V for every token.
    Returns the host bits [S, maxL, Hkv, D] of K and V (zeros past each length)."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    S, L = len(lens), max(lens)
    kh = np.zeros((S, L, Hkv, D), np.uint16)
    vh = np.zeros((S, L, Hkv, D), np.uint16)
    slots, pos = [], []
    for s, n in enumerate(lens):
        vc.reserve(s, n)
        kh[s, :n] = workloads.normal_bits([seed, 1, s], (n, Hkv, D), dtype)
        vh[s, :n] = workloads.normal_bits([seed, 2, s], (n, Hkv, D), dtype)
        slots += [s] * n
        pos += list(range(n))
    rows = [(s, j) for s, n in enumerate(lens) for j in range(n)]
    k_new = np.stack([kh[s, j] for s, j in rows])
    v_new = np.stack([vh[s, j] for s, j in rows])
    kvp.reshape_and_cache_vcache(from_bits(k_new, dtype), from_bits(v_new, dtype), vc,
                                 torch.tensor(slots, dtype=torch.int32, device="cuda"),
                                 torch.tensor(pos, dtype=torch.int32, device="cuda"))
    kvp.check_device_error()
    return kh, vh


def _oracle(q_bits, kh, vh, lens, dtype, scale):
    """fp64 oracle through an identity block table over a block-size-1 pool."""
    S, L, Hkv, _ = kh.shape
    k_pool = kh.reshape(S * L, Hkv, 1, D)
    v_pool = vh.reshape(S * L, Hkv, 1, D)
    tables = np.full((S, L), -1, np.int32)
    for s, n in enumerate(lens):
        tables[s, :n] = s * L + np.arange(n)
    return attention.paged_decode(to_f64(q_bits, dtype), k_pool, v_pool, tables, lens, scale, 1,
                                  dtype=dtype)


CASES = [
    # (Hq, Hkv, lens, dtype, partition): CUDA cores (G = 1) and tensor cores (G > 1)
    (8, 8, [1, 15, 16, 17, 300, 2048], "f16", 0),
    (8, 8, [1, 15, 16, 17, 300, 2048], "f16", 512),
    (8, 8, [5, 700, 1500], "bf16", 512),
    (32, 8, [1, 100, 129, 5000, 9000], "bf16", 512),
    (16, 4, [7, 128, 256, 3000], "f16", 1024),
    (64, 4, [33, 1024, 2500], "bf16", 512),
    # 130 sequences: the CUDA cores' one-stage shape for large batches
    (8, 8, [1, 16, 17, 200, 511] * 26, "f16", 256),
]


@pytest.mark.parametrize("Hq,Hkv,lens,dtype,part", CASES)
def test_vcache_decode_matches_the_oracle(Hq, Hkv, lens, dtype, part):
    import torch
    import paged_kv_cache_319_b200 as kvp

    S = len(lens)
    vc = kvp.VCache(S + 2, max(lens) + 37, Hkv, D, dtype)
    try:
        kh, vh = _fill(vc, lens, Hkv, dtype, seed=11 + Hq)
        # the writes, bit for bit, through views of the mapped ranges
        for s, n in enumerate(lens):
            assert np.array_equal(to_bits(vc.view("k", s, n)), kh[s, :n])
            assert np.array_equal(to_bits(vc.view("v", s, n)), vh[s, :n])
        q_bits = workloads.normal_bits([17, Hq, S], (S, Hq, D), dtype)
        scale = 1 / np.sqrt(D)
        out = kvp.attention_decode_vcache(
            from_bits(q_bits, dtype), vc, torch.arange(S, dtype=torch.int32, device="cuda"),
            torch.tensor(lens, dtype=torch.int32, device="cuda"), scale,
            max_context_len=max(lens), partition_size=part)
        kvp.check_device_error()
        # short bf16 contexts: half a bf16 ulp on top of 2e-3, as the other bf16 cases
        check_close(to_bits(out), _oracle(q_bits, kh, vh, np.asarray(lens), dtype, scale), dtype,
                    allow_ulp=dtype == "bf16")
    finally:
        vc.close()


def test_vcache_slots_in_any_order():
    # sequence s reads slot seq_slots[s]: a permuted assignment permutes nothing else
    import torch
    import paged_kv_cache_319_b200 as kvp

    lens = [40, 900, 1, 333]
    vc = kvp.VCache(6, 1024, 8, D, "f16")
    try:
        kh, vh = _fill(vc, lens, 8, "f16", seed=5)
        order = [2, 0, 3, 1]
        q_bits = workloads.normal_bits([9], (4, 8, D), "f16")
        out = kvp.attention_decode_vcache(
            from_bits(q_bits, "f16"), vc, torch.tensor(order, dtype=torch.int32, device="cuda"),
            torch.tensor([lens[o] for o in order], dtype=torch.int32, device="cuda"),
            1 / np.sqrt(D), max_context_len=1024, partition_size=256)
        kvp.check_device_error()
        want = _oracle(q_bits, kh[order], vh[order], np.asarray([lens[o] for o in order]), "f16",
                       1 / np.sqrt(D))
        check_close(to_bits(out), want, "f16")
    finally:
        vc.close()


@pytest.mark.parametrize("part,lens", [(0, [1, 16, 17, 511, 1200, 2048]),
                                       (512, [1, 16, 17, 511, 1200, 2048]),
                                       # 130 sequences: both take the one-stage shape
                                       (256, [1, 16, 17, 200, 511] * 26)])
def test_vcache_equals_paged_decode_bit_for_bit_on_the_cuda_cores(part, lens):
    # same tiles (16 tokens), same warps, same order: only the address differs
    import torch
    import paged_kv_cache_319_b200 as kvp

    S, Hkv, bs = len(lens), 8, 16
    vc = kvp.VCache(S, max(lens), Hkv, D, "f16")
    try:
        kh, vh = _fill(vc, lens, Hkv, "f16", seed=23)
        need = [-(-n // bs) for n in lens]
        nb = sum(need) + 3
        perm = np.random.default_rng(3).permutation(nb).astype(np.int32)
        tables = np.full((S, max(need)), -1, np.int32)
        kp = np.zeros((nb, Hkv, bs, D), np.uint16)
        vp = np.zeros((nb, Hkv, bs, D), np.uint16)
        i = 0
        for s, n in enumerate(lens):
            for b in range(need[s]):
                blk = perm[i]
                tables[s, b] = blk
                m = min(bs, n - b * bs)
                kp[blk, :, :m] = kh[s, b * bs:b * bs + m].transpose(1, 0, 2)
                vp[blk, :, :m] = vh[s, b * bs:b * bs + m].transpose(1, 0, 2)
                i += 1
        q = from_bits(workloads.normal_bits([29], (S, Hkv, D), "f16"), "f16")
        cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        paged = kvp.paged_attention_decode(q, from_bits(kp, "f16"), from_bits(vp, "f16"),
                                           torch.from_numpy(tables).cuda(), cl, 0.088,
                                           max_context_len=max(lens), partition_size=part)
        contig = kvp.attention_decode_vcache(q, vc, torch.arange(S, dtype=torch.int32, device="cuda"),
                                             cl, 0.088, max_context_len=max(lens), partition_size=part)
        kvp.check_device_error()
        assert np.array_equal(to_bits(paged), to_bits(contig))
    finally:
        vc.close()


def test_vcache_clamps_to_capacity_and_skips_bad_slots():
    import torch
    import paged_kv_cache_319_b200 as kvp

    lens = [300, 50]
    vc = kvp.VCache(2, 4096, 8, D, "f16")
    try:
        kh, vh = _fill(vc, lens, 8, "f16", seed=31)
        cap0 = vc.capacity(0)
        assert 300 <= cap0 < 4096
        # the capacity past token 300 holds whatever the chunk held: write zeros there
        nz = cap0 - 300
        z = from_bits(np.zeros((nz, 8, D), np.uint16), "f16")
        kvp.reshape_and_cache_vcache(z, z, vc, torch.zeros(nz, dtype=torch.int32, device="cuda"),
                                     torch.arange(300, cap0, dtype=torch.int32, device="cuda"))
        kvp.check_device_error()
        # a context past the capacity reads only the capacity, and is reported
        q_bits = workloads.normal_bits([37], (2, 8, D), "f16")
        q = from_bits(q_bits, "f16")
        big = torch.tensor([cap0 + 500, 50], dtype=torch.int32, device="cuda")
        out = kvp.attention_decode_vcache(q, vc, torch.tensor([0, 1], dtype=torch.int32,
                                                              device="cuda"),
                                          big, 0.1, max_context_len=4096, partition_size=512)
        with pytest.raises(kvp.KvpError) as e:
            kvp.check_device_error()
        assert e.value.kind == "bounds"
        k_cap = to_bits(vc.view("k", 0, cap0))
        v_cap = to_bits(vc.view("v", 0, cap0))
        want = _oracle(q_bits[:1], k_cap[None], v_cap[None], np.asarray([cap0]), "f16", 0.1)
        check_close(to_bits(out)[:1], want, "f16")
        # a slot out of range reads nothing: zero row, reported
        out = kvp.attention_decode_vcache(q, vc, torch.tensor([0, 7], dtype=torch.int32,
                                                              device="cuda"),
                                          torch.tensor([300, 50], dtype=torch.int32, device="cuda"),
                                          0.1, max_context_len=4096, partition_size=512)
        with pytest.raises(kvp.KvpError):
            kvp.check_device_error()
        assert not to_bits(out)[1].any()
        check_close(to_bits(out)[:1], _oracle(q_bits[:1], kh[:1], vh[:1], np.asarray([300]),
                                              "f16", 0.1), "f16")
        # writes past the capacity are skipped and reported, never made
        k1 = from_bits(np.ones((1, 8, D), np.uint16), "f16")
        kvp.reshape_and_cache_vcache(k1, k1, vc, torch.tensor([1], dtype=torch.int32, device="cuda"),
                                     torch.tensor([vc.capacity(1)], dtype=torch.int32, device="cuda"))
        with pytest.raises(kvp.KvpError) as e:
            kvp.check_device_error()
        assert e.value.kind == "bounds"
    finally:
        vc.close()


def test_vcache_grows_trims_and_reuses_chunks():
    import torch
    import paged_kv_cache_319_b200 as kvp

    Hkv = 40
    vc = kvp.VCache(4, 2048, Hkv, D, "f16")
    try:
        st0 = vc.stats()
        chunk = st0["chunk_bytes"]
        token_bytes = Hkv * D * 2
        assert st0["mapped_chunks"] == 0 and vc.capacity(0) == 0
        assert st0["slot_tokens"] * token_bytes % chunk == 0
        vc.reserve(0, 1)
        st1 = vc.stats()
        # one token plus the mapped tail, K and V
        per = -(-(1 + 256) * token_bytes // chunk)
        assert st1["mapped_chunks"] == 2 * per
        assert vc.capacity(0) == min(2048, per * chunk // token_bytes - 256)
        vc.reserve(0, 2048)
        full = 2 * -(-(2048 + 256) * token_bytes // chunk)
        assert vc.stats()["mapped_chunks"] == full and vc.capacity(0) == 2048
        created = vc.stats()["create_calls"]
        vc.trim(0, 0)
        st = vc.stats()
        assert st["mapped_chunks"] == 0 and st["spare_chunks"] == full and vc.capacity(0) == 0
        vc.reserve(3, 2048)  # another slot takes the spares: no new physical chunks
        st = vc.stats()
        assert st["create_calls"] == created and st["spare_chunks"] == 0
        # the reused memory is the new slot's own: write and read back
        kh, vh = _fill(vc, [0, 0, 0, 700], Hkv, "f16", seed=41)
        assert np.array_equal(to_bits(vc.view("k", 3, 700)), kh[3, :700])
        with pytest.raises(ValueError):
            vc.view("k", 0, 1)  # slot 0 is unmapped now
        with pytest.raises(kvp.KvpError):
            vc.reserve(1, 2049)  # beyond max_tokens
        vc.release_spares()
        torch.cuda.synchronize()
    finally:
        vc.close()


def test_vcache_reserve_batch_all_or_nothing():
    import paged_kv_cache_319_b200 as kvp

    vc = kvp.VCache(3, 3000, 8, D, "bf16")
    try:
        vc.reserve_batch(np.array([0, 2]), np.array([100, 2500]))
        assert vc.capacity(0) >= 100 and vc.capacity(2) >= 2500 and vc.capacity(1) == 0
        before = (vc.stats(), [vc.capacity(s) for s in range(3)])
        for slots, toks in (([1, 5], [10, 10]), ([1, 0], [10, 3001]), ([1], [-1])):
            with pytest.raises(kvp.KvpError) as e:
                vc.reserve_batch(np.array(slots), np.array(toks))
            assert e.value.kind == "invalid"
            assert (vc.stats(), [vc.capacity(s) for s in range(3)]) == before
    finally:
        vc.close()
