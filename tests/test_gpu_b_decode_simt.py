"""paged_attention_decode, one query head per KV head (CUDA-core kernel), against the oracle."""

import math

import numpy as np
import pytest

from oracle import attention
from oracle.numerics import to_f64
from parity import check_close, from_bits, random_paged_batch, to_bits

pytestmark = pytest.mark.gpu


def run_gpu(q, k, v, tables, lens, dtype, scale, partition, max_ctx=None):
    import torch
    import paged_kv_cache_319_b200 as kvp

    out = kvp.paged_attention_decode(
        from_bits(q, dtype), from_bits(k, dtype), from_bits(v, dtype),
        torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(), scale,
        max_context_len=int(max(lens.max(), 1)) if max_ctx is None else max_ctx,
        partition_size=partition)
    kvp.check_device_error()
    return to_bits(out)


def oracle(q, k, v, tables, lens, dtype, scale, bs):
    return attention.paged_decode(to_f64(q, dtype), k, v, tables, lens, scale, bs, dtype=dtype)


CASES = [
    # (Hq, D, bs, lens, dtype, partition)
    (4, 64, 16, [1, 15, 16, 37], "f16", 0),
    (8, 128, 16, [1, 2, 15, 16, 17, 100, 513, 1000, 2048], "f16", 0),
    (8, 128, 16, [1, 2, 15, 16, 17, 100, 513, 1000, 2048], "f16", 512),
    (8, 128, 16, [511, 512, 513, 1024, 1537], "f16", 256),
    (6, 128, 32, [3, 31, 32, 33, 700], "f16", 512),
    (6, 128, 8, [3, 7, 8, 9, 300], "f16", 64),
    (5, 64, 8, [1, 9, 129, 555], "bf16", 128),
    (5, 128, 16, [40, 600, 1300], "bf16", 512),
]


@pytest.mark.parametrize("Hq,D,bs,lens,dtype,partition", CASES)
def test_matches_oracle(Hq, D, bs, lens, dtype, partition):
    S = len(lens)
    q, k, v, t, l = random_paged_batch(hash((Hq, D, bs, partition)) % 10**6, S, Hq, Hq, D, bs,
                                       lens, dtype)
    scale = 1 / math.sqrt(D)
    got = run_gpu(q, k, v, t, l, dtype, scale, partition)
    ref = oracle(q, k, v, t, l, dtype, scale, bs)
    check_close(got, ref, dtype, allow_ulp=(dtype == "bf16"))


def test_split_equals_unsplit_within_rounding():
    q, k, v, t, l = random_paged_batch(77, 4, 8, 8, 128, 16, [900, 1500, 2048, 40], "f16")
    a = to_f64(run_gpu(q, k, v, t, l, "f16", 0.09, 0), "f16")
    b = to_f64(run_gpu(q, k, v, t, l, "f16", 0.09, 512), "f16")
    assert np.abs(a - b).max() < 2e-3


def test_physical_placement_does_not_change_output_bits():
    q, k, v, t, l = random_paged_batch(5, 3, 4, 4, 128, 16, [300, 77, 1024], "f16")
    rng = np.random.default_rng(1)
    perm = rng.permutation(k.shape[0])
    k2, v2 = np.empty_like(k), np.empty_like(v)
    k2[perm], v2[perm] = k, v
    t2 = np.where(t >= 0, perm[np.maximum(t, 0)], -1).astype(np.int32)
    for part in (0, 256):
        a = run_gpu(q, k, v, t, l, "f16", 0.1, part)
        b = run_gpu(q, k2, v2, t2, l, "f16", 0.1, part)
        assert np.array_equal(a, b)


def test_context_of_one_returns_v_exactly_and_zero_gives_zeros():
    q, k, v, t, l = random_paged_batch(9, 3, 4, 4, 128, 16, [1, 0, 1], "f16")
    got = run_gpu(q, k, v, t, l, "f16", 0.1, 0, max_ctx=16)
    assert np.array_equal(got[0], v[t[0, 0], :, 0, :])
    assert np.array_equal(got[2], v[t[2, 0], :, 0, :])
    assert not got[1].any()


def test_non_finite_values_past_the_end_do_not_leak():
    q, k, v, t, l = random_paged_batch(11, 2, 4, 4, 128, 16, [20, 33], "f16")
    ref = oracle(q, k, v, t, l, "f16", 0.1, 16)
    nan16, inf16 = np.uint16(0x7E00), np.uint16(0x7C00)
    for s, L in enumerate(l):
        blk = t[s, (L - 1) // 16]
        k[blk, :, L % 16:, :] = nan16
        v[blk, :, L % 16:, :] = inf16
    for part in (0, 16):
        got = run_gpu(q, k, v, t, l, "f16", 0.1, part)
        check_close(got, ref, "f16")


def test_bad_block_id_is_reported():
    import paged_kv_cache_319_b200 as kvp

    q, k, v, t, l = random_paged_batch(3, 2, 4, 4, 64, 16, [40, 20], "f16")
    t[0, 1] = k.shape[0] + 5
    with pytest.raises(kvp.KvpError) as e:
        run_gpu(q, k, v, t, l, "f16", 0.1, 0)
    assert e.value.kind == "bounds"
    kvp.check_device_error()
