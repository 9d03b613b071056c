"""paged_attention_decode for grouped-query heads (tcgen05 tensor-core kernel) against the oracle."""

import math

import numpy as np
import pytest

from oracle.numerics import to_f64
from parity import check_close, random_paged_batch
from test_gpu_b_decode_simt import oracle, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # (Hq, Hkv, bs, lens, dtype, partition)
    (8, 2, 16, [1, 100, 128, 129, 511, 512, 513, 2000], "bf16", 512),
    (8, 2, 16, [1, 100, 128, 129, 511, 512, 513, 2000], "f16", 512),
    (32, 8, 32, [5, 127, 640, 1500, 3001], "bf16", 512),
    (32, 8, 16, [5, 127, 640, 1500, 3001], "bf16", 0),
    (16, 8, 16, [64, 700, 1200], "f16", 1024),
    (64, 8, 16, [257, 1025], "bf16", 512),
    (48, 3, 32, [300, 900], "f16", 128),
    (12, 4, 16, [50, 1000], "bf16", 256),
]


@pytest.mark.parametrize("Hq,Hkv,bs,lens,dtype,partition", CASES)
def test_matches_oracle(Hq, Hkv, bs, lens, dtype, partition):
    S = len(lens)
    q, k, v, t, l = random_paged_batch(hash((Hq, Hkv, bs, partition)) % 10**6, S, Hq, Hkv, 128,
                                       bs, lens, dtype)
    scale = 1 / math.sqrt(128)
    got = run_gpu(q, k, v, t, l, dtype, scale, partition)
    ref = oracle(q, k, v, t, l, dtype, scale, bs)
    check_close(got, ref, dtype, allow_ulp=True)


def test_physical_placement_does_not_change_output_bits():
    q, k, v, t, l = random_paged_batch(21, 3, 16, 4, 128, 16, [300, 77, 1024], "bf16")
    rng = np.random.default_rng(2)
    perm = rng.permutation(k.shape[0])
    k2, v2 = np.empty_like(k), np.empty_like(v)
    k2[perm], v2[perm] = k, v
    t2 = np.where(t >= 0, perm[np.maximum(t, 0)], -1).astype(np.int32)
    for part in (0, 512):
        a = run_gpu(q, k, v, t, l, "bf16", 0.1, part)
        b = run_gpu(q, k2, v2, t2, l, "bf16", 0.1, part)
        assert np.array_equal(a, b)


def test_context_edge_cases():
    q, k, v, t, l = random_paged_batch(23, 3, 8, 2, 128, 16, [1, 0, 2], "bf16")
    got = run_gpu(q, k, v, t, l, "bf16", 0.1, 512, max_ctx=16)
    assert not got[1].any()
    ref = oracle(q, k, v, t, l, "bf16", 0.1, 16)
    check_close(got, ref, "bf16", allow_ulp=True)


def test_non_finite_values_past_the_end_do_not_leak():
    q, k, v, t, l = random_paged_batch(25, 2, 8, 2, 128, 16, [20, 200], "bf16")
    ref = oracle(q, k, v, t, l, "bf16", 0.1, 16)
    nan, inf = np.uint16(0x7FC0), np.uint16(0x7F80)
    for s, L in enumerate(l):
        blk = t[s, (L - 1) // 16]
        k[blk, :, L % 16:, :] = nan
        v[blk, :, L % 16:, :] = inf
    for part in (0, 128):
        got = run_gpu(q, k, v, t, l, "bf16", 0.1, part)
        check_close(got, ref, "bf16", allow_ulp=True)


def test_bad_block_id_is_reported():
    import paged_kv_cache_319_b200 as kvp

    q, k, v, t, l = random_paged_batch(27, 2, 8, 2, 128, 16, [400, 20], "bf16")
    t[0, 3] = -7
    with pytest.raises(kvp.KvpError) as e:
        run_gpu(q, k, v, t, l, "bf16", 0.1, 0)
    assert e.value.kind == "bounds"
    kvp.check_device_error()
