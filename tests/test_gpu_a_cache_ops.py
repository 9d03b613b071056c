"""reshape_and_cache and copy_blocks on the GPU against the oracle: bit-exact pools."""

import numpy as np
import pytest

from oracle import cache as ocache
from parity import from_bits, to_bits
import workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("Hkv,bs,D,dtype", [(3, 16, 64, "f16"), (40, 16, 128, "f16"),
                                            (8, 32, 128, "bf16"), (2, 8, 128, "bf16")])
def test_reshape_and_cache_bit_exact(Hkv, bs, D, dtype):
    import torch
    import paged_kv_cache_319_b200 as kvp

    rng = np.random.default_rng(Hkv * 1000 + bs)
    nb = 37
    T = 150
    slots = rng.choice(nb * bs, size=T, replace=False).astype(np.int64)
    slots[rng.choice(T, size=9, replace=False)] = -1          # padding tokens
    k0 = workloads.normal_bits([1, Hkv], (nb, Hkv, bs, D), dtype)
    v0 = workloads.normal_bits([2, Hkv], (nb, Hkv, bs, D), dtype)
    kn = workloads.normal_bits([3, Hkv], (T, Hkv, D), dtype)
    vn = workloads.normal_bits([4, Hkv], (T, Hkv, D), dtype)
    kc, vc = from_bits(k0, dtype), from_bits(v0, dtype)
    kvp.reshape_and_cache(from_bits(kn, dtype), from_bits(vn, dtype), kc, vc,
                          torch.from_numpy(slots).cuda())
    kvp.check_device_error()
    ko, vo = k0.copy(), v0.copy()
    ocache.reshape_and_cache(ko, vo, kn, vn, slots, bs)
    assert np.array_equal(to_bits(kc), ko)
    assert np.array_equal(to_bits(vc), vo)


def test_reshape_and_cache_out_of_range_slot_is_reported():
    import torch
    import paged_kv_cache_319_b200 as kvp

    nb, Hkv, bs, D = 4, 2, 16, 64
    kc = torch.zeros((nb, Hkv, bs, D), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.ones((2, Hkv, D), dtype=torch.float16, device="cuda")
    slots = torch.tensor([5, nb * bs], dtype=torch.int64, device="cuda")
    kvp.reshape_and_cache(kn, kn, kc, vc, slots)
    with pytest.raises(kvp.KvpError) as e:
        kvp.check_device_error()
    assert e.value.kind == "bounds"
    assert float(kc.float().sum()) == Hkv * D          # only the valid token was written
    kvp.check_device_error()                           # the word was cleared


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_copy_blocks_bit_exact(dtype):
    import torch
    import paged_kv_cache_319_b200 as kvp

    nb, Hkv, bs, D = 30, 40, 16, 128
    k0 = workloads.normal_bits([5], (nb, Hkv, bs, D), dtype)
    v0 = workloads.normal_bits([6], (nb, Hkv, bs, D), dtype)
    pairs = [(3, 17), (3, 18), (9, 0), (29, 5)]
    kc, vc = from_bits(k0, dtype), from_bits(v0, dtype)
    kvp.copy_blocks(kc, vc, torch.tensor(pairs, dtype=torch.int32, device="cuda"))
    kvp.check_device_error()
    ko, vo = k0.copy(), v0.copy()
    ocache.copy_blocks(ko, vo, pairs)
    assert np.array_equal(to_bits(kc), ko)
    assert np.array_equal(to_bits(vc), vo)


def test_copy_blocks_bad_pair_is_reported():
    import torch
    import paged_kv_cache_319_b200 as kvp

    kc = torch.zeros((4, 1, 16, 64), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    kvp.copy_blocks(kc, vc, torch.tensor([[0, 4]], dtype=torch.int32, device="cuda"))
    with pytest.raises(kvp.KvpError) as e:
        kvp.check_device_error()
    assert e.value.kind == "bounds"
