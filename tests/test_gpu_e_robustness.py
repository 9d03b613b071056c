"""Failure paths on the GPU that neither fault nor hang: bounded waits, bad lengths, empty calls."""

import ctypes as C

import numpy as np
import pytest

from parity import check_close, random_paged_batch
from test_gpu_b_decode_simt import oracle, run_gpu

pytestmark = pytest.mark.gpu


def test_a_wait_that_never_completes_ends_with_a_status():
    import torch
    import paged_kv_cache_319_b200 as kvp
    from paged_kv_cache_319_b200 import _lib

    lib = _lib.lib()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.kvp_selftest_bounded_wait(50, stream) == 0
    with pytest.raises(kvp.KvpError) as e:
        kvp.check_device_error()
    assert e.value.kind == "cuda" and "timed out" in str(e.value)
    # the context is still usable: a decode right after is correct
    q, k, v, t, l = random_paged_batch(31, 2, 4, 4, 128, 16, [40, 300], "f16")
    got = run_gpu(q, k, v, t, l, "f16", 0.1, 0)
    check_close(got, oracle(q, k, v, t, l, "f16", 0.1, 16), "f16")
    assert lib.kvp_selftest_bounded_wait(0, stream) == _lib.KVP_ERR_INVALID


@pytest.mark.parametrize("Hq,Hkv,dtype", [(4, 4, "f16"), (16, 4, "bf16")])
def test_context_length_beyond_the_maximum_is_reported_and_clamped(Hq, Hkv, dtype):
    import torch
    import paged_kv_cache_319_b200 as kvp
    from parity import from_bits

    q, k, v, t, l = random_paged_batch(33, 2, Hq, Hkv, 128, 16, [64, 64], dtype)
    bad = l.copy()
    bad[1] = 500                       # more than max_context_len = 64
    out = kvp.paged_attention_decode(from_bits(q, dtype), from_bits(k, dtype), from_bits(v, dtype),
                                     torch.from_numpy(t).cuda(), torch.from_numpy(bad).cuda(),
                                     0.1, max_context_len=64, partition_size=0)
    with pytest.raises(kvp.KvpError) as e:
        kvp.check_device_error()
    assert e.value.kind == "bounds"
    # clamped to 64 tokens: the same as the valid call
    from parity import to_bits
    ref = oracle(q, k, v, t, l, dtype, 0.1, 16)
    check_close(to_bits(out), ref, dtype, allow_ulp=True)


def test_empty_calls_launch_nothing_and_succeed():
    import torch
    import paged_kv_cache_319_b200 as kvp

    kc = torch.zeros((4, 2, 16, 64), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    kvp.reshape_and_cache(torch.empty((0, 2, 64), dtype=torch.float16, device="cuda"),
                          torch.empty((0, 2, 64), dtype=torch.float16, device="cuda"), kc, vc,
                          torch.empty((0,), dtype=torch.int64, device="cuda"))
    kvp.copy_blocks(kc, vc, torch.empty((0, 2), dtype=torch.int32, device="cuda"))
    out = kvp.paged_attention_decode(torch.empty((0, 2, 64), dtype=torch.float16, device="cuda"),
                                     kc, vc, torch.empty((0, 1), dtype=torch.int32, device="cuda"),
                                     torch.empty((0,), dtype=torch.int32, device="cuda"), 0.1)
    assert out.shape == (0, 2, 64)
    kvp.check_device_error()
    assert float(kc.float().abs().sum()) == 0.0


@pytest.mark.parametrize("Hq,Hkv,dtype,part", [(4, 4, "f16", 0), (4, 4, "f16", 256),
                                               (8, 2, "bf16", 512), (8, 2, "bf16", 0)])
def test_contexts_that_fill_the_block_table_exactly(Hq, Hkv, dtype, part):
    lens = [2048, 2048, 1]
    q, k, v, t, l = random_paged_batch(35, 3, Hq, Hkv, 128, 16, lens, dtype, extra_blocks=0)
    assert t.shape[1] * 16 == 2048
    got = run_gpu(q, k, v, t, l, dtype, 0.09, part, max_ctx=2048)
    check_close(got, oracle(q, k, v, t, l, dtype, 0.09, 16), dtype, allow_ulp=True)
