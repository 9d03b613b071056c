"""paged_attention_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: an engine whose allocator has already
reserved all free device memory for its KV pool, or a latency-critical path
that cannot afford cudaMalloc's implicit synchronisation. For them the library
serves the split-context scratch from one static device array instead of a
caller-given workspace. These tests call that entry point through the C ABI
and check, on two calls in a row (the second with different inputs, so stale
scratch from the first would show), that its output matches the output of the
workspace-taking entry point within the parity tolerance of the other tests,
and that both match the fp64 oracle within that tolerance (for bf16, plus
half a bf16 ulp of the reference, as the other short-context bf16 tests). Batches whose
contexts fit one partition (or that do not split at all) need no scratch;
they are checked the same way. This file is collected last on purpose.
"""

import ctypes as C

import numpy as np
import pytest

from oracle import attention
from oracle.numerics import to_f64
from parity import ATOL, RTOL_NORM, check_close, from_bits, random_paged_batch, to_bits

pytestmark = pytest.mark.gpu

CASES = [
    # (Hq, Hkv, block_size, context lengths, dtype), partitions of 512 tokens:
    # one CUDA-core case (one query head per KV head) and one tensor-core case.
    (8, 8, 16, [1, 700, 1500, 2048, 3000], "f16"),
    (32, 8, 16, [100, 5000, 9000], "bf16"),
]
PART = 512
SCALE = 1 / np.sqrt(128.0)


def _inputs(seed, Hq, Hkv, bs, lens, dtype):
    import torch

    bits = random_paged_batch(seed, len(lens), Hq, Hkv, 128, bs, lens, dtype)
    q, k, v, t, l = bits
    dev = (from_bits(q, dtype), from_bits(k, dtype), from_bits(v, dtype),
           torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda())
    return dev, bits


def _common_args(q, k, t, l, Hq, Hkv, bs, max_ctx, part=PART):
    S = q.shape[0]
    return [q.data_ptr(), k.data_ptr(), None, t.data_ptr(), l.data_ptr(), S, Hq, Hkv, 128, bs,
            k.shape[0], t.shape[1], max_ctx, C.c_float(SCALE), part]


def _close(a, b):
    assert not np.isnan(a).any()
    assert np.abs(a - b).max() <= ATOL
    assert np.linalg.norm(a - b) <= RTOL_NORM * np.linalg.norm(b)


def _run_both(lib, _lib, case, seed, part, expect_scratch):
    """One call of each entry point on the same seeded batch; both compared with
    each other and with the fp64 oracle."""
    import torch

    Hq, Hkv, bs, lens, dtype = case
    code = _lib.KVP_F16 if dtype == "f16" else _lib.KVP_BF16
    (q, k, v, t, l), (qb, kb, vb, tb, lb) = _inputs(seed, Hq, Hkv, bs, lens, dtype)
    max_ctx = int(max(lens))
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = _common_args(q, k, t, l, Hq, Hkv, bs, max_ctx, part)
    args[2] = v.data_ptr()
    need = lib.kvp_decode_workspace_bytes(q.shape[0], Hq, 128, max_ctx, part)
    assert need <= _lib.KVP_STATIC_SCRATCH_BYTES
    assert (need > 0) == expect_scratch
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(q)
    got = torch.full_like(q, float("nan"))
    rc = lib.paged_attention_decode(*args, ws.data_ptr() if need else None, need, ref.data_ptr(),
                                    code, stream)
    assert rc == 0, lib.kvp_last_error_message()
    rc = lib.paged_attention_decode_noalloc(*args, got.data_ptr(), code, stream)
    assert rc == 0, lib.kvp_last_error_message()
    assert lib.kvp_check_device_error(stream) == 0, lib.kvp_last_error_message()
    a = to_f64(to_bits(got), dtype)
    b = to_f64(to_bits(ref), dtype)
    _close(a, b)
    want = attention.paged_decode(to_f64(qb, dtype), kb, vb, tb, lb, SCALE, bs, dtype=dtype)
    # short bf16 contexts give outputs near 1, which bf16 holds only to half an
    # ulp: the parity tests' rule for them allows that on top of 2e-3
    check_close(to_bits(got), want, dtype, allow_ulp=dtype == "bf16")


def test_noalloc_matches_the_workspace_entry_on_two_calls_in_a_row():
    from paged_kv_cache_319_b200 import _lib

    lib = _lib.lib()
    for case in CASES:
        for call in range(2):
            _run_both(lib, _lib, case, 1000 * call + case[0], PART, expect_scratch=True)


@pytest.mark.parametrize("part", [PART, 0])
def test_noalloc_without_scratch_on_two_calls_in_a_row(part):
    # contexts within one partition (or no split): the call uses no scratch at all
    from paged_kv_cache_319_b200 import _lib

    lib = _lib.lib()
    for case in [(8, 8, 16, [1, 16, 300, 512], "f16"), (32, 8, 16, [5, 129, 512], "bf16")]:
        for call in range(2):
            _run_both(lib, _lib, case, 77 + 1000 * call + case[0], part, expect_scratch=False)


def test_noalloc_rejects_a_batch_beyond_its_static_scratch():
    import torch
    from paged_kv_cache_319_b200 import _lib

    lib = _lib.lib()
    (q, k, v, t, l), _ = _inputs(7, 64, 64, 16, [16] * 64, "f16")
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    max_ctx = 65536  # 128 partitions x 64 seqs x 64 heads: far more than the static area
    need = lib.kvp_decode_workspace_bytes(64, 64, 128, max_ctx, PART)
    assert need > _lib.KVP_STATIC_SCRATCH_BYTES
    t_big = torch.full((64, max_ctx // 16), -1, dtype=torch.int32, device="cuda")
    t_big[:, :1] = t[:, :1]
    args = _common_args(q, k, t_big, l, 64, 64, 16, max_ctx)
    args[2] = v.data_ptr()
    out = torch.empty_like(q)
    rc = lib.paged_attention_decode_noalloc(*args, out.data_ptr(), _lib.KVP_F16, stream)
    assert rc == _lib.KVP_ERR_INVALID
    assert b"scratch" in lib.kvp_last_error_message()
