"""FP8 (E4M3) KV cache on the GPU against the oracle (oracle/fp8.py).

reshape_and_cache_fp8 is byte work: its codes must equal the oracle's bit for
bit, over scales that make the fp32 division round (0.37, 0.013, ...), ties
between two codes, saturation past 448, negative zero, padding slots, fp16 and
bf16 inputs. paged_attention_decode_fp8 is held to the decode tolerance against
fp64 attention over the dequantised cache, on caches of uniform codes (every
magnitude from 2^-9 to 448) and on caches the oracle quantised from N(0, 1)
data: block sizes 8, 16 and 32, split and unsplit partitions, contexts of 0, 1,
a block and one past it, grouped-query heads (G = 2 to 16, on the tensor
cores), NaN codes in the slots past the contexts, the full OPT-13B batch (64
sequences, 40 heads, contexts U[1, 2048]) and the long-context GQA batch (32
sequences, 32 / 8 heads, contexts U[16384, 32768]), both on every row.
copy_blocks copies E4M3 blocks byte for byte.
"""

import math

import numpy as np
import pytest

from oracle import cache as cache_oracle
from oracle import fp8
from oracle.numerics import to_f64
from parity import check_close, from_bits, random_e4m3_codes, to_bits
import workloads

pytestmark = pytest.mark.gpu


def _torch():
    import torch

    return torch


def _dev(x):
    return _torch().from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_reshape_and_cache_fp8_matches_oracle_bit_for_bit(dtype):
    import paged_kv_cache_319_b200 as kvp

    T, Hkv, D, bs, NB = 37, 5, 128, 16, 12
    kb = workloads.normal_bits([91, 1], (T, Hkv, D), dtype).copy()
    vb = workloads.normal_bits([91, 2], (T, Hkv, D), dtype).copy()
    k = to_f64(kb, dtype)
    # ties: every midpoint between two neighbouring positive codes, scale 1 (head 1)
    lo, hi = fp8.decode(np.arange(0, 0x7E, dtype=np.uint8)), fp8.decode(np.arange(1, 0x7F, dtype=np.uint8))
    mid = (lo + hi) / 2
    n = min(mid.size, D)
    k[0, 1, :n] = mid[:n]
    k[1, 1, :n] = -mid[:n]
    k[2] *= 1000.0     # saturation
    k[3, 0, :8] = -0.0
    torch = _torch()
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    kt = torch.from_numpy(k.astype(np.float32)).to(tdt)
    kb = kt.view(torch.int16).numpy().view(np.uint16)
    k_f = to_f64(kb, dtype)
    assert np.array_equal(k_f[0, 1, :n], mid[:n])  # the midpoints survive the 16-bit type
    v_f = to_f64(vb, dtype)
    k_scale = np.float32([0.37, 1.0, 2.0**-4, 0.013, 5.5])
    v_scale = np.float32([1.0, 0.05, 3.0, 0.2, 1e-3])
    slots = np.random.default_rng(5).permutation(NB * bs)[:T].astype(np.int64)
    slots[[4, 20]] = -1
    fill = np.full((NB, Hkv, bs, D), 0x55, np.uint8)
    kc, vc = _dev(fill.copy()), _dev(fill.copy())
    kvp.reshape_and_cache_fp8(from_bits(kb, dtype), from_bits(vb, dtype), kc, vc, _dev(slots),
                              _dev(k_scale), _dev(v_scale))
    kvp.check_device_error()
    ref_k, ref_v = fill.copy(), fill.copy()
    fp8.reshape_and_cache(ref_k, ref_v, k_f, v_f, slots, bs, k_scale, v_scale)
    assert np.array_equal(kc.cpu().numpy(), ref_k)
    assert np.array_equal(vc.cpu().numpy(), ref_v)


def _tables(seed, lens, bs, extra=5):
    rng = np.random.default_rng(seed)
    need = [-(-L // bs) for L in lens]
    NB = sum(need) + extra
    perm = rng.permutation(NB).astype(np.int32)
    t = np.full((len(lens), max(1, max(need))), -1, np.int32)
    i = 0
    for s, m in enumerate(need):
        t[s, :m] = perm[i:i + m]
        i += m
    return t, NB


def _run(q_bits, kc, vc, ks, vs, t, lens, dtype, scale, partition):
    import paged_kv_cache_319_b200 as kvp

    out = kvp.paged_attention_decode_fp8(
        from_bits(q_bits, dtype), _dev(kc), _dev(vc), _dev(ks), _dev(vs), _dev(t),
        _dev(np.asarray(lens, np.int32)), scale, max_context_len=int(max(max(lens), 1)),
        partition_size=partition)
    kvp.check_device_error()
    return to_bits(out)


CASES = [
    # (Hq, Hkv, bs, lens, dtype, partition, codes)
    (8, 8, 16, [1, 15, 16, 17, 300, 1100], "f16", 512, "uniform"),
    (8, 8, 8, [5, 64, 700], "bf16", 0, "uniform"),
    (8, 8, 32, [33, 1030, 2048], "f16", 256, "quantised"),
    (16, 4, 16, [0, 100, 900], "bf16", 512, "quantised"),   # G = 4, a context of 0
    (40, 40, 16, [2048, 1, 517], "f16", 512, "quantised"),  # OPT-13B heads
    # grouped-query heads run on the tensor cores (codes widened in shared memory)
    (16, 8, 16, [1, 2, 511, 512, 513, 3000], "f16", 512, "quantised"),  # G = 2
    (32, 8, 32, [0, 31, 32, 33, 1025, 4000], "bf16", 512, "uniform"),   # G = 4, bs 32
    (32, 4, 16, [7, 700, 2500], "f16", 0, "quantised"),                 # G = 8, unsplit
    (32, 2, 16, [200, 1300], "bf16", 256, "quantised"),                 # G = 16
    (32, 8, 16, [100, 900, 37], "f16", 512, "nan_tail"),                # NaN codes past the contexts
    (32, 8, 32, [5, 1000], "bf16", 0, "nan_tail"),
]


@pytest.mark.parametrize("Hq,Hkv,bs,lens,dtype,partition,codes", CASES)
def test_decode_fp8_matches_oracle(Hq, Hkv, bs, lens, dtype, partition, codes):
    D = 128
    seed = Hq * 100 + bs + len(lens)
    t, NB = _tables(seed, lens, bs)
    if codes == "uniform":
        kc = random_e4m3_codes([seed, 1], (NB, Hkv, bs, D))
        vc = random_e4m3_codes([seed, 2], (NB, Hkv, bs, D))
        ks = np.float32(np.linspace(1 / 448, 3 / 448, Hkv))
        vs = np.float32(np.linspace(0.5 / 448, 2 / 448, Hkv))
    elif codes == "nan_tail":
        # finite codes where the sequences have tokens; the NaN code (0x7F) in
        # the rest of each last block and in the spare blocks: p is 0 there, and
        # 0 times NaN must not reach the output
        kc = np.full((NB, Hkv, bs, D), 0x7F, np.uint8)
        vc = np.full((NB, Hkv, bs, D), 0x7F, np.uint8)
        kr = random_e4m3_codes([seed, 1], (NB, Hkv, bs, D))
        vr = random_e4m3_codes([seed, 2], (NB, Hkv, bs, D))
        for si, L in enumerate(lens):
            for j in range(L):
                b = t[si, j // bs]
                kc[b, :, j % bs] = kr[b, :, j % bs]
                vc[b, :, j % bs] = vr[b, :, j % bs]
        ks = np.float32(np.linspace(1 / 448, 3 / 448, Hkv))
        vs = np.float32(np.linspace(0.5 / 448, 2 / 448, Hkv))
    else:
        ks = np.float32(np.linspace(0.006, 0.011, Hkv))
        vs = np.float32(np.linspace(0.004, 0.009, Hkv))
        kf = to_f64(workloads.normal_bits([seed, 3], (NB, Hkv, bs, D), "f16"), "f16")
        vf = to_f64(workloads.normal_bits([seed, 4], (NB, Hkv, bs, D), "f16"), "f16")
        kc = fp8.quantize(kf, ks[None, :, None, None])
        vc = fp8.quantize(vf, vs[None, :, None, None])
    q = workloads.normal_bits([seed, 5], (len(lens), Hq, D), dtype)
    scale = 1 / math.sqrt(D)
    got = _run(q, kc, vc, ks, vs, t, lens, dtype, scale, partition)
    ref = fp8.paged_decode(to_f64(q, dtype), kc, vc, t, lens, scale, bs, ks, vs)
    check_close(got, ref, dtype, allow_ulp=(dtype == "bf16"))


def test_decode_fp8_opt13b_batch_every_row():
    """The bench's workload: 64 sequences, 40 heads x 128, contexts U[1, 2048],
    block size 16, partitions of 512; every row checked against the oracle."""
    wl = workloads.opt13b()
    lens = np.asarray(wl.info["context_lens"], np.int32)
    bs, Hkv, D = 16, 40, 128
    t, NB = _tables(77, lens.tolist(), bs, extra=64)
    kc = random_e4m3_codes([77, 1], (NB, Hkv, bs, D))
    vc = random_e4m3_codes([77, 2], (NB, Hkv, bs, D))
    ks = np.float32(np.linspace(1 / 448, 2 / 448, Hkv))
    vs = np.float32(np.linspace(1 / 448, 4 / 448, Hkv))
    q = workloads.normal_bits([77, 3], (len(lens), Hkv, D), "f16")
    got = _run(q, kc, vc, ks, vs, t, lens.tolist(), "f16", 1 / math.sqrt(D), 512)
    ref = fp8.paged_decode(to_f64(q, "f16"), kc, vc, t, lens, 1 / math.sqrt(D), bs, ks, vs)
    check_close(got, ref, "f16")


def test_decode_fp8_gqa_long_every_row():
    """Long-context GQA over an E4M3 cache: 32 sequences, 32 query / 8 KV heads
    x 128, block size 16, contexts U[16384, 32768], partitions of 512, bf16
    queries; every row checked against the oracle."""
    wl = workloads.gqa_long(16)
    lens = np.asarray(wl.info["context_lens"], np.int32)
    bs, Hq, Hkv, D = 16, 32, 8, 128
    t, NB = _tables(4004, lens.tolist(), bs, extra=16)
    kc = random_e4m3_codes([4004, 1], (NB, Hkv, bs, D))
    vc = random_e4m3_codes([4004, 2], (NB, Hkv, bs, D))
    ks = np.float32(np.linspace(1 / 448, 2 / 448, Hkv))
    vs = np.float32(np.linspace(1 / 448, 4 / 448, Hkv))
    q = workloads.normal_bits([4004, 3], (len(lens), Hq, D), "bf16")
    got = _run(q, kc, vc, ks, vs, t, lens.tolist(), "bf16", 1 / math.sqrt(D), 512)
    ref = fp8.paged_decode(to_f64(q, "bf16"), kc, vc, t, lens, 1 / math.sqrt(D), bs, ks, vs)
    check_close(got, ref, "bf16", allow_ulp=True)


def test_copy_blocks_fp8_byte_for_byte():
    import paged_kv_cache_319_b200 as kvp

    NB, Hkv, bs, D = 20, 4, 16, 128
    kc = random_e4m3_codes([3, 1], (NB, Hkv, bs, D))
    vc = random_e4m3_codes([3, 2], (NB, Hkv, bs, D))
    pairs = np.array([[0, 7], [3, 12], [19, 1]], np.int32)
    dk, dv = _dev(kc), _dev(vc)
    kvp.copy_blocks(dk, dv, _dev(pairs))
    kvp.check_device_error()
    cache_oracle.copy_blocks(kc, vc, pairs.tolist())
    assert np.array_equal(dk.cpu().numpy(), kc) and np.array_equal(dv.cpu().numpy(), vc)


def test_fp8_entry_points_reject_bad_arguments():
    import paged_kv_cache_319_b200 as kvp
    from paged_kv_cache_319_b200 import _lib

    torch = _torch()
    q = torch.zeros((2, 4, 64), dtype=torch.float16, device="cuda")
    kc = torch.zeros((4, 4, 16, 64), dtype=torch.uint8, device="cuda")
    s = torch.ones(4, dtype=torch.float32, device="cuda")
    t = torch.zeros((2, 1), dtype=torch.int32, device="cuda")
    lens = torch.ones(2, dtype=torch.int32, device="cuda")
    with pytest.raises(_lib.KvpError):  # head_dim 64
        kvp.paged_attention_decode_fp8(q, kc, kc, s, s, t, lens, 0.1)
    q = torch.zeros((2, 4, 128), dtype=torch.float16, device="cuda")
    kc = torch.zeros((4, 4, 16, 128), dtype=torch.uint8, device="cuda")
    rc = kvp.lib().paged_attention_decode_fp8(q.data_ptr(), kc.data_ptr(), kc.data_ptr(), None, None,
                                             t.data_ptr(), lens.data_ptr(), 2, 4, 4, 128, 16, 4, 1,
                                             16, 0.1, 0, None, 0, q.data_ptr(), 0, None)
    assert rc == _lib.KVP_ERR_INVALID  # NULL scales
    with pytest.raises(ValueError):  # scales of the wrong length
        kvp.paged_attention_decode_fp8(q, kc, kc, s[:2], s, t, lens, 0.1)
