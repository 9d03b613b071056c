"""Argument checks of the newer entry points, on the host: each call below is refused
with KVP_ERR_INVALID before any CUDA call, so these run without a GPU. The pointers are
fake but aligned; none is dereferenced."""

import ctypes as C

import pytest

from paged_kv_cache_319_b200 import _lib

FAKE = C.c_void_p(1 << 20)  # 16-byte aligned, never dereferenced
F16, BF16, FP8 = _lib.KVP_F16, _lib.KVP_BF16, _lib.KVP_FP8_E4M3
INVALID = _lib.KVP_ERR_INVALID


@pytest.fixture(scope="module")
def lib():
    return _lib.lib()


def _decode_fp8(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, ks=FAKE, vs=FAKE, t=FAKE, l=FAKE, S=2, Hq=8, Hkv=8, D=128,
             bs=16, NB=4, MB=1, mcl=16, scale=0.1, part=0, ws=None, wsb=0, out=FAKE, dt=F16)
    a.update(kw)
    return lib.paged_attention_decode_fp8(a["q"], a["k"], a["v"], a["ks"], a["vs"], a["t"], a["l"],
                                          a["S"], a["Hq"], a["Hkv"], a["D"], a["bs"], a["NB"],
                                          a["MB"], a["mcl"], a["scale"], a["part"], a["ws"],
                                          a["wsb"], a["out"], a["dt"], None)


@pytest.mark.parametrize("bad", [dict(D=64), dict(ks=None), dict(vs=None), dict(dt=FP8),
                                 dict(Hq=6, Hkv=4), dict(bs=12), dict(scale=float("inf")),
                                 dict(mcl=17), dict(part=8 + 16)])
def test_decode_fp8_refuses(lib, bad):
    assert _decode_fp8(lib, **bad) == INVALID


def _scatter_fp8(lib, **kw):
    a = dict(kn=FAKE, vn=FAKE, kc=FAKE, vc=FAKE, sl=FAKE, ks=FAKE, vs=FAKE, T=4, Hkv=2, D=128,
             bs=16, NB=8, dt=BF16)
    a.update(kw)
    return lib.reshape_and_cache_fp8(a["kn"], a["vn"], a["kc"], a["vc"], a["sl"], a["ks"], a["vs"],
                                     a["T"], a["Hkv"], a["D"], a["bs"], a["NB"], a["dt"], None)


@pytest.mark.parametrize("bad", [dict(dt=FP8), dict(D=96), dict(bs=24), dict(ks=None),
                                 dict(T=-1), dict(kc=C.c_void_p((1 << 20) + 4))])
def test_reshape_and_cache_fp8_refuses(lib, bad):
    assert _scatter_fp8(lib, **bad) == INVALID


def test_reshape_and_cache_fp8_of_no_tokens_is_a_no_op(lib):
    assert _scatter_fp8(lib, T=0) == _lib.KVP_OK


def test_copy_blocks_block_bytes_follow_the_dtype(lib):
    # 24 E4M3 elements are 24 bytes: not a multiple of 16; as fp16 they are 48 bytes
    assert lib.copy_blocks(FAKE, FAKE, FAKE, 1, 4, 24, FP8, None) == INVALID
    assert lib.copy_blocks(FAKE, FAKE, FAKE, 0, 4, 24, F16, None) == _lib.KVP_OK


def _prefill(lib, **kw):
    a = dict(T=4, Hq=32, Hkv=8, D=128, bs=16, part=512)
    a.update(kw)
    return lib.paged_attention_prefill(FAKE, FAKE, FAKE, FAKE, FAKE, 2, a["T"], a["Hq"], a["Hkv"],
                                       a["D"], a["bs"], 64, 4, 64, 0.1, a["part"], FAKE, 1 << 30,
                                       FAKE, F16, None)


@pytest.mark.parametrize("bad", [dict(T=0), dict(D=64), dict(bs=8), dict(Hq=136, Hkv=4),
                                 dict(part=16 * 9)])
def test_prefill_refuses(lib, bad):
    assert _prefill(lib, **bad) == INVALID


def test_prefix_cache_calls_refuse_bad_arguments(lib):
    pool = C.c_void_p()
    assert lib.kv_pool_create(8, 4, 1, 64, FP8, None, C.byref(pool)) == _lib.KVP_OK
    try:
        sid, cached = C.c_int64(), C.c_int32()
        toks = (C.c_int32 * 3)(1, 2, 3)
        # off by default
        assert lib.kv_seq_create_prefixed(pool, toks, 3, C.byref(sid), C.byref(cached)) == INVALID
        assert lib.kv_pool_set_prefix_caching(pool, 1) == _lib.KVP_OK
        assert lib.kv_seq_create_prefixed(pool, None, 3, C.byref(sid), C.byref(cached)) == INVALID
        assert lib.kv_seq_create_prefixed(pool, toks, -1, C.byref(sid), C.byref(cached)) == INVALID
        assert lib.kv_seq_create_prefixed(pool, toks, 3, None, C.byref(cached)) == INVALID
        assert lib.kv_seq_create_prefixed(pool, toks, 3, C.byref(sid), C.byref(cached)) == _lib.KVP_OK
        assert cached.value == 0
        slots = (C.c_int64 * 3)()
        assert lib.kv_seq_append_tokens(pool, sid.value, None, 3, slots) == INVALID
        assert lib.kv_seq_append_tokens(pool, sid.value + 99, toks, 3, slots) == _lib.KVP_ERR_NO_SEQ
        assert lib.kv_seq_append_tokens(pool, sid.value, toks, 3, slots) == _lib.KVP_OK
        assert list(slots) == [0, 1, 2]
        n = C.c_int32()
        assert lib.kv_pool_evictable_list(pool, None, 0, C.byref(n)) == _lib.KVP_OK and n.value == 0
        r, e, h = C.c_int64(), C.c_int64(), C.c_int64()
        assert lib.kv_pool_prefix_stats(pool, None, C.byref(e), C.byref(h)) == INVALID
        assert lib.kv_pool_prefix_stats(pool, C.byref(r), C.byref(e), C.byref(h)) == _lib.KVP_OK
    finally:
        lib.kv_pool_destroy(pool)


@pytest.mark.parametrize("bad", [dict(n=0), dict(mt=0), dict(hkv=0), dict(d=64), dict(dt=FP8),
                                 dict(out=None)])
def test_vcache_create_refuses(lib, bad):
    a = dict(n=4, mt=1024, hkv=8, d=128, dt=F16, out=C.byref(C.c_void_p()))
    a.update(bad)
    assert lib.kv_vcache_create(a["n"], a["mt"], a["hkv"], a["d"], a["dt"], a["out"]) == INVALID


def test_vcache_calls_refuse_a_null_cache(lib):
    n = C.c_int32()
    assert lib.kv_vcache_reserve(None, 0, 1, None) == INVALID
    assert lib.kv_vcache_trim(None, 0, 0, None) == INVALID
    assert lib.kv_vcache_capacity(None, 0, C.byref(n)) == INVALID
    assert lib.kv_vcache_release_spares(None) == INVALID
    assert lib.kv_vcache_destroy(None) == _lib.KVP_OK
    assert lib.reshape_and_cache_vcache(FAKE, FAKE, None, FAKE, FAKE, 4, None) == INVALID
    assert lib.attention_decode_vcache(FAKE, None, FAKE, FAKE, 2, 8, 16, 0.1, 0, None, 0, FAKE,
                                       None) == INVALID
