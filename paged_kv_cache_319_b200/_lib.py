"""ctypes loader and signatures of libkvp.so (the C ABI in include/kvp.h)."""

from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvp.so")

KVP_OK = 0
KVP_ERR_INVALID = -1
KVP_ERR_OOM = -2
KVP_ERR_NO_SEQ = -3
KVP_ERR_CUDA = -4
KVP_ERR_BOUNDS = -5
KVP_ERR_CAPACITY = -6
KVP_F16 = 0
KVP_BF16 = 1
KVP_FP8_E4M3 = 2
KVP_STATIC_SCRATCH_BYTES = 40 * 1024 * 1024  # include/kvp.h

ERROR_KINDS = {
    KVP_ERR_INVALID: "invalid",
    KVP_ERR_OOM: "oom",
    KVP_ERR_NO_SEQ: "no_seq",
    KVP_ERR_CUDA: "cuda",
    KVP_ERR_BOUNDS: "bounds",
    KVP_ERR_CAPACITY: "capacity",
}


class KvpError(RuntimeError):
    """A libkvp call returned a non-zero status."""

    def __init__(self, code: int, message: str):
        super().__init__(f"{ERROR_KINDS.get(code, code)}: {message}")
        self.code = code
        self.kind = ERROR_KINDS.get(code, str(code))


class PoolStats(C.Structure):
    _fields_ = [(n, C.c_int64) for n in ("num_blocks", "num_free", "num_used", "num_shared",
                                         "waste_slots", "cow_copies_total", "num_seqs")]


class VCacheStats(C.Structure):
    _fields_ = [(n, C.c_int64) for n in ("chunk_bytes", "mapped_chunks", "spare_chunks",
                                         "mapped_bytes", "reserved_bytes", "map_calls",
                                         "create_calls", "slot_tokens")]


i32, i64, u64, f32 = C.c_int32, C.c_int64, C.c_uint64, C.c_float
vp, sz = C.c_void_p, C.c_size_t
P_i32, P_i64 = C.POINTER(C.c_int32), C.POINTER(C.c_int64)

# name -> (restype, argtypes); must match include/kvp.h
SIGNATURES = {
    "kv_pool_create": (C.c_int, [i32, i32, i32, i32, i32, P_i32, C.POINTER(vp)]),
    "kv_pool_destroy": (C.c_int, [vp]),
    "kv_pool_num_free": (C.c_int, [vp, P_i32]),
    "kv_pool_free_list": (C.c_int, [vp, P_i32, i32, P_i32]),
    "kv_pool_refcount": (C.c_int, [vp, i32, P_i32]),
    "kv_pool_refcounts": (C.c_int, [vp, P_i32, i32]),
    "kv_pool_stats": (C.c_int, [vp, C.POINTER(PoolStats)]),
    "kv_seq_create": (C.c_int, [vp, P_i64]),
    "kv_seq_append": (C.c_int, [vp, i64, i32, P_i64]),
    "kv_seq_append_batch": (C.c_int, [vp, P_i64, i32, i32, P_i64]),
    "kv_seq_fork": (C.c_int, [vp, i64, P_i64]),
    "kv_seq_release": (C.c_int, [vp, i64]),
    "kv_seq_len": (C.c_int, [vp, i64, P_i32]),
    "kv_seq_block_table": (C.c_int, [vp, i64, P_i32, i32, P_i32]),
    "kv_pool_take_copies": (C.c_int, [vp, P_i32, i32, P_i32]),
    "kv_pool_pending_copies": (C.c_int, [vp, P_i32, i32, P_i32]),
    "kv_build_batch": (C.c_int, [vp, P_i64, i32, i32, P_i32, P_i32]),
    "kvp_kv_bytes_per_token": (C.c_int64, [i64, i64, i64]),
    "reshape_and_cache": (C.c_int, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp]),
    "copy_blocks": (C.c_int, [vp, vp, vp, i32, i32, i64, i32, vp]),
    "kvp_decode_workspace_bytes": (sz, [i32, i32, i32, i32, i32]),
    "paged_attention_decode": (C.c_int, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                         i32, f32, i32, vp, sz, vp, i32, vp]),
    "kvp_decode_grouped_workspace_bytes": (sz, [i32, i32, i32, i32, i32]),
    "paged_attention_decode_grouped": (C.c_int, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                 i32, i32, f32, i32, vp, vp, vp, sz, vp, i32, vp]),
    "kvp_decode_group_plan_words": (sz, [i32]),
    "kvp_prefill_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
    "paged_attention_prefill": (C.c_int, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                          i32, i32, f32, i32, vp, sz, vp, i32, vp]),
    "reshape_and_cache_fp8": (C.c_int, [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                        vp]),
    "paged_attention_decode_fp8": (C.c_int, [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                             i32, i32, i32, f32, i32, vp, sz, vp, i32, vp]),
    "kv_pool_set_prefix_caching": (C.c_int, [vp, i32]),
    "kv_seq_create_prefixed": (C.c_int, [vp, P_i32, i32, P_i64, P_i32]),
    "kv_seq_append_tokens": (C.c_int, [vp, i64, P_i32, i32, P_i64]),
    "kv_seq_append_tokens_batch": (C.c_int, [vp, P_i64, i32, i32, P_i32, P_i64]),
    "kv_pool_evictable_list": (C.c_int, [vp, P_i32, i32, P_i32]),
    "kv_pool_prefix_stats": (C.c_int, [vp, P_i64, P_i64, P_i64]),
    "kv_decode_group_plan": (C.c_int, [P_i32, P_i32, i32, i32, i32, i32, i32, i32, i32, i32, P_i32,
                                       sz]),
    "paged_attention_decode_noalloc": (C.c_int, [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                                 i32, i32, f32, i32, vp, i32, vp]),
    "kv_vcache_create": (C.c_int, [i32, i32, i32, i32, i32, C.POINTER(vp)]),
    "kv_vcache_destroy": (C.c_int, [vp]),
    "kv_vcache_reserve": (C.c_int, [vp, i32, i32, vp]),
    "kv_vcache_reserve_batch": (C.c_int, [vp, P_i32, P_i32, i32, vp]),
    "kv_vcache_trim": (C.c_int, [vp, i32, i32, vp]),
    "kv_vcache_release_spares": (C.c_int, [vp]),
    "kv_vcache_capacity": (C.c_int, [vp, i32, P_i32]),
    "kv_vcache_layout": (C.c_int, [vp, C.POINTER(vp), C.POINTER(vp), P_i32]),
    "kv_vcache_stats": (C.c_int, [vp, C.POINTER(VCacheStats)]),
    "reshape_and_cache_vcache": (C.c_int, [vp, vp, vp, vp, vp, i32, vp]),
    "attention_decode_vcache": (C.c_int, [vp, vp, vp, vp, i32, i32, i32, f32, i32, vp, sz, vp,
                                          vp]),
    "kvp_decode_pack_plan_words": (sz, [i32, i32]),
    "kv_decode_pack_plan": (C.c_int, [P_i32, P_i32, i32, i32, i32, i32, i32, i32, i32, P_i32, sz]),
    "kvp_decode_packed_workspace_bytes": (sz, [P_i32, i32, i32, i32]),
    "paged_attention_decode_packed": (C.c_int, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                                f32, P_i32, vp, vp, sz, vp, i32, vp]),
    "kvp_check_device_error": (C.c_int, [vp]),
    "kvp_selftest_bounded_wait": (C.c_int, [i32, vp]),
    "kvp_last_error_message": (C.c_char_p, []),
    "kvp_version": (C.c_char_p, []),
}

_lib = None


def lib():
    """The loaded library; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libkvp.so not found at {LIB_PATH}; build it with "
                "`python -m paged_kv_cache_319_b200.build`")
        h = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


def check(rc: int) -> None:
    if rc != KVP_OK:
        msg = lib().kvp_last_error_message()
        raise KvpError(rc, msg.decode() if msg else "")
