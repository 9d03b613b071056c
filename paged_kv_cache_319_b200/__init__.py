"""Paged KV cache and decode attention for NVIDIA B200 (sm_100a).

Python binding of libkvp (C ABI in ``include/kvp.h``). This module only
marshals arguments: every step of the path - block bookkeeping, cache
writes, copy-on-write copies, attention - runs in the native library. There
is no Python or CPU fallback; calls fail loudly if ``libkvp.so`` is missing.

Host side: :class:`BlockPool` (fixed-size physical blocks, per-sequence block
tables, allocation on growth, fork with refcounted copy-on-write, release).
Device side (torch CUDA tensors, the current torch stream):
:func:`reshape_and_cache`, :func:`copy_blocks`, :func:`paged_attention_decode`.
"""

from __future__ import annotations

import ctypes as C

import numpy as np

from ._lib import (KVP_BF16, KVP_F16, KVP_FP8_E4M3, KvpError, P_i32, P_i64, PoolStats,
                   VCacheStats, check, lib)

__all__ = [
    "BlockPool", "KvpError", "reshape_and_cache", "copy_blocks", "paged_attention_decode",
    "paged_attention_prefill", "reshape_and_cache_fp8", "paged_attention_decode_fp8",
    "decode_workspace_bytes", "decode_grouped_workspace_bytes", "group_plan", "check_device_error",
    "VCache", "reshape_and_cache_vcache", "attention_decode_vcache", "pack_plan",
    "paged_attention_decode_packed",
    "kv_bytes_per_token", "version",
    "KVP_F16", "KVP_BF16", "KVP_FP8_E4M3",
]

_DTYPES = {"f16": KVP_F16, "bf16": KVP_BF16, "fp8_e4m3": KVP_FP8_E4M3}


def version() -> str:
    return lib().kvp_version().decode()


def kv_bytes_per_token(hidden: int, layers: int, elem_bytes: int) -> int:
    return int(lib().kvp_kv_bytes_per_token(hidden, layers, elem_bytes))


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(P_i32)


def _i64p(a: np.ndarray):
    return a.ctypes.data_as(P_i64)


class BlockPool:
    """Host-side block allocator of one KV pool (wraps ``kv_pool_*`` / ``kv_seq_*``)."""

    def __init__(self, num_blocks: int, block_size: int, num_kv_heads: int, head_dim: int,
                 dtype: str = "f16", free_order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        self._h = C.c_void_p()
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            if order.shape != (self.num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
        check(lib().kv_pool_create(num_blocks, block_size, num_kv_heads, head_dim, _DTYPES[dtype],
                                   _i32p(order) if order is not None else None, C.byref(self._h)))

    def close(self):
        if self._h:
            lib().kv_pool_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- sequences ----------------------------------------------------------
    def create(self) -> int:
        sid = C.c_int64()
        check(lib().kv_seq_create(self._h, C.byref(sid)))
        return sid.value

    def append(self, seq: int, n: int) -> list[int]:
        out = np.empty(max(int(n), 0), dtype=np.int64)
        check(lib().kv_seq_append(self._h, seq, int(n), _i64p(out) if n > 0 else None))
        return out.tolist()

    def append_batch(self, seqs, n_each: int = 1, out: np.ndarray | None = None) -> np.ndarray:
        s = np.ascontiguousarray(np.asarray(seqs, dtype=np.int64))
        if out is None:
            out = np.empty(len(s) * n_each, dtype=np.int64)
        check(lib().kv_seq_append_batch(self._h, _i64p(s), len(s), int(n_each), _i64p(out)))
        return out

    def append_tokens(self, seq: int, tokens) -> list[int]:
        """``append`` with the token ids given (registers filled blocks when prefix
        caching is on)."""
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).reshape(-1))
        out = np.empty(len(t), dtype=np.int64)
        check(lib().kv_seq_append_tokens(self._h, seq, _i32p(t) if len(t) else None, len(t),
                                         _i64p(out) if len(t) else None))
        return out.tolist()

    def append_tokens_batch(self, seqs, tokens, out: np.ndarray | None = None) -> np.ndarray:
        """``append_batch`` with token ids ``tokens [len(seqs), n_each]``."""
        s = np.ascontiguousarray(np.asarray(seqs, dtype=np.int64))
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).reshape(len(s), -1))
        n_each = t.shape[1] if len(s) else 0
        if out is None:
            out = np.empty(len(s) * n_each, dtype=np.int64)
        check(lib().kv_seq_append_tokens_batch(self._h, _i64p(s), len(s), int(n_each), _i32p(t),
                                               _i64p(out)))
        return out

    # ---- prefix caching ---------------------------------------------------------
    def set_prefix_caching(self, enable: bool = True) -> None:
        check(lib().kv_pool_set_prefix_caching(self._h, 1 if enable else 0))

    def create_prefixed(self, tokens) -> tuple[int, int]:
        """A sequence holding the longest cached prefix of ``tokens``: (id, cached tokens)."""
        t = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).reshape(-1))
        sid, cached = C.c_int64(), C.c_int32()
        check(lib().kv_seq_create_prefixed(self._h, _i32p(t) if len(t) else None, len(t),
                                           C.byref(sid), C.byref(cached)))
        return sid.value, cached.value

    def evictable(self) -> list[int]:
        out = np.empty(self.num_blocks, dtype=np.int32)
        n = C.c_int32()
        check(lib().kv_pool_evictable_list(self._h, _i32p(out), self.num_blocks, C.byref(n)))
        return out[:n.value].tolist()

    def prefix_stats(self) -> dict:
        r, e, h = C.c_int64(), C.c_int64(), C.c_int64()
        check(lib().kv_pool_prefix_stats(self._h, C.byref(r), C.byref(e), C.byref(h)))
        return {"registered": r.value, "evictable": e.value, "hit_tokens": h.value}

    def fork(self, parent: int) -> int:
        cid = C.c_int64()
        check(lib().kv_seq_fork(self._h, parent, C.byref(cid)))
        return cid.value

    def release(self, seq: int) -> None:
        check(lib().kv_seq_release(self._h, seq))

    def seq_len(self, seq: int) -> int:
        n = C.c_int32()
        check(lib().kv_seq_len(self._h, seq, C.byref(n)))
        return n.value

    def block_table(self, seq: int) -> list[int]:
        n = C.c_int32()
        rc = lib().kv_seq_block_table(self._h, seq, None, 0, C.byref(n))
        if rc not in (0, -6):
            check(rc)
        out = np.empty(n.value, dtype=np.int32)
        check(lib().kv_seq_block_table(self._h, seq, _i32p(out), n.value, C.byref(n)))
        return out.tolist()

    # ---- pool ---------------------------------------------------------------------
    def num_free(self) -> int:
        n = C.c_int32()
        check(lib().kv_pool_num_free(self._h, C.byref(n)))
        return n.value

    def free_list(self) -> list[int]:
        out = np.empty(self.num_blocks, dtype=np.int32)
        n = C.c_int32()
        check(lib().kv_pool_free_list(self._h, _i32p(out), self.num_blocks, C.byref(n)))
        return out[:n.value].tolist()

    def refcount(self, block: int) -> int:
        r = C.c_int32()
        check(lib().kv_pool_refcount(self._h, block, C.byref(r)))
        return r.value

    def refcounts(self) -> list[int]:
        out = np.empty(self.num_blocks, dtype=np.int32)
        check(lib().kv_pool_refcounts(self._h, _i32p(out), self.num_blocks))
        return out.tolist()

    def stats(self) -> dict:
        s = PoolStats()
        check(lib().kv_pool_stats(self._h, C.byref(s)))
        return {f: getattr(s, f) for f, _ in PoolStats._fields_}

    def _pairs(self, fn) -> list[tuple[int, int]]:
        n = C.c_int32()
        rc = fn(self._h, None, 0, C.byref(n))
        if rc not in (0, -6):
            check(rc)
        buf = np.empty(2 * max(n.value, 1), dtype=np.int32)
        check(fn(self._h, _i32p(buf), n.value, C.byref(n)))
        return [(int(buf[2 * i]), int(buf[2 * i + 1])) for i in range(n.value)]

    def take_copies(self) -> list[tuple[int, int]]:
        return self._pairs(lib().kv_pool_take_copies)

    def pending_copies(self) -> list[tuple[int, int]]:
        return self._pairs(lib().kv_pool_pending_copies)

    def build_batch(self, seqs, max_blocks: int, tables: np.ndarray | None = None,
                    lens: np.ndarray | None = None):
        """Block tables ``int32 [n, max_blocks]`` (padded with -1) and lengths ``int32 [n]``."""
        s = np.ascontiguousarray(np.asarray(seqs, dtype=np.int64))
        if tables is None:
            tables = np.empty((len(s), max_blocks), dtype=np.int32)
        if lens is None:
            lens = np.empty(len(s), dtype=np.int32)
        check(lib().kv_build_batch(self._h, _i64p(s), len(s), int(max_blocks), _i32p(tables),
                                   _i32p(lens)))
        return tables, lens


# ---- device operations (torch tensors on a CUDA device) -------------------------------
def _torch():
    import torch

    return torch


def _code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return KVP_F16
    if t.dtype == torch.bfloat16:
        return KVP_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _is_e4m3(t) -> bool:
    """An E4M3 cache: uint8 codes, or torch's float8_e4m3fn over the same bytes."""
    torch = _torch()
    return t.dtype == torch.uint8 or t.dtype == getattr(torch, "float8_e4m3fn", None)


def _cuda(*ts):
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda or t.device != dev:
            raise ValueError("all tensors must be on the same CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return dev


def _stream(dev) -> C.c_void_p:
    return C.c_void_p(_torch().cuda.current_stream(dev).cuda_stream)


def reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping) -> None:
    """Writes ``k_new/v_new [T, Hkv, D]`` into ``k_cache/v_cache [NB, Hkv, bs, D]`` at ``slot_mapping [T]``."""
    torch = _torch()
    dev = _cuda(k_new, v_new, k_cache, v_cache, slot_mapping)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    T, Hkv, D = k_new.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv, D) != (Hkv2, D2) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if not (k_new.dtype == v_new.dtype == k_cache.dtype == v_cache.dtype):
        raise TypeError("dtype mismatch")
    check(lib().reshape_and_cache(k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(),
                                  v_cache.data_ptr(), slot_mapping.data_ptr(), T, Hkv, D, bs, NB,
                                  _code(k_cache), _stream(dev)))


def copy_blocks(k_cache, v_cache, pairs) -> None:
    """Copy-on-write block copies; ``pairs`` is a CUDA ``int32 [n, 2]`` of (src, dst)."""
    torch = _torch()
    dev = _cuda(k_cache, v_cache, pairs)
    if pairs.dtype != torch.int32 or pairs.dim() != 2 or pairs.shape[1] != 2:
        raise TypeError("pairs must be int32 [n, 2]")
    NB = k_cache.shape[0]
    elems = k_cache[0].numel()
    code = KVP_FP8_E4M3 if _is_e4m3(k_cache) else _code(k_cache)
    if k_cache.dtype != v_cache.dtype:
        raise TypeError("dtype mismatch")
    check(lib().copy_blocks(k_cache.data_ptr(), v_cache.data_ptr(), pairs.data_ptr(),
                            pairs.shape[0], NB, elems, code, _stream(dev)))


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int, max_context_len: int,
                           partition_size: int) -> int:
    return int(lib().kvp_decode_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len,
                                                partition_size))


def decode_grouped_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int,
                                   max_context_len: int, partition_size: int) -> int:
    return int(lib().kvp_decode_grouped_workspace_bytes(num_seqs, num_q_heads, head_dim,
                                                        max_context_len, partition_size))


def group_plan(block_tables: np.ndarray, context_lens: np.ndarray, *, block_size: int,
               partition_size: int, num_q_heads: int, num_kv_heads: int, num_blocks: int,
               max_context_len: int | None = None) -> np.ndarray:
    """The grouping plan of ``paged_attention_decode_grouped``, built on the host
    (``kv_decode_group_plan``) from host block tables [S, MB] and lengths [S]."""
    t = np.ascontiguousarray(block_tables, dtype=np.int32)
    l = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, MB = t.shape
    mcl = MB * block_size if max_context_len is None else int(max_context_len)
    n = int(lib().kvp_decode_group_plan_words(S))
    plan = np.zeros(max(n, 1), np.int32)
    check(lib().kv_decode_group_plan(_i32p(t), _i32p(l), S, max(MB, 1), mcl, block_size,
                                     partition_size, num_q_heads, num_kv_heads, num_blocks,
                                     _i32p(plan), n))
    return plan


def pack_plan(block_tables: np.ndarray, context_lens: np.ndarray, *, block_size: int,
              num_q_heads: int, num_kv_heads: int, num_blocks: int,
              max_context_len: int | None = None) -> np.ndarray:
    """The packed plan of ``paged_attention_decode_packed`` (``kv_decode_pack_plan``),
    built on the host from host block tables [S, MB] and lengths [S]; trimmed to the
    words its header says it uses."""
    t = np.ascontiguousarray(block_tables, dtype=np.int32)
    l = np.ascontiguousarray(context_lens, dtype=np.int32)
    S, MB = t.shape
    mcl = MB * block_size if max_context_len is None else int(max_context_len)
    n = int(lib().kvp_decode_pack_plan_words(S, max(MB, 1)))
    plan = np.zeros(max(n, 1), np.int32)
    check(lib().kv_decode_pack_plan(_i32p(t), _i32p(l), S, max(MB, 1), mcl, block_size,
                                    num_q_heads, num_kv_heads, num_blocks, _i32p(plan), n))
    used = int(plan[7]) + 2 * int(plan[2])
    return plan[:used].copy()


def paged_attention_decode_packed(q, k_cache, v_cache, context_lens, scale: float, host_plan,
                                  out=None, *, max_context_len: int | None = None,
                                  device_plan=None, workspace=None):
    """Decode attention of forked sequences through the packed grouped decode (every
    shared block read once per group); ``host_plan`` from :func:`pack_plan`."""
    torch = _torch()
    dev = _cuda(q, k_cache, v_cache, context_lens)
    if context_lens.dtype != torch.int32:
        raise TypeError("context_lens must be int32")
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    plan = np.ascontiguousarray(host_plan, dtype=np.int32)
    mcl = int(context_lens.max().item()) if max_context_len is None else int(max_context_len)
    if out is None:
        out = torch.empty_like(q)
    need = int(lib().kvp_decode_packed_workspace_bytes(_i32p(plan), S, Hq, D))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _cuda(out, workspace)
    dp = None
    if device_plan is not None:
        _cuda(device_plan)
        dp = device_plan.data_ptr()
    check(lib().paged_attention_decode_packed(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), context_lens.data_ptr(), S, Hq, Hkv,
        D, bs, NB, mcl, float(scale), _i32p(plan), dp, workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), out.data_ptr(), _code(q), _stream(dev)))
    return out


def paged_attention_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                           out=None, *, max_context_len: int | None = None,
                           partition_size: int = 0, workspace=None, grouped: bool = False,
                           host_plan: np.ndarray | None = None, device_plan=None):
    """Decode attention over the paged cache; returns ``out [S, Hq, D]`` (dtype of q).

    ``max_context_len`` bounds every ``context_lens`` entry (default: the
    block-table capacity); ``partition_size > 0`` selects the split-context
    kernel pair. ``grouped`` calls ``paged_attention_decode_grouped``, which
    reads blocks shared by several sequences once per subgroup of them, with
    ``host_plan`` (from :func:`group_plan` on the same tables; ``device_plan``,
    an int32 CUDA tensor holding a copy of it, saves the call its upload) or a
    plan built on the GPU. A workspace is allocated with torch when needed and
    none is given.
    """
    torch = _torch()
    dev = _cuda(q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape or q.dtype != k_cache.dtype:
        raise ValueError("q / cache mismatch")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("batch metadata mismatch")
    mcl = MB * bs if max_context_len is None else int(max_context_len)
    if out is None:
        out = torch.empty_like(q)
    else:
        _cuda(out)
        if out.shape != q.shape or out.dtype != q.dtype:
            raise ValueError("out mismatch")
    size_fn = decode_grouped_workspace_bytes if grouped else decode_workspace_bytes
    need = size_fn(S, Hq, D, mcl, partition_size)
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        _cuda(workspace)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    args = [q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
            context_lens.data_ptr(), S, Hq, Hkv, D, bs, NB, max(MB, 1), mcl, float(scale),
            int(partition_size), ws_ptr, ws_bytes, out.data_ptr(), _code(q), _stream(dev)]
    if grouped:
        if host_plan is not None:
            host_plan = np.ascontiguousarray(host_plan, dtype=np.int32)
        dp = None
        if device_plan is not None:
            _cuda(device_plan)
            if device_plan.dtype != torch.int32:
                raise TypeError("device_plan must be int32")
            dp = device_plan.data_ptr()
        args[15:15] = [host_plan.ctypes.data if host_plan is not None else None, dp]
        check(lib().paged_attention_decode_grouped(*args))
    else:
        check(lib().paged_attention_decode(*args))
    return out


def paged_attention_prefill(q, k_cache, v_cache, block_tables, context_lens, scale: float,
                            out=None, *, max_context_len: int | None = None,
                            partition_size: int = 0, workspace=None):
    """Attention of a chunk of T new tokens per sequence, causal within the chunk;
    ``q [S, T, Hq, D]`` (dtype of the cache), returns ``out`` of the same shape.
    ``context_lens[s]`` counts the chunk, whose K/V must already be in the cache."""
    torch = _torch()
    dev = _cuda(q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    S, T, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape or q.dtype != k_cache.dtype:
        raise ValueError("q / cache mismatch")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("batch metadata mismatch")
    mcl = MB * bs if max_context_len is None else int(max_context_len)
    if out is None:
        out = torch.empty_like(q)
    else:
        _cuda(out)
        if out.shape != q.shape or out.dtype != q.dtype:
            raise ValueError("out mismatch")
    need = int(lib().kvp_prefill_workspace_bytes(S, T, Hq, D, mcl, partition_size))
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        _cuda(workspace)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    check(lib().paged_attention_prefill(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                        block_tables.data_ptr(), context_lens.data_ptr(), S, T,
                                        Hq, Hkv, D, bs, NB, max(MB, 1), mcl, float(scale),
                                        int(partition_size), ws_ptr, ws_bytes, out.data_ptr(),
                                        _code(q), _stream(dev)))
    return out


def _fp8_scales(k_scale, v_scale, Hkv, dev):
    torch = _torch()
    for t in (k_scale, v_scale):
        _cuda(t)
        if t.device != dev or t.dtype != torch.float32 or t.shape != (Hkv,):
            raise ValueError("k_scale / v_scale must be CUDA float32 [num_kv_heads] on the cache's device")


def reshape_and_cache_fp8(k_new, v_new, k_cache, v_cache, slot_mapping, k_scale, v_scale) -> None:
    """Quantises ``k_new/v_new [T, Hkv, D]`` (fp16 / bf16) into the E4M3 caches
    ``k_cache/v_cache [NB, Hkv, bs, D]`` (uint8 or float8_e4m3fn) at
    ``slot_mapping [T]``: KV head h is divided by ``k_scale[h]`` (values:
    ``v_scale[h]``, CUDA float32 ``[Hkv]``) and rounded to E4M3."""
    torch = _torch()
    dev = _cuda(k_new, v_new, k_cache, v_cache, slot_mapping)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    T, Hkv, D = k_new.shape
    NB, Hkv2, bs, D2 = k_cache.shape
    if (Hkv, D) != (Hkv2, D2) or v_new.shape != k_new.shape or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch")
    if k_new.dtype != v_new.dtype or not (_is_e4m3(k_cache) and _is_e4m3(v_cache)):
        raise TypeError("k_new/v_new must share a 16-bit dtype and the caches must be E4M3 (uint8)")
    _fp8_scales(k_scale, v_scale, Hkv, dev)
    check(lib().reshape_and_cache_fp8(k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(),
                                      v_cache.data_ptr(), slot_mapping.data_ptr(), k_scale.data_ptr(),
                                      v_scale.data_ptr(), T, Hkv, D, bs, NB, _code(k_new),
                                      _stream(dev)))


def paged_attention_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                               scale: float, out=None, *, max_context_len: int | None = None,
                               partition_size: int = 0, workspace=None):
    """Decode attention over E4M3 caches (uint8 or float8_e4m3fn ``[NB, Hkv, bs, D]``)
    with per-KV-head scales; q and ``out [S, Hq, D]`` are fp16 / bf16. The other
    arguments as for :func:`paged_attention_decode`."""
    torch = _torch()
    dev = _cuda(q, k_cache, v_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if D2 != D or v_cache.shape != k_cache.shape or not (_is_e4m3(k_cache) and _is_e4m3(v_cache)):
        raise ValueError("q / cache mismatch")
    _fp8_scales(k_scale, v_scale, Hkv, dev)
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    if block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("batch metadata mismatch")
    mcl = MB * bs if max_context_len is None else int(max_context_len)
    if out is None:
        out = torch.empty_like(q)
    else:
        _cuda(out)
        if out.shape != q.shape or out.dtype != q.dtype:
            raise ValueError("out mismatch")
    need = decode_workspace_bytes(S, Hq, D, mcl, partition_size)
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        _cuda(workspace)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    check(lib().paged_attention_decode_fp8(
        q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), k_scale.data_ptr(), v_scale.data_ptr(),
        block_tables.data_ptr(), context_lens.data_ptr(), S, Hq, Hkv, D, bs, NB, max(MB, 1), mcl,
        float(scale), int(partition_size), ws_ptr, ws_bytes, out.data_ptr(), _code(q), _stream(dev)))
    return out


class VCache:
    """A virtually contiguous KV cache (``kv_vcache_*``): per sequence slot one
    reserved virtual range of K and of V, token-major ``[slot][token][Hkv][D]``,
    backed by physical chunks mapped as the slot's capacity grows. Created on
    the current CUDA device."""

    def __init__(self, num_slots: int, max_tokens: int, num_kv_heads: int, head_dim: int,
                 dtype: str):
        h = C.c_void_p()
        check(lib().kv_vcache_create(num_slots, max_tokens, num_kv_heads, head_dim, _DTYPES[dtype],
                                     C.byref(h)))
        self._h = h
        self.num_slots, self.max_tokens = num_slots, max_tokens
        self.num_kv_heads, self.head_dim, self.dtype = num_kv_heads, head_dim, dtype
        kb, vb, st = C.c_void_p(), C.c_void_p(), C.c_int32()
        check(lib().kv_vcache_layout(h, C.byref(kb), C.byref(vb), C.byref(st)))
        self.k_base, self.v_base, self.slot_tokens = kb.value, vb.value, st.value

    @property
    def handle(self):
        if self._h is None:
            raise RuntimeError("cache destroyed")
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None:
            lib().kv_vcache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # pragma: no cover - interpreter shutdown
            pass

    def reserve(self, slot: int, tokens: int) -> None:
        """Capacity of ``slot`` >= ``tokens`` (maps chunks; the device copy is updated
        on the current stream)."""
        torch = _torch()
        check(lib().kv_vcache_reserve(self.handle, slot, tokens,
                                      _stream(torch.device("cuda", torch.cuda.current_device()))))

    def reserve_batch(self, slots: np.ndarray, tokens: np.ndarray) -> None:
        """reserve() for every (slot, tokens) pair in one call (all or nothing)."""
        torch = _torch()
        sl = np.ascontiguousarray(slots, dtype=np.int32)
        tk = np.ascontiguousarray(tokens, dtype=np.int32)
        if sl.shape != tk.shape:
            raise ValueError("one token count per slot")
        check(lib().kv_vcache_reserve_batch(self.handle, _i32p(sl), _i32p(tk), sl.size,
                                            _stream(torch.device("cuda", torch.cuda.current_device()))))

    def trim(self, slot: int, tokens: int) -> None:
        torch = _torch()
        check(lib().kv_vcache_trim(self.handle, slot, tokens,
                                   _stream(torch.device("cuda", torch.cuda.current_device()))))

    def release_spares(self) -> None:
        check(lib().kv_vcache_release_spares(self.handle))

    def capacity(self, slot: int) -> int:
        n = C.c_int32()
        check(lib().kv_vcache_capacity(self.handle, slot, C.byref(n)))
        return n.value

    def stats(self) -> dict:
        st = VCacheStats()
        check(lib().kv_vcache_stats(self.handle, C.byref(st)))
        return {name: getattr(st, name) for name, _ in VCacheStats._fields_}

    def view(self, which: str, slot: int, tokens: int):
        """A torch view ``[tokens, Hkv, D]`` of the first ``tokens`` tokens of a slot's
        K or V range; refused beyond the slot's capacity (unmapped memory)."""
        torch = _torch()
        if not 0 <= slot < self.num_slots or not 0 <= tokens <= self.capacity(slot):
            raise ValueError("view outside the slot's mapped capacity")
        base = self.k_base if which == "k" else self.v_base
        elem = 2
        row = self.num_kv_heads * self.head_dim
        ptr = base + slot * self.slot_tokens * row * elem

        class _Arr:
            __cuda_array_interface__ = {"shape": (tokens, self.num_kv_heads, self.head_dim),
                                        "typestr": "<f2", "data": (ptr, False), "version": 3,
                                        "strides": None}
        t = torch.as_tensor(_Arr(), device=torch.device("cuda", torch.cuda.current_device()))
        return t.view(torch.float16 if self.dtype == "f16" else torch.bfloat16)


def reshape_and_cache_vcache(k_new, v_new, vc: VCache, slots, positions) -> None:
    """Writes ``k_new/v_new [T, Hkv, D]`` to position ``positions[t]`` of slot ``slots[t]``
    (CUDA int32 [T]) of a virtually contiguous cache."""
    torch = _torch()
    dev = _cuda(k_new, v_new, slots, positions)
    if slots.dtype != torch.int32 or positions.dtype != torch.int32:
        raise TypeError("slots and positions must be int32")
    T = k_new.shape[0]
    if tuple(k_new.shape) != (T, vc.num_kv_heads, vc.head_dim) or v_new.shape != k_new.shape:
        raise ValueError("shape mismatch")
    if slots.numel() != T or positions.numel() != T:
        raise ValueError("one slot and one position per token")
    if _code(k_new) != _DTYPES[vc.dtype] or v_new.dtype != k_new.dtype:
        raise TypeError("dtype mismatch")
    check(lib().reshape_and_cache_vcache(k_new.data_ptr(), v_new.data_ptr(), vc.handle,
                                         slots.data_ptr(), positions.data_ptr(), T, _stream(dev)))


def attention_decode_vcache(q, vc: VCache, seq_slots, context_lens, scale: float, out=None, *,
                            max_context_len: int | None = None, partition_size: int = 0,
                            workspace=None):
    """Decode attention over a virtually contiguous cache: sequence s reads slot
    ``seq_slots[s]``; returns ``out [S, Hq, D]``."""
    torch = _torch()
    dev = _cuda(q, seq_slots, context_lens)
    if seq_slots.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("seq_slots and context_lens must be int32")
    S, Hq, D = q.shape
    if D != vc.head_dim or _code(q) != _DTYPES[vc.dtype]:
        raise ValueError("q does not match the cache")
    mcl = vc.max_tokens if max_context_len is None else int(max_context_len)
    if out is None:
        out = torch.empty_like(q)
    _cuda(out)
    ws_ptr, ws_bytes = None, 0
    need = decode_workspace_bytes(S, Hq, D, mcl, partition_size)
    if need:
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        _cuda(workspace)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    check(lib().attention_decode_vcache(q.data_ptr(), vc.handle, seq_slots.data_ptr(),
                                        context_lens.data_ptr(), S, Hq, mcl, float(scale),
                                        int(partition_size), ws_ptr, ws_bytes, out.data_ptr(),
                                        _stream(dev)))
    return out


def check_device_error(device=None) -> None:
    """Synchronises the current stream and raises if a kernel recorded an out-of-range index."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    check(lib().kvp_check_device_error(_stream(dev)))
