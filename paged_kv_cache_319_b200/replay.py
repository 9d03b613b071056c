"""Runs a workload's operation schedule through libkvp on one GPU.

The host allocator (:class:`BlockPool`) turns create / append / fork /
release into block tables, slots and copy-on-write pairs; at each ``sync``
the pending copies run (``copy_blocks``) and then every token appended since
the previous sync is written to its slot (``reshape_and_cache``); at each
``attend`` the batch's block tables and lengths go to the device and
``paged_attention_decode`` (or, with ``grouped``, ``paged_attention_decode_grouped``) runs. Per-step order: copies, then scatter, then
attention, because a new token may land in a block copied in the same step.

Inputs (K/V of appended tokens, q of each attend) are drawn from
:mod:`workloads` keyed by the op's index, the same draws any other consumer
of the schedule sees. With ``device_values`` they are drawn on the GPU
instead (seeded by the op's index, normal, rounded to the cache type): the
same shapes and distribution without the host draws, for timing runs that do
not compare with the oracle.
"""

from __future__ import annotations

import numpy as np

from workloads.values import K_STREAM, Q_STREAM, V_STREAM, normal_bits, value_seed_words

import time

from . import (BlockPool, copy_blocks, group_plan, pack_plan, paged_attention_decode,
               paged_attention_decode_packed, reshape_and_cache)


def bits_to_tensor(bits: np.ndarray, dtype: str, device):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    t = t.view(torch.float16 if dtype == "f16" else torch.bfloat16)
    return t.to(device, non_blocking=False)


class DeviceReplay:
    def __init__(self, wl, device="cuda", keep_outputs: bool = True, time_decode: bool = False,
                 grouped: bool = False, time_reps: int = 1, plan_on: str = "host",
                 device_values: bool = False, packed: bool = False):
        import torch

        g = wl.geometry
        self.wl, self.g = wl, g
        self.device = torch.device(device)
        self.tdtype = torch.float16 if g.dtype == "f16" else torch.bfloat16
        self.pool = BlockPool(wl.num_blocks, g.block_size, g.num_kv_heads, g.head_dim, g.dtype,
                              wl.free_order)
        shape = (wl.num_blocks, g.num_kv_heads, g.block_size, g.head_dim)
        self.k_cache = torch.zeros(shape, dtype=self.tdtype, device=self.device)
        self.v_cache = torch.zeros(shape, dtype=self.tdtype, device=self.device)
        self.ids: dict[int, int] = {}
        self._pending = []
        self.events = []
        self.attends = []          # (op_index, seq ids, tables, lens)
        self.outputs = {}          # op_index -> out tensor
        self.keep_outputs = keep_outputs
        self.time_decode = time_decode
        self.grouped = grouped     # decode through paged_attention_decode_grouped
        self.plan_on = plan_on     # grouped: "host" (kv_decode_group_plan) or "device"
        self.plan_us = []          # host time of each grouping plan
        self.time_reps = max(1, int(time_reps))  # timed calls per attend op (time_decode)
        self.decode_events = []    # (op_index, start event, end event) around each decode call
        self.next_index = 0
        self.device_values = device_values
        self.packed = packed       # decode through paged_attention_decode_packed (host plan)

    def _device_normal(self, stream: int, op_index: int, shape):
        import torch

        gen = torch.Generator(device=self.device)
        gen.manual_seed((int(self.wl.value_seed) * 1000003 + stream) * 1000003 + int(op_index))
        return torch.randn(shape, generator=gen, device=self.device,
                           dtype=torch.float32).to(self.tdtype)

    def kv_values(self, op_index: int, n: int):
        g = self.g
        if self.device_values:
            shape = (n, g.num_kv_heads, g.head_dim)
            return (self._device_normal(K_STREAM, op_index, shape),
                    self._device_normal(V_STREAM, op_index, shape))
        shape = (n, g.num_kv_heads, g.head_dim)
        k = normal_bits(value_seed_words(self.wl.value_seed, K_STREAM, op_index), shape, g.dtype)
        v = normal_bits(value_seed_words(self.wl.value_seed, V_STREAM, op_index), shape, g.dtype)
        return k, v

    def q_values(self, op_index: int, num_seqs: int):
        g = self.g
        shape = (num_seqs, g.num_q_heads, g.head_dim)
        if self.device_values:
            return self._device_normal(Q_STREAM, op_index, shape)
        return normal_bits(value_seed_words(self.wl.value_seed, Q_STREAM, op_index), shape, g.dtype)

    def run(self, ops=None, start_index=None, attend_kwargs=None):
        ops = self.wl.ops if ops is None else ops
        i = self.next_index if start_index is None else start_index
        for op in ops:
            self._apply(i, op, attend_kwargs or {})
            i += 1
        self.next_index = i

    def _apply(self, i, op, kw):
        import torch

        kind = op[0]
        pool = self.pool
        if kind == "create":
            self.ids[op[1]] = pool.create()
            self.events.append((i, "create", self.ids[op[1]]))
        elif kind == "append":
            slots = pool.append(self.ids[op[1]], op[2])
            self._pending.append((slots, i, op[2]))
            self.events.append((i, "append", slots))
        elif kind == "fork":
            self.ids[op[2]] = pool.fork(self.ids[op[1]])
            self.events.append((i, "fork", self.ids[op[2]]))
        elif kind == "release":
            pool.release(self.ids[op[1]])
            self.events.append((i, "release", None))
        elif kind == "sync":
            copies = pool.take_copies()
            self.events.append((i, "sync", copies))
            if copies:
                pairs = torch.tensor(copies, dtype=torch.int32, device=self.device)
                copy_blocks(self.k_cache, self.v_cache, pairs)
            work = [(s, j, n) for s, j, n in self._pending if n]
            if work:
                ks, vs, sl = [], [], []
                for slots, j, n in work:
                    k, v = self.kv_values(j, n)
                    ks.append(k)
                    vs.append(v)
                    sl.extend(slots)
                if self.device_values:
                    k_new, v_new = torch.cat(ks), torch.cat(vs)
                else:
                    k_new = bits_to_tensor(np.concatenate(ks), self.g.dtype, self.device)
                    v_new = bits_to_tensor(np.concatenate(vs), self.g.dtype, self.device)
                slot_t = torch.tensor(sl, dtype=torch.int64, device=self.device)
                reshape_and_cache(k_new, v_new, self.k_cache, self.v_cache, slot_t)
            self._pending = []
        elif kind == "attend":
            seqs = [self.ids[h] for h in op[1]]
            lens_host = [pool.seq_len(s) for s in seqs]
            bs = self.g.block_size
            max_blocks = max(1, max(-(-L // bs) for L in lens_host))
            tables, lens = pool.build_batch(seqs, max_blocks)
            self.attends.append((i, seqs, tables, lens))
            q = self.q_values(i, len(seqs))
            if not self.device_values:
                q = bits_to_tensor(q, self.g.dtype, self.device)
            bt = torch.from_numpy(tables).to(self.device)
            cl = torch.from_numpy(lens).to(self.device)
            part = kw.get("partition_size", self.wl.partition_size)
            grouped = kw.get("grouped", self.grouped)
            mcl = int(lens.max()) if len(lens) else 0
            plan = dplan = None
            if grouped and self.plan_on == "host" and part > 0 and len(lens):
                t0 = time.perf_counter()
                plan = group_plan(tables, lens, block_size=bs, partition_size=part,
                                  num_q_heads=self.g.num_q_heads, num_kv_heads=self.g.num_kv_heads,
                                  num_blocks=self.wl.num_blocks, max_context_len=mcl)
                self.plan_us.append((time.perf_counter() - t0) * 1e6)
                # uploaded with the block tables, as an engine would
                dplan = torch.from_numpy(plan).to(self.device)
            call = lambda: paged_attention_decode(q, self.k_cache, self.v_cache, bt, cl,  # noqa: E731
                                                  self.wl.scale, max_context_len=mcl,
                                                  partition_size=part, grouped=grouped,
                                                  host_plan=plan, device_plan=dplan)
            if kw.get("packed", self.packed) and len(lens):
                t0 = time.perf_counter()
                pplan = pack_plan(tables, lens, block_size=bs, num_q_heads=self.g.num_q_heads,
                                  num_kv_heads=self.g.num_kv_heads, num_blocks=self.wl.num_blocks,
                                  max_context_len=max(mcl, 1))
                self.plan_us.append((time.perf_counter() - t0) * 1e6)
                dpp = torch.from_numpy(pplan).to(self.device)  # uploaded with the tables
                call = lambda: paged_attention_decode_packed(  # noqa: E731
                    q, self.k_cache, self.v_cache, cl, self.wl.scale, pplan,
                    max_context_len=max(mcl, 1), device_plan=dpp)
            if self.time_decode:
                # an untimed call, then before each timed call an L2 flush: a
                # 256 MB write, then a 256 MB read of another buffer, which writes
                # the dirty lines back before the timed region (a write alone would
                # leave L2 full of dirty lines that the timed call's reads evict,
                # adding up to L2's size of write-back to its traffic); the flush
                # also keeps the stream busy while the timed call is issued
                call()
                if not hasattr(self, "_l2_flush"):
                    self._l2_flush = torch.empty(256 << 20, dtype=torch.uint8, device=self.device)
                    self._l2_clean = torch.ones(256 << 20, dtype=torch.uint8, device=self.device)
                for _ in range(self.time_reps):
                    self._l2_flush.fill_(1)
                    self._l2_clean.amax()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    out = call()
                    e1.record()
                    self.decode_events.append((i, e0, e1))
            else:
                out = call()
            if self.keep_outputs:
                self.outputs[i] = out
        else:
            raise ValueError(f"unknown op {op!r}")
