#!/usr/bin/env python
"""Benchmark of the paged decode-attention hot path on B200.

One step = one decode step of the workload over one layer: host bookkeeping
(append one token to every sequence, pack block tables / lengths / slots),
host-to-device copy of that metadata, copy-on-write copies if any,
``reshape_and_cache`` of the new tokens, ``paged_attention_decode`` (with the
split-context reduce). Metric: KV GB/s = algorithmic bytes of the attention
call (K and V of every context token, q, out, block-table entries, lengths)
per second of step time, plus context tokens per second.

Default workload: OPT-13B geometry, one layer - 64 sequences, 40 heads x 128,
block size 16, context lengths U[1, 2048], pool 1.25x the need, fp16,
partitions of 512 tokens. Inputs are synthetic and resident in HBM before the
timed region; the KV pool (about 1.7 GB) exceeds L2, so no flush is needed.

Every step grows each sequence by one token. So that the timed lengths stay
those of the workload whatever the step count, the loop round-robins over R
identical copies of the one-layer workload (as a model's layers would), and
each copy starts short by half the steps it will take, so its lengths during
timing are centred on the configured ones.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload opt13b|gqa_long_bs16|gqa_long_bs32]
For N > 1 launch with torchrun; every rank runs an independent shard (its own
pool and batch: weak scaling, no data-path collective).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402
from workloads.values import K_STREAM, Q_STREAM, V_STREAM, normal_bits, value_seed_words  # noqa: E402

METRIC = "paged decode attention: KV GB/s (% of HBM peak) and seq-tokens/s per layer"
# Workloads whose batch changes every step; measured by replaying their schedule.
SCHEDULE_WORKLOADS = ("llama13b_churn", "sharing_A", "sharing_B", "beam")
# batches of forked sequences: decoded by default through the grouped entry point,
# which reads each shared block once per subgroup of the sequences holding it
GROUPED_WORKLOADS = ("sharing_A", "sharing_B", "beam")
UNIT = "GB/s"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peaks():
    """Dense bf16 (= fp16) tensor throughput, TFLOP/s: (sustained, burst, source)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1400.0, 1590.0, "fallback"


# DRAM traffic (read + write) of one launch of each decode kernel, as a multiple of
# its algorithmic bytes, from the ncu captures summarised in profiles/; valid only
# while the kernel source hashes to the value it had when captured.
PROFILED_TRAFFIC = {
    # profiles/decode_simt_opt13b.md: 1243.12 MB read + 4.00 MB written, 1233.81 MB algorithmic
    "decode_simt": {"ratio": (1243.12e6 + 4.00e6) / 1233812540.0, "sha": "1b93c4dcb021595d",
                    "files": ["common.cuh", "decode_simt.cuh"]},
    # profiles/decode_tc_gqa_long_bs16.md: 3102.54 MB read + 7.05 MB written, 3101.52 MB algorithmic
    "decode_tc": {"ratio": (3102.54e6 + 7.05e6) / 3101520896.0, "sha": "9263e4ab2818c45c",
                  "files": ["common.cuh", "decode_group.cuh", "decode_simt.cuh", "decode_tc.cuh"]},
    # profiles/decode_simt_fp8_opt13b.md: 621.85 MB read + 4.39 MB written, 617.57 MB algorithmic
    "decode_simt_fp8": {"ratio": (621.85e6 + 4.39e6) / 617569340.0, "sha": "1b93c4dcb021595d",
                        "files": ["common.cuh", "decode_simt.cuh"]},
    # profiles/decode_tc_fp8_gqa_long.md: 1551.56 MB read + 8.50 MB written, 1551.12 MB algorithmic
    "decode_tc_fp8": {"ratio": (1551.56e6 + 8.50e6) / 1551117312.0, "sha": "9263e4ab2818c45c",
                      "files": ["common.cuh", "decode_group.cuh", "decode_simt.cuh", "decode_tc.cuh"]},
}


def kernel_sha(files):
    import hashlib

    d = os.path.join(ROOT, "paged_kv_cache_319_b200", "csrc", "kernels")
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_per_launch(kernel, alg_bytes):
    p = PROFILED_TRAFFIC.get(kernel)
    if p is None or kernel_sha(p["files"]) != p["sha"]:
        return None
    return int(p["ratio"] * alg_bytes)


def algorithmic_bytes(lens, g):
    """Bytes one attention call must move: K and V of every context token, q, out,
    block-table entries and context lengths."""
    lens = np.asarray(lens, dtype=np.int64)
    e = g.elem_bytes
    kv = int(lens.sum()) * g.num_kv_heads * g.head_dim * e * 2
    qo = len(lens) * g.num_q_heads * g.head_dim * e * 2
    meta = 4 * int(np.sum(-(-lens // g.block_size))) + 4 * len(lens)
    return kv + qo + meta


# ---------------------------------------------------------------- clocks (NVML)
REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}


def _clock_worker(uuid, stop, out):
    """Child process: samples the SM clock and throttle reasons every ~1 ms."""
    try:
        import pynvml as nv

        nv.nvmlInit()
        h = nv.nvmlDeviceGetHandleByUUID(uuid.encode())
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        out.put(("max", nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)))
        out.put(("ready", None))
        buf = []
        while not stop.is_set():
            buf.append((time.time(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), reasons_fn(h)))
            time.sleep(0.001)
        out.put(("samples", buf))
    except Exception as e:  # pragma: no cover - depends on the box
        out.put(("error", repr(e)))
        out.put(("samples", []))


class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU from a separate process (no
    GIL contention) and keeps the samples taken inside the ``with`` block."""

    def __init__(self, torch_device):
        import multiprocessing as mp

        import torch

        self.uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
        ctx = mp.get_context("spawn")
        self._stop = ctx.Event()
        self._q = ctx.Queue()
        self._p = ctx.Process(target=_clock_worker, args=(self.uuid, self._stop, self._q),
                              daemon=True)
        self._p.start()
        self.max_mhz, self.error, self.window = None, None, (0.0, 0.0)
        while True:  # wait until the child samples
            kind, v = self._q.get(timeout=60)
            if kind == "max":
                self.max_mhz = v
            elif kind == "error":
                self.error = v
            if kind in ("ready", "samples"):
                break
        self.samples = []

    def __enter__(self):
        self._t0 = time.time()
        return self

    def __exit__(self, *a):
        self.window = (self._t0, time.time())
        self._stop.set()
        try:
            while True:
                kind, v = self._q.get(timeout=30)
                if kind == "samples":
                    self.samples = v
                    break
                if kind == "error":
                    self.error = v
        except Exception:
            pass
        self._p.join(timeout=10)

    def summary(self, min_samples: int = 3):
        """Median SM clock and the throttle reasons seen inside the timed window. A
        window shorter than a few NVML queries is widened 25 ms at a time on both
        sides (the warm-up just before it runs the same work) until it holds
        ``min_samples`` samples, at most 0.5 s; ``window_padded_ms`` says by how much."""
        t0, t1 = self.window
        pad = 0.0
        inside = [(c, r) for t, c, r in self.samples if t0 <= t <= t1]
        while len(inside) < min_samples and pad < 0.5:
            pad += 0.025
            inside = [(c, r) for t, c, r in self.samples if t0 - pad <= t <= t1 + pad]
        reasons = sorted({n for _, r in inside for n, b in REASON_BITS.items() if r & b})
        res = {"sm_mhz": float(statistics.median([c for c, _ in inside])) if inside else None,
               "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
               "window_ms": round((t1 - t0) * 1e3, 1)}
        if pad:
            res["window_padded_ms"] = round(pad * 1e3, 1)
        if self.error:
            res["error"] = self.error
        return res


# ---------------------------------------------------------------- distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def _reduce(x: float, world: int, op: str) -> float:
    """All-reduce of one timing number across ranks (CPU tensor under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def dist_max(x: float, world: int) -> float:
    return _reduce(x, world, "max")


def dist_sum(x: float, world: int) -> float:
    return _reduce(x, world, "sum")


def shard_value_seed(value_seed: int, rank: int) -> int:
    """Each rank's independent shard draws its own values; lengths and schedule are shared."""
    return value_seed + 7919 * rank


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def make_workload(args):
    kw = {} if getattr(args, "num_seqs", None) is None else {"num_seqs": args.num_seqs}
    return workloads.by_name(args.workload, **kw)


# ---------------------------------------------------------------- our arm
class Replica:
    """One copy of the one-layer workload: host pool, sequences, device KV pool."""

    def __init__(self, wl, start_lens, device, prefill_k, prefill_v):
        import torch
        import paged_kv_cache_319_b200 as kvp

        g = wl.geometry
        self.pool = kvp.BlockPool(wl.num_blocks, g.block_size, g.num_kv_heads, g.head_dim, g.dtype,
                                  wl.free_order)
        self.seqs = np.array([self.pool.create() for _ in start_lens], dtype=np.int64)
        slots = []
        for s, L in zip(self.seqs, start_lens):
            slots.extend(self.pool.append(int(s), int(L)))
        tdt = torch.float16 if g.dtype == "f16" else torch.bfloat16
        shape = (wl.num_blocks, g.num_kv_heads, g.block_size, g.head_dim)
        self.k = torch.zeros(shape, dtype=tdt, device=device)
        self.v = torch.zeros(shape, dtype=tdt, device=device)
        st = torch.tensor(slots, dtype=torch.int64, device=device)
        kvp.reshape_and_cache(prefill_k, prefill_v, self.k, self.v, st)
        self.lens = np.array(start_lens, dtype=np.int64)  # own copy per replica


class StepMeta:
    """One step's metadata in one pinned buffer (slots int64 [S], lengths int32 [S],
    block tables int32 [S, MB]) and its device mirror, so one H2D copy moves it all."""

    def __init__(self, S, MB, device):
        import torch

        nbytes = S * 8 + S * 4 + S * MB * 4
        self.host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
        self.dev = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.nbytes = nbytes

        def views(buf):
            slots = buf[: S * 8].view(torch.int64)
            lens = buf[S * 8: S * 12].view(torch.int32)
            tables = buf[S * 12:].view(torch.int32).view(S, MB)
            return slots, lens, tables

        self.slot_h, self.len_h, self.tab_h = views(self.host)
        self.slot_d, self.len_d, self.tab_d = views(self.dev)

    def upload(self):
        self.dev.copy_(self.host, non_blocking=True)


def to_dev(bits, dtype, device):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "f16" else torch.bfloat16).to(device)


def run_ours(args, world, rank, local):
    import torch
    import paged_kv_cache_319_b200 as kvp

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = make_workload(args)
    g = wl.geometry
    part = wl.partition_size if args.partition is None else args.partition
    ctx = np.asarray(wl.info["context_lens"], dtype=np.int64)
    S = len(ctx)
    W, K = args.warmup, args.steps

    # Replicas: none grows by more than ~64 tokens over warm-up, timing and the
    # end-to-end pass; each starts short by its warm-up steps plus half its
    # timed steps, so the timed lengths are centred on the configured ones.
    K_e2e = max(1, min(K, 64)) + max(1, min(K, 32))  # graph-replay pass + eager pass
    pool_bytes = 2 * wl.num_blocks * g.num_kv_heads * g.block_size * g.head_dim * g.elem_bytes
    free_b = torch.cuda.mem_get_info(device)[0]
    r_cap = max(1, int(0.6 * free_b // pool_bytes))
    R = max(1, min(r_cap, math.ceil((W + K + K_e2e) / 64)))
    shift = math.ceil(W / R) + math.ceil(K / R) // 2
    start = np.maximum(ctx - shift, 1)
    grow = math.ceil((W + K + K_e2e) / R) + 8  # + the e2e breakdown's few steps
    need_end = int(np.sum(-(-(start + grow) // g.block_size)))
    if need_end > wl.num_blocks:
        raise SystemExit(f"pool of {wl.num_blocks} blocks too small for {W + K} steps")

    seed_rank = shard_value_seed(wl.value_seed, rank)
    n_pre = int(start.sum())
    pk = to_dev(normal_bits(value_seed_words(seed_rank, K_STREAM, 0), (max(n_pre, 1), g.num_kv_heads, g.head_dim), g.dtype), g.dtype, device)
    pv = to_dev(normal_bits(value_seed_words(seed_rank, V_STREAM, 0), (max(n_pre, 1), g.num_kv_heads, g.head_dim), g.dtype), g.dtype, device)
    reps = [Replica(wl, start, device, pk[:n_pre], pv[:n_pre]) for _ in range(R)]
    del pk, pv

    # per-step inputs, resident in HBM (a cycle of NI sets)
    NI = min(W + K, 32)
    qs = [to_dev(normal_bits(value_seed_words(seed_rank, Q_STREAM, 1 + i), (S, g.num_q_heads, g.head_dim), g.dtype), g.dtype, device) for i in range(NI)]
    kn = [to_dev(normal_bits(value_seed_words(seed_rank, K_STREAM, 1 + i), (S, g.num_kv_heads, g.head_dim), g.dtype), g.dtype, device) for i in range(NI)]
    vn = [to_dev(normal_bits(value_seed_words(seed_rank, V_STREAM, 1 + i), (S, g.num_kv_heads, g.head_dim), g.dtype), g.dtype, device) for i in range(NI)]

    max_ctx_total = int(start.max()) + grow
    MB = -(-max_ctx_total // g.block_size)
    NBUF = 3
    meta = [StepMeta(S, MB, device) for _ in range(NBUF)]
    done = [None] * NBUF
    out = torch.empty((S, g.num_q_heads, g.head_dim), dtype=qs[0].dtype, device=device)
    ws_bytes = kvp.decode_workspace_bytes(S, g.num_q_heads, g.head_dim, max_ctx_total, part)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    step_bytes, step_tokens, launches, host_us = [], [], [], []
    ev_pairs = []

    def step(i, timed):
        rep = reps[i % R]
        b = i % NBUF
        if done[b] is not None:
            done[b].synchronize()
        m = meta[b]
        th = time.perf_counter()
        rep.pool.append_batch(rep.seqs, 1, out=m.slot_h.numpy())
        copies = rep.pool.take_copies()
        rep.pool.build_batch(rep.seqs, MB, m.tab_h.numpy(), m.len_h.numpy())
        if timed:
            host_us.append((time.perf_counter() - th) * 1e6)
        rep.lens += 1
        m.upload()
        n_launch = 0
        if copies:
            pairs = torch.tensor(copies, dtype=torch.int32).to(device, non_blocking=True)
            kvp.copy_blocks(rep.k, rep.v, pairs)
            n_launch += 1
        j = i % NI
        kvp.reshape_and_cache(kn[j], vn[j], rep.k, rep.v, m.slot_d)
        n_launch += 1
        if timed:
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        kvp.paged_attention_decode(qs[j], rep.k, rep.v, m.tab_d, m.len_d, wl.scale, out,
                                   max_context_len=max_ctx_total, partition_size=part,
                                   workspace=ws)
        n_launch += 2 if (part and int(rep.lens.max()) > part) else 1
        if timed:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(stream)
            ev_pairs.append((e0, e1))
            packed = m.len_h.numpy()  # the lengths this step's kernels read
            assert np.array_equal(packed, rep.lens)
            step_bytes.append(algorithmic_bytes(packed, g))
            step_tokens.append(int(packed.sum()))
            launches.append(n_launch)
        ev = torch.cuda.Event()
        ev.record(stream)
        done[b] = ev

    clk = ClockSampler(device)  # started before warm-up so the GPU is not idle before timing
    for i in range(W):
        step(i, False)
    torch.cuda.synchronize(device)
    kvp.check_device_error(device)
    barrier(world)
    torch.cuda.synchronize(device)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with clk:
        t0.record(stream)
        for i in range(W, W + K):
            step(i, True)
        t1.record(stream)
        torch.cuda.synchronize(device)
    kvp.check_device_error(device)
    barrier(world)
    elapsed_ms = t0.elapsed_time(t1)
    max_ms = dist_max(elapsed_ms, world)
    total_bytes = dist_sum(float(sum(step_bytes)), world)
    total_tokens = dist_sum(float(sum(step_tokens)), world)
    kernel_name = "decode_tc" if g.num_q_heads > g.num_kv_heads else "decode_simt"
    dec_ms = [a.elapsed_time(b) for a, b in ev_pairs]
    dec_avg_ms = sum(dec_ms) / len(dec_ms)
    dec_bytes_avg = sum(step_bytes) / len(step_bytes)
    achieved = dec_bytes_avg / (dec_avg_ms * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers
    rows = measure_rows(wl, reps[0], device, kn[0], vn[0], host_us)
    e2e = run_e2e(args, wl, reps, device, seed_rank, MB, max_ctx_total, part, ws, world)

    peak, peak_kind = peaks()
    value = total_bytes / (max_ms * 1e-3) / 1e9
    res = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(max_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": g.dtype,
        "data": "synthetic (seeded N(0,1) q/K/V; lengths and placement as configured)",
        "config": {
            "workload": wl.description,
            "name": wl.name,
            "num_seqs_per_gpu": S,
            "num_q_heads": g.num_q_heads,
            "num_kv_heads": g.num_kv_heads,
            "head_dim": g.head_dim,
            "block_size": g.block_size,
            "partition_size": part,
            "mean_context_len_timed": round(float(np.mean(step_tokens)) / S, 1),
            "replicas": R,
            "l2": "inputs larger than L2 (KV pool %.2f GB per replica)" % (pool_bytes / 1e9),
            "parallelism": f"replicas x{world} (independent shards, no collective)",
        },
        "seq_tokens_per_s": round(total_tokens / (max_ms * 1e-3), 1),
        "decode_tokens_per_s": round(world * S * K / (max_ms * 1e-3), 1),
        "hbm_frac_of_step": round(value / peak, 4),
        "gpu_launches": int(sum(launches)),
        "roofline": {
            "kernel": f"paged_attention_decode: {kernel_name} + decode_reduce_kernel",
            "bound": "hbm",
            "achieved": round(achieved, 1),
            "peak": peak,
            "peak_source": peak_kind,
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
            "traffic": traffic_per_launch(kernel_name, dec_bytes_avg),
            "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch "
                              "(profiles/), scaled by algorithmic bytes; null if the kernel changed",
            "avg_launch_us": round(dec_avg_ms * 1e3, 2),
            "algorithmic_bytes_per_launch": int(dec_bytes_avg),
            # the first timed launch: the one a profiler skipping the warm-up launches sees
            "algorithmic_bytes_first_timed": int(step_bytes[0]),
        },
        "e2e": e2e,
        "rows": rows,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_seconds)
    if rank == 0 and world == 1 and not args.headline_only:
        del reps, qs, kn, vn, ws, out
        release_memory()
        # the same decode call over a window long enough for the clock sampler, and
        # one record per other workload, each measured as its own --workload run is
        res["decode_window"] = decode_record(wl.name, device, calls=DECODE_WINDOW_CALLS)
        release_memory()
        res["workloads"] = workload_records(args, device)
    if rank == 0:
        print(json.dumps(res), flush=True)


def release_memory():
    import gc

    import torch

    gc.collect()
    torch.cuda.empty_cache()


def l2_flusher(device):
    """Before each timed call: a 256 MB write, then a 256 MB read of another buffer,
    which writes the dirty lines back before the timed region."""
    import torch

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    clean = torch.ones(256 << 20, dtype=torch.uint8, device=device)

    def run():
        flush.fill_(1)
        clean.amax()
    return run


DECODE_WINDOW_CALLS = 400


def decode_record(name, device, calls=DECODE_WINDOW_CALLS):
    """paged_attention_decode alone on one workload's batch (its configured lengths
    and placement; keys, values and q drawn on the device), `calls` calls each after
    an L2 flush, timed with CUDA events: a window of tens to hundreds of
    milliseconds, so the clock sampler sees it under load."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    wl = workloads.by_name(name)
    g = wl.geometry
    lens = np.asarray(wl.info["context_lens"], np.int64)
    S, bs = len(lens), g.block_size
    pool = kvp.BlockPool(wl.num_blocks, bs, g.num_kv_heads, g.head_dim, g.dtype, wl.free_order)
    seqs = np.array([pool.create() for _ in lens], dtype=np.int64)
    slots = np.concatenate([np.asarray(pool.append(int(s), int(L)), np.int64)
                            for s, L in zip(seqs, lens)])
    tdt = torch.float16 if g.dtype == "f16" else torch.bfloat16
    shape = (wl.num_blocks, g.num_kv_heads, bs, g.head_dim)
    k = torch.zeros(shape, dtype=tdt, device=device)
    v = torch.zeros(shape, dtype=tdt, device=device)
    gen = torch.Generator(device=device).manual_seed(5001)
    st = torch.from_numpy(slots).to(device)
    for t0 in range(0, len(slots), 65536):  # fill in chunks (fp32 draws, then rounded)
        n = min(65536, len(slots) - t0)
        kn = torch.randn((n, g.num_kv_heads, g.head_dim), generator=gen, device=device).to(tdt)
        vn = torch.randn((n, g.num_kv_heads, g.head_dim), generator=gen, device=device).to(tdt)
        kvp.reshape_and_cache(kn, vn, k, v, st[t0:t0 + n])
    MB = int(-(-lens.max() // bs))
    tables, cl = pool.build_batch(list(seqs), MB)
    tt = torch.from_numpy(tables).to(device)
    ct = torch.from_numpy(cl).to(device)
    q = torch.randn((S, g.num_q_heads, g.head_dim), generator=gen, device=device).to(tdt)
    out = torch.empty_like(q)
    part = wl.partition_size
    mcl = int(lens.max())
    ws = torch.empty(max(256, kvp.decode_workspace_bytes(S, g.num_q_heads, g.head_dim, mcl, part)),
                     dtype=torch.uint8, device=device)
    call = lambda: kvp.paged_attention_decode(q, k, v, tt, ct, wl.scale, out,  # noqa: E731
                                              max_context_len=mcl, partition_size=part,
                                              workspace=ws)
    flush = l2_flusher(device)
    for _ in range(5):
        call()
    kvp.check_device_error(device)
    stream = torch.cuda.current_stream(device)
    pairs = []
    with ClockSampler(device) as clk:
        for _ in range(calls):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            pairs.append((e0, e1))
        torch.cuda.synchronize(device)
    kvp.check_device_error(device)
    ms = np.array([a.elapsed_time(b) for a, b in pairs])
    alg = algorithmic_bytes(cl, g)
    peak, peak_kind = peaks()
    achieved = alg / (float(np.median(ms)) * 1e-3) / 1e9
    kernel = "decode_tc" if g.num_q_heads > g.num_kv_heads else "decode_simt"
    pool.close()
    return {"name": wl.name, "workload": wl.description, "calls": calls,
            "timed": f"paged_attention_decode alone, {calls} calls, L2 flushed before each",
            "call_us_median": round(float(np.median(ms)) * 1e3, 2),
            "call_us_mean": round(float(ms.mean()) * 1e3, 2),
            "seq_tokens_per_s": round(float(lens.sum()) / (float(np.median(ms)) * 1e-3), 1),
            "roofline": {"kernel": f"paged_attention_decode: {kernel} + decode_reduce_kernel",
                         "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "peak_source": peak_kind, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
                         "algorithmic_bytes_per_launch": int(alg),
                         "traffic": traffic_per_launch(kernel, alg)},
            "clocks": clk.summary(min_samples=20)}


def vcache_record(name, device, calls=200, grow_steps=256):
    """A/B of the block table's translation cost: the same batch (a workload's
    lengths; keys, values and q drawn once on the device and written to both
    caches) decoded from the paged pool and from the virtually contiguous cache
    (CUDA virtual memory management), each `calls` calls after an L2 flush, at
    equal algorithmic bytes. Host side: the growth of every sequence by one
    token per step over `grow_steps` steps, kv_seq_append_batch + kv_build_batch
    (paged) against kv_vcache_reserve_batch (contiguous: no table), and the cost
    of mapping a physical chunk."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    wl = workloads.by_name(name)
    g = wl.geometry
    lens = np.asarray(wl.info["context_lens"], np.int64)
    S, bs, Hkv, D = len(lens), g.block_size, g.num_kv_heads, g.head_dim
    tdt = torch.float16 if g.dtype == "f16" else torch.bfloat16
    max_tokens = int(lens.max()) + grow_steps + 16
    # paged pool, sized for the growth steps too
    nb = int(np.sum(-(-(lens + grow_steps) // bs))) + 16
    free_order = np.random.default_rng(wl.value_seed).permutation(nb).astype(np.int32)
    pool = kvp.BlockPool(nb, bs, Hkv, D, g.dtype, free_order)
    seqs = np.array([pool.create() for _ in lens], dtype=np.int64)
    slots = np.concatenate([np.asarray(pool.append(int(s), int(L)), np.int64)
                            for s, L in zip(seqs, lens)])
    k = torch.zeros((nb, Hkv, bs, D), dtype=tdt, device=device)
    v = torch.zeros_like(k)
    vc = kvp.VCache(S, max_tokens, Hkv, D, g.dtype)
    stream = torch.cuda.current_stream(device)
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    vc.reserve_batch(np.arange(S), lens)
    torch.cuda.synchronize(device)
    map_s = time.perf_counter() - t0
    st_map = vc.stats()
    vslot = torch.from_numpy(np.repeat(np.arange(S), lens).astype(np.int32)).to(device)
    vpos = torch.from_numpy(np.concatenate([np.arange(L) for L in lens]).astype(np.int32)).to(device)
    st = torch.from_numpy(slots).to(device)
    gen = torch.Generator(device=device).manual_seed(5101)
    for t0_ in range(0, len(slots), 65536):
        n = min(65536, len(slots) - t0_)
        kn = torch.randn((n, Hkv, D), generator=gen, device=device).to(tdt)
        vn = torch.randn((n, Hkv, D), generator=gen, device=device).to(tdt)
        kvp.reshape_and_cache(kn, vn, k, v, st[t0_:t0_ + n])
        kvp.reshape_and_cache_vcache(kn, vn, vc, vslot[t0_:t0_ + n], vpos[t0_:t0_ + n])
    MB = int(-(-lens.max() // bs))
    tables, cl = pool.build_batch(list(seqs), MB)
    tt = torch.from_numpy(tables).to(device)
    ct = torch.from_numpy(cl).to(device)
    sl = torch.arange(S, dtype=torch.int32, device=device)
    q = torch.randn((S, g.num_q_heads, D), generator=gen, device=device).to(tdt)
    out_p, out_c = torch.empty_like(q), torch.empty_like(q)
    part = wl.partition_size
    mcl = int(lens.max())
    ws = torch.empty(max(256, kvp.decode_workspace_bytes(S, g.num_q_heads, D, mcl, part)),
                     dtype=torch.uint8, device=device)
    paged = lambda: kvp.paged_attention_decode(q, k, v, tt, ct, wl.scale, out_p,  # noqa: E731
                                               max_context_len=mcl, partition_size=part,
                                               workspace=ws)
    contig = lambda: kvp.attention_decode_vcache(q, vc, sl, ct, wl.scale, out_c,  # noqa: E731
                                                 max_context_len=mcl, partition_size=part,
                                                 workspace=ws)
    flush = l2_flusher(device)

    def timed(fn):
        for _ in range(5):
            fn()
        pairs = []
        for _ in range(calls):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            pairs.append((e0, e1))
        torch.cuda.synchronize(device)
        return float(np.median([a.elapsed_time(b) for a, b in pairs]))

    with ClockSampler(device) as clk:
        ms_p = timed(paged)
        ms_c = timed(contig)
    kvp.check_device_error(device)
    same_bits = bool(torch.equal(out_p.view(torch.int16), out_c.view(torch.int16)))
    err = float((out_p.float() - out_c.float()).abs().max())
    alg = algorithmic_bytes(cl, g)
    # the contiguous call reads a slot index per sequence instead of table entries
    alg_c = alg - 4 * int(np.sum(-(-lens // bs))) + 4 * S
    peak, peak_kind = peaks()
    # host: one token per sequence per step
    cur = lens.copy()
    slot_buf = np.empty(S, np.int64)
    tab_buf = np.empty((S, MB + grow_steps // bs + 2), np.int32)
    len_buf = np.empty(S, np.int32)
    t_paged, t_vc = [], []
    maps_before = vc.stats()["map_calls"]
    all_slots = np.arange(S, dtype=np.int32)
    for _ in range(grow_steps):
        t0 = time.perf_counter()
        pool.append_batch(seqs, 1, out=slot_buf)
        pool.build_batch(seqs, tab_buf.shape[1], tab_buf, len_buf)
        t_paged.append(time.perf_counter() - t0)
        cur += 1
        t0 = time.perf_counter()
        vc.reserve_batch(all_slots, cur)
        t_vc.append(time.perf_counter() - t0)
    torch.cuda.synchronize(device)
    st_end = vc.stats()
    grow_maps = st_end["map_calls"] - maps_before
    paged_bytes = 2 * int(np.sum(-(-lens // bs))) * Hkv * bs * D * g.elem_bytes
    res = {
        "name": f"vcache_{name}", "workload": wl.description,
        "timed": f"paged_attention_decode and attention_decode_vcache on the same batch and data, "
                 f"{calls} calls each, L2 flushed before each",
        "paged_call_us": round(ms_p * 1e3, 2), "contiguous_call_us": round(ms_c * 1e3, 2),
        "translation_cost": round(ms_p / ms_c, 4),
        "outputs_bit_identical": same_bits, "outputs_max_abs_diff": err,
        "roofline": {"kernel": "attention_decode_vcache: " + (
            "decode_tc (contiguous, 128-token boxes)" if g.num_q_heads > Hkv else
            "decode_simt (contiguous, 16-token boxes)") + " + decode_reduce_kernel",
            "bound": "hbm", "achieved": round(alg_c / (ms_c * 1e-3) / 1e9, 1),
            "achieved_paged": round(alg / (ms_p * 1e-3) / 1e9, 1), "peak": peak,
            "peak_source": peak_kind, "unit": "GB/s",
            "frac": round(alg_c / (ms_c * 1e-3) / 1e9 / peak, 4),
            "frac_paged": round(alg / (ms_p * 1e-3) / 1e9 / peak, 4),
            "algorithmic_bytes_per_launch": int(alg_c)},
        "memory": {"chunk_bytes": st_map["chunk_bytes"],
                   "vcache_mapped_bytes": st_map["mapped_bytes"],
                   "paged_block_bytes": paged_bytes,
                   "vcache_over_paged": round(st_map["mapped_bytes"] / paged_bytes, 4)},
        "host": {"initial_map_ms": round(map_s * 1e3, 2), "initial_chunks": st_map["map_calls"],
                 "us_per_chunk_mapped": round(map_s * 1e6 / max(1, st_map["map_calls"]), 2),
                 "grow_steps": grow_steps,
                 "paged_append_batch_and_build_us_per_step": round(float(np.median(t_paged)) * 1e6, 2),
                 "vcache_reserve_batch_us_per_step_median": round(float(np.median(t_vc)) * 1e6, 2),
                 "vcache_reserve_batch_us_per_step_mean": round(float(np.mean(t_vc)) * 1e6, 2),
                 "chunks_mapped_while_growing": int(grow_maps)},
        "clocks": clk.summary(min_samples=20),
    }
    vc.close()
    pool.close()
    return res


# Workloads measured after the headline in the default run, each as its own
# --workload run measures it (calls: timed calls of a single-call workload).
OTHER_WORKLOADS = [
    ("gqa_long_bs16", "decode", 0), ("gqa_long_bs32", "decode", 0),
    ("llama13b_churn", "schedule", 0), ("sharing_A", "schedule", 200),
    ("sharing_B", "schedule", 200), ("beam", "schedule", 200),
    ("opt13b_fp8", "fp8", 200), ("gqa_long_bs16_fp8", "fp8", 100),
    ("prefill_opt13b_t16", "prefill", 200),
    ("prefill_gqa_bs16_t4", "prefill", 200), ("prefill_prompt512", "prefill", 50),
    ("vcache_opt13b", "vcache", 200), ("vcache_gqa_long_bs16", "vcache", 100),
]


def _summary(rec):
    """The parts of a workload's line that the default line carries."""
    keep = ("value", "unit", "steps", "warmup", "ms_per_step", "dtype", "config", "roofline",
            "clocks", "seq_tokens_per_s", "query_tokens_per_s", "attention_tflops",
            "f16_cache_same_batch", "rows", "call_us_median", "call_us_mean", "calls", "timed", "hbm_view",
            "workload", "name", "paged_call_us", "contiguous_call_us", "translation_cost",
            "outputs_bit_identical", "outputs_max_abs_diff", "memory", "host")
    return {k: v for k, v in rec.items() if k in keep}


def workload_records(args, device):
    import types

    out = {}
    for name, kind, calls in OTHER_WORKLOADS:
        t0 = time.perf_counter()
        try:
            if kind == "decode":
                rec = decode_record(name, device)
            elif kind == "vcache":
                rec = vcache_record(name[len("vcache_"):], device, calls=calls)
            else:
                a = types.SimpleNamespace(**vars(args))
                a.workload, a.partition, a.num_seqs, a.decode = name, None, None, "auto"
                if calls:
                    a.steps = calls
                a.warmup = max(3, args.warmup)
                rec = {"schedule": schedule_record, "fp8": fp8_record,
                       "prefill": prefill_record}[kind](a)
            rec = _summary(rec)
        except Exception as exc:  # one workload's failure must not lose the others
            rec = {"error": repr(exc)[:300]}
        rec["wall_s"] = round(time.perf_counter() - t0, 1)
        out[name] = rec
        release_memory()
    return out


def measure_rows(wl, rep, device, k_step, v_step, host_us):
    """The other rows of the hot path, each against its own roofline: host
    bookkeeping per step (a1), copy_blocks (a2) and reshape_and_cache (a3).
    Copies and scatters target free blocks of the pool, so no live sequence
    changes."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    g = wl.geometry
    peak, _ = peaks()
    stream = torch.cuda.current_stream(device)
    free = np.asarray(rep.pool.free_list(), dtype=np.int64)
    used = np.setdiff1d(np.arange(wl.num_blocks), free)
    block_bytes = 2 * g.num_kv_heads * g.block_size * g.head_dim * g.elem_bytes

    def timed(fn, reps=20):
        """Device time per call: the calls are captured in a CUDA graph and the
        graph replayed, so host launch overhead of small calls is not timed."""
        for _ in range(3):
            fn()
        torch.cuda.synchronize(device)
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for _ in range(reps):
                    fn()
        stream.wait_stream(side)
        graph.replay()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        del graph
        return e0.elapsed_time(e1) / reps * 1e3  # us

    out = {"a1_host_bookkeeping_us_per_step": round(float(np.median(host_us)), 1)}
    # a2: copy-on-write copies, up to 1024 pairs (sources in use, destinations free)
    n = int(min(1024, len(free), len(used)))
    if n > 0:
        pairs = torch.tensor(np.stack([used[:n], free[:n]], 1), dtype=torch.int32, device=device)
        us = timed(lambda: kvp.copy_blocks(rep.k, rep.v, pairs))
        moved = 2 * n * block_bytes  # read + write
        out["a2_copy_blocks"] = {"pairs": n, "us": round(us, 2), "GBps": round(moved / us / 1e3, 1),
                                 "frac": round(moved / us / 1e3 / peak, 3)}
    # a3: one decode step's scatter (launch-bound) and a bulk prefill-sized scatter
    S = k_step.shape[0]
    slots = torch.tensor(free[:S] * g.block_size, dtype=torch.int64, device=device)
    us = timed(lambda: kvp.reshape_and_cache(k_step, v_step, rep.k, rep.v, slots))
    out["a3_reshape_and_cache_step"] = {"tokens": S, "us": round(us, 2)}
    nb = int(min(len(free), 2048))
    T = nb * g.block_size
    bulk_slots = torch.from_numpy((free[:nb, None] * g.block_size +
                                   np.arange(g.block_size)[None, :]).reshape(-1)).to(device)
    kb = torch.randn((T, g.num_kv_heads, g.head_dim), dtype=k_step.dtype, device=device)
    vb = torch.randn_like(kb)
    us = timed(lambda: kvp.reshape_and_cache(kb, vb, rep.k, rep.v, bulk_slots), reps=10)
    moved = 2 * 2 * T * g.num_kv_heads * g.head_dim * g.elem_bytes + 8 * T
    out["a3_reshape_and_cache_bulk"] = {"tokens": T, "us": round(us, 1),
                                        "GBps": round(moved / us / 1e3, 1),
                                        "frac": round(moved / us / 1e3 / peak, 3)}
    kvp.check_device_error(device)
    return out


def run_e2e(args, wl, reps, device, seed_rank, MB, max_ctx_total, part, ws, world):
    """Same metric with host inputs: per step, pinned host -> device copies of q, the
    new K/V and the metadata, the kernels, and the output copied back, synchronised.
    The host bookkeeping of step i + 1 (appends, block tables) runs while the GPU
    runs step i (two pinned metadata buffers), as an engine's scheduler would; the
    inputs go up, the result comes down and the host waits for it every step."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    g = wl.geometry
    S = len(reps[0].seqs)
    K = max(1, min(args.steps, 64))
    R = len(reps)
    pin = lambda t: t.pin_memory()
    host_q = pin(torch.from_numpy(normal_bits(value_seed_words(seed_rank, Q_STREAM, 999), (S, g.num_q_heads, g.head_dim), g.dtype).view(np.int16)))
    host_k = pin(torch.from_numpy(normal_bits(value_seed_words(seed_rank, K_STREAM, 999), (S, g.num_kv_heads, g.head_dim), g.dtype).view(np.int16)))
    host_v = pin(torch.from_numpy(normal_bits(value_seed_words(seed_rank, V_STREAM, 999), (S, g.num_kv_heads, g.head_dim), g.dtype).view(np.int16)))
    tdt = torch.float16 if g.dtype == "f16" else torch.bfloat16
    host_out = torch.empty((S, g.num_q_heads, g.head_dim), dtype=torch.int16).pin_memory()
    metas = [StepMeta(S, MB, device), StepMeta(S, MB, device)]
    q_d = torch.empty((S, g.num_q_heads, g.head_dim), dtype=tdt, device=device)
    k_d = torch.empty((S, g.num_kv_heads, g.head_dim), dtype=tdt, device=device)
    v_d = torch.empty_like(k_d)
    out = torch.empty_like(q_d)
    h2d = (host_q.numel() + host_k.numel() + host_v.numel()) * 2 + metas[0].nbytes
    d2h = host_out.numel() * 2
    stream = torch.cuda.current_stream(device)

    def up(m):
        q_d.view(torch.int16).copy_(host_q, non_blocking=True)
        k_d.view(torch.int16).copy_(host_k, non_blocking=True)
        v_d.view(torch.int16).copy_(host_v, non_blocking=True)
        m.upload()

    def kernels(rep, m):
        kvp.reshape_and_cache(k_d, v_d, rep.k, rep.v, m.slot_d)
        kvp.paged_attention_decode(q_d, rep.k, rep.v, m.tab_d, m.len_d, wl.scale, out,
                                   max_context_len=max_ctx_total, partition_size=part, workspace=ws)

    def down():
        host_out.copy_(out.view(torch.int16), non_blocking=True)

    def device_part(rep, m):
        """One step's stream work: inputs up, scatter, decode, result down."""
        up(m)
        kernels(rep, m)
        down()

    def book(rep, m):
        """Host bookkeeping of a step into a pinned metadata buffer; CoW pairs."""
        rep.pool.append_batch(rep.seqs, 1, out=m.slot_h.numpy())
        copies = rep.pool.take_copies()
        rep.pool.build_batch(rep.seqs, MB, m.tab_h.numpy(), m.len_h.numpy())
        rep.lens += 1
        return copies

    # One CUDA graph per (replica, metadata buffer), captured once; it reads the
    # pinned buffers the bookkeeping fills in. A step with copy-on-write pairs runs
    # eagerly.
    graphs = {}
    try:
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            for ri, rep in enumerate(reps):
                for b, m in enumerate(metas):
                    gr = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(gr, stream=side):
                        device_part(rep, m)
                    graphs[(ri, b)] = gr
        stream.wait_stream(side)
        torch.cuda.synchronize(device)
    except Exception as exc:  # capture unsupported here: eager steps
        graphs = {}
        print(f"e2e: CUDA graph capture failed ({exc}); eager steps", file=sys.stderr)
    total_bytes = 0
    barrier(world)
    torch.cuda.synchronize(device)
    t = time.perf_counter()
    eager = 0
    copies = book(reps[0], metas[0])
    for i in range(K):
        rep, b = reps[i % R], i % 2
        m = metas[b]
        if copies or not graphs:
            if copies:
                kvp.copy_blocks(rep.k, rep.v, torch.tensor(copies, dtype=torch.int32).to(device))
            device_part(rep, m)
            eager += 1
        else:
            graphs[(i % R, b)].replay()
        step_bytes = algorithmic_bytes(m.len_h.numpy(), g)
        if i + 1 < K:  # the next step's bookkeeping, while this one runs
            copies = book(reps[(i + 1) % R], metas[(i + 1) % 2])
        stream.synchronize()  # this step's result is on the host
        total_bytes += step_bytes
    el = time.perf_counter() - t
    el = dist_max(el, world)
    total_bytes = dist_sum(float(total_bytes), world)
    # The same steps eagerly: every step calls the library (argument checks, tensor-map
    # encoding, launches) through its binding, as a caller without graphs would.
    K_eager = max(1, min(args.steps, 32))
    eager_bytes = 0
    barrier(world)
    torch.cuda.synchronize(device)
    t = time.perf_counter()
    copies = book(reps[K % R], metas[K % 2])
    for i in range(K, K + K_eager):
        rep, m = reps[i % R], metas[i % 2]
        if copies:
            kvp.copy_blocks(rep.k, rep.v, torch.tensor(copies, dtype=torch.int32).to(device))
        device_part(rep, m)
        step_bytes = algorithmic_bytes(m.len_h.numpy(), g)
        if i + 1 < K + K_eager:
            copies = book(reps[(i + 1) % R], metas[(i + 1) % 2])
        stream.synchronize()
        eager_bytes += step_bytes
    el_eager = dist_max(time.perf_counter() - t, world)
    eager_bytes = dist_sum(float(eager_bytes), world)
    # Where a step's time goes (not part of the timed loop): host bookkeeping,
    # and each piece of the device work timed alone with CUDA events.
    brk = {}
    try:
        rep, m = reps[0], metas[0]
        hb = []
        for _ in range(5):
            t0 = time.perf_counter()
            book(rep, m)
            hb.append(time.perf_counter() - t0)
        rep.pool.take_copies()

        def ev_time(fn, n=10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            fn()
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
            torch.cuda.synchronize(device)
            return e0.elapsed_time(e1) / n * 1e3

        def wall(fn, n=10):
            fn()
            torch.cuda.synchronize(device)
            t0 = time.perf_counter()
            for _ in range(n):
                fn()
                stream.synchronize()
            return (time.perf_counter() - t0) / n * 1e6

        brk = {"host_bookkeeping_us": round(float(np.median(hb)) * 1e6, 1),
               "h2d_us": round(ev_time(lambda: up(m)), 1),
               "kernels_us": round(ev_time(lambda: kernels(rep, m)), 1),
               "d2h_us": round(ev_time(down), 1),
               "graph_step_wall_us": round(wall(lambda: graphs[(0, 0)].replay()), 1) if graphs else None,
               "step_us_in_timed_loop": round(el / K * 1e6, 1)}
    except Exception as exc:  # pragma: no cover - diagnostics only
        brk = {"error": repr(exc)[:200]}
    graphs.clear()
    return {"value": round(total_bytes / el / 1e9, 2), "unit": UNIT, "steps": K,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "how": "per step: one CUDA graph replay (inputs from pinned host memory up, scatter, "
                   "decode, result down) and a synchronize; the next step's host bookkeeping "
                   "runs while the graph runs" + (f"; {eager} steps eager" if eager else ""),
            "breakdown": brk,
            "eager": {"value": round(eager_bytes / el_eager / 1e9, 2), "unit": UNIT,
                      "steps": K_eager, "step_us": round(el_eager / K_eager * 1e6, 1),
                      "how": "the same steps without graphs: every step calls the C ABI through "
                             "the binding (copies up, reshape_and_cache, paged_attention_decode, "
                             "copy down) and synchronizes"}}


# ---------------------------------------------------------------- CPU oracle
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info

        return max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        return int(os.environ.get("OMP_NUM_THREADS", "1"))


def cpu_baseline(wl, budget_s=15.0, seqs_per_step=None):
    """The fp64 oracle on the host: gather + softmax(qK^T)V per sequence, timed on a
    bounded sample of the workload's decode step (the first sequences of the batch)."""
    from oracle.replay import OracleReplay

    rp = OracleReplay(wl)
    rp.run()
    (i, seqs, tables, lens), = rp.attends[-1:]
    g = wl.geometry
    done, nbytes = 0, 0
    t0 = time.perf_counter()
    order = list(range(len(lens)))
    while time.perf_counter() - t0 < budget_s and done < len(order):
        s = order[done]
        rp.decode(i, tables, lens, seqs=[s], split=False)
        nbytes += algorithmic_bytes([lens[s]], g)
        done += 1
    el = time.perf_counter() - t0
    return {"value": round(nbytes / el / 1e9, 4), "unit": UNIT,
            "cores": len(os.sched_getaffinity(0)), "blas_threads": cpu_threads(), "kind": "oracle",
            "sample": f"{done} of {len(lens)} sequences of one decode step ({wl.name}), "
                      f"{nbytes / 1e9:.3f} GB of K/V, {el:.1f} s"}


def unique_bytes(tables, lens, g):
    """Bytes of the distinct physical blocks a batch reads (each block's valid slots
    counted once, however many sequences share it), plus q, out and metadata."""
    valid = {}
    bs = g.block_size
    for row, L in zip(np.asarray(tables), np.asarray(lens)):
        for i in range(-(-int(L) // bs)):
            b = int(row[i])
            valid[b] = max(valid.get(b, 0), min(bs, int(L) - i * bs))
    kv = sum(valid.values()) * g.num_kv_heads * g.head_dim * g.elem_bytes * 2
    qo = len(lens) * g.num_q_heads * g.head_dim * g.elem_bytes * 2
    return kv + qo + 4 * int(np.sum(-(-np.asarray(lens) // bs))) + 4 * len(lens)


def schedule_record(args):
    """Workloads whose steps change the batch (churn, sharing, beam): the schedule is
    replayed once through libkvp and every attention call is timed with CUDA events.
    Values are drawn on the device (the parity tests replay the seeded host draws)."""
    import torch
    import paged_kv_cache_319_b200 as kvp
    from paged_kv_cache_319_b200.replay import DeviceReplay

    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    kw = {}
    if args.workload in ("llama13b_churn", "beam"):
        kw["steps"] = max(args.warmup + 1, min(args.steps + args.warmup, 32 if args.workload ==
                                                "llama13b_churn" else 64))
    wl = workloads.by_name(args.workload, **kw)
    g = wl.geometry
    packed = args.decode == "packed"
    grouped = args.decode == "grouped" or (args.decode == "auto" and
                                            args.workload in GROUPED_WORKLOADS)
    # a workload with one attend op (sampling, beam) times that call `steps` times
    n_att = sum(1 for op in wl.ops if op[0] == "attend")
    reps = max(1, args.steps) if n_att == 1 else 1
    rp = DeviceReplay(wl, device, keep_outputs=False, time_decode=True, grouped=grouped and not packed,
                      time_reps=reps, device_values=True, packed=packed)
    with ClockSampler(device) as clk:
        rp.run()
        torch.cuda.synchronize(device)
    kvp.check_device_error(device)
    attends = {i: (t, l) for (i, _, t, l) in rp.attends}
    per_op = {}
    for i, e0, e1 in rp.decode_events:
        per_op.setdefault(i, []).append(e0.elapsed_time(e1))
    rows = []
    for i in sorted(per_op):
        t, l = attends[i]
        ms = float(np.median(per_op[i]))  # median of the op's timed calls
        rows.append((ms, algorithmic_bytes(l, g), unique_bytes(t, l, g), int(np.sum(l))))
    timed = rows[args.warmup:] if len(rows) > args.warmup else rows
    ms = np.array([r[0] for r in timed])
    logical = np.array([r[1] for r in timed], dtype=np.float64)
    uniq = np.array([r[2] for r in timed], dtype=np.float64)
    toks = np.array([r[3] for r in timed], dtype=np.float64)
    peak, peak_kind = peaks()
    if packed:
        kernel = ("paged_attention_decode_packed (plan built on the host): decode_tc (packed: "
                  "shared prefixes and own blocks in one stream per group)")
    elif grouped:
        kernel = ("paged_attention_decode_grouped (plan built on the host): decode_tc (grouped, "
                  "shared prefixes) + " + ("decode_tc (own ranges)" if g.num_q_heads > g.num_kv_heads
                                           else "decode_simt (own ranges)"))
    else:
        kernel = "paged_attention_decode: " + (
            "decode_tc" if g.num_q_heads > g.num_kv_heads else "decode_simt")
    st = rp.pool.stats()
    achieved_u = float(uniq.sum() / (ms.sum() * 1e-3) / 1e9)
    res = {
        "metric": METRIC, "value": round(float(logical.sum() / (ms.sum() * 1e-3) / 1e9), 2),
        "unit": UNIT, "n_gpus": 1, "steps": len(timed), "warmup": len(rows) - len(timed),
        "ms_per_step": round(float(ms.mean()), 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": g.dtype, "data": "synthetic",
        "config": {"workload": wl.description, "name": wl.name,
                   "timed": "attention calls only" + (
                       f" (median of {reps} calls, L2 flushed before each)" if reps > 1 else ""),
                   "decode": "packed" if packed else ("grouped" if grouped else "per-sequence")},
        "seq_tokens_per_s": round(float(toks.sum() / (ms.sum() * 1e-3)), 1),
        "roofline": {"kernel": f"{kernel} + decode_reduce_kernel",
                     "bound": "hbm", "achieved_unique": round(achieved_u, 1),
                     "achieved_logical": round(float(logical.sum() / (ms.sum() * 1e-3) / 1e9), 1),
                     "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                     "frac": round(achieved_u / peak, 4),
                     "avg_launch_us": round(float(ms.mean() * 1e3), 2),
                     "unique_bytes_per_launch": int(uniq.mean()),
                     "logical_bytes_per_launch": int(logical.mean())},
        "pool": {k: int(v) for k, v in st.items()},
        "clocks": clk.summary(),
    }
    return res


# Paged prefill workloads: a chunk of T new tokens per sequence, causal within
# the chunk, over a pool already holding every context (chunk included).
# Partitions of 2048 tokens: the chunk's columns make each partition's partial
# (written by pass 1, read by the reduce) T times larger than in decode, and
# fewer, longer units keep the tensor-core pipeline full (measured on B200,
# 16-token chunks of the OPT-13B batch: 485 / 392 / 314 us at 512 / 1024 / 2048).
PREFILL_PARTITION = 2048
PREFILL_WORKLOADS = {
    "prefill_opt13b_t16": ("opt13b", 16),        # OPT-13B batch, 16-token chunks
    "prefill_gqa_bs16_t4": ("gqa_long_bs16", 4),  # long-context GQA, 4-token chunks
    "prefill_prompt512": ("prompt512", 512),     # 64 whole prompts of 512 tokens
}


def prefill_record(args):
    """paged_attention_prefill, timed with CUDA events (median of --steps calls, L2
    flushed before each); roofline on algorithmic bytes: K/V of every context token
    read once, q, out, block tables and lengths."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    base, T = PREFILL_WORKLOADS[args.workload]
    if base == "prompt512":
        g = workloads.Geometry(40, 40, 128, 16, "f16")
        lens = np.full(64, 512, np.int64)
        part, desc = 512, "OPT-13B geometry, 64 prompts of 512 tokens prefilled whole (ctx = T = 512)"
    else:
        wl = workloads.by_name(base)
        g = wl.geometry
        lens = np.asarray(wl.info["context_lens"], np.int64)
        part, desc = PREFILL_PARTITION, f"{wl.description}; a chunk of the last {T} tokens per sequence"
    if args.partition:
        part = args.partition
    if getattr(args, "num_seqs", None):  # a smaller case of the same workload (profiling)
        lens = lens[:args.num_seqs]
        desc += f"; first {len(lens)} sequences"
    S, Hq, Hkv, D, bs = len(lens), g.num_q_heads, g.num_kv_heads, g.head_dim, g.block_size
    rng = np.random.default_rng(3001)
    need = -(-lens // bs)
    NB = int(need.sum()) + 8
    perm = rng.permutation(NB).astype(np.int32)
    tables = np.full((S, int(need.max())), -1, np.int32)
    i = 0
    for s_, n in enumerate(need):
        tables[s_, :n] = perm[i:i + n]
        i += n
    tdt = torch.float16 if g.dtype == "f16" else torch.bfloat16
    gen = torch.Generator(device=device).manual_seed(3002)
    k = torch.randn((NB, Hkv, bs, D), generator=gen, device=device, dtype=torch.float32).to(tdt)
    v = torch.randn((NB, Hkv, bs, D), generator=gen, device=device, dtype=torch.float32).to(tdt)
    q = torch.randn((S, T, Hq, D), generator=gen, device=device, dtype=torch.float32).to(tdt)
    tt = torch.from_numpy(tables).to(device)
    cl = torch.from_numpy(lens.astype(np.int32)).to(device)
    mcl = int(lens.max())
    out = torch.empty_like(q)
    ws = torch.empty(max(1, kvp.lib().kvp_prefill_workspace_bytes(S, T, Hq, D, mcl, part)),
                     dtype=torch.uint8, device=device)
    call = lambda: kvp.paged_attention_prefill(q, k, v, tt, cl, 1 / math.sqrt(D), out,  # noqa: E731
                                               max_context_len=mcl, partition_size=part,
                                               workspace=ws)
    for _ in range(max(3, args.warmup)):
        call()
    kvp.check_device_error(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    clean = torch.ones(256 << 20, dtype=torch.uint8, device=device)
    pairs = []
    with ClockSampler(device) as clk:
        for _ in range(max(1, args.steps)):
            flush.fill_(1)
            clean.amax()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            pairs.append((e0, e1))
        torch.cuda.synchronize(device)
    ms = float(np.median([a.elapsed_time(b) for a, b in pairs]))
    kv = float(lens.sum()) * Hkv * D * g.elem_bytes * 2
    alg = kv + S * T * Hq * D * g.elem_bytes * 2 + 4 * float(need.sum()) + 4 * S
    G = Hq // Hkv
    # the library's routing: chunks of at least 64 query rows (T x G, G a power of two) run on
    # the prompt-shaped kernel in one launch, shorter ones 16 columns per launch
    prompt_tiles = T > 1 and (G & (G - 1)) == 0 and T * G >= 64
    launches = 1 if prompt_tiles else (-(-T // max(1, 16 // G)) if T > 1 else 1)
    vis = np.clip(lens[:, None] - T + np.arange(T)[None, :] + 1, 0, None)  # visible tokens per query
    flops = 4.0 * float(vis.sum()) * D * Hq
    peak, peak_kind = peaks()
    achieved = alg / (ms * 1e-3) / 1e9
    tflops = flops / (ms * 1e-3) / 1e12
    split = part < int(lens.max())
    kname = ("paged_attention_prefill: prefill_tc (128 query rows x 128 keys per tcgen05 tile)"
             if prompt_tiles else "paged_attention_prefill: decode_tc (multi-query)") + \
        (" + decode_reduce_kernel" if split else "")
    hbm_view = {"kernel": kname, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "peak_source": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                "algorithmic_bytes_per_launch": int(alg),
                "note": f"algorithmic bytes count the keys and values once per call; "
                        f"each of the call's {launches} launch(es) reads the tokens that its "
                        f"queries see",
                "avg_launch_us": round(ms * 1e3, 2)}
    if prompt_tiles:
        sus, burst, tkind = tensor_peaks()
        roofline = {"kernel": kname, "bound": "tensor", "achieved": round(tflops, 1), "peak": sus,
                    "peak_source": tkind + " (bf16_tflops_sustained; fp16 has the same dense rate)",
                    "unit": "TFLOP/s", "frac": round(tflops / sus, 4),
                    "frac_of_burst": round(tflops / burst, 4),
                    "flops_per_launch": flops, "flops": "4 * head_dim * Hq per visible (query, key) pair",
                    "avg_launch_us": round(ms * 1e3, 2), "traffic": None}
    else:
        roofline = hbm_view
    res = {
        "metric": METRIC, "value": round(achieved, 2), "unit": UNIT, "n_gpus": 1,
        "steps": len(pairs), "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": g.dtype,
        "data": "synthetic (seeded normal q/K/V on the device)",
        "config": {"workload": desc, "name": args.workload, "chunk_tokens": T,
                   "launches_per_call": launches, "partition_size": part,
                   "timed": f"paged_attention_prefill (median of {len(pairs)} calls, L2 "
                            "flushed before each)"},
        "query_tokens_per_s": round(S * T / (ms * 1e-3), 1),
        "attention_tflops": round(tflops, 2),
        "roofline": roofline,
        "hbm_view": hbm_view,
        "clocks": clk.summary(),
    }
    return res


FP8_WORKLOADS = ("opt13b_fp8", "gqa_long_bs16_fp8")
# the virtually contiguous cache against the paged one, on a workload's batch
VCACHE_WORKLOADS = {"vcache_opt13b": "opt13b", "vcache_gqa_long_bs16": "gqa_long_bs16"}


def fp8_record(args):
    """paged_attention_decode_fp8 on a decode batch (OPT-13B, or long-context GQA)
    with an E4M3 cache, timed with CUDA events (median of --steps calls, L2 flushed
    before each), beside the 16-bit decode of the same batch; roofline on the E4M3
    algorithmic bytes."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(device)
    base = args.workload[:-len("_fp8")]
    wl = workloads.by_name(base)
    g = wl.geometry
    qdt = torch.float16 if g.dtype == "f16" else torch.bfloat16
    nsub = getattr(args, "num_seqs", None)  # a smaller case of the same workload (profiling)
    lens = np.asarray(wl.info["context_lens"], np.int64)
    if nsub:
        lens = lens[:nsub]
    S, Hq, Hkv, D, bs, part = len(lens), g.num_q_heads, g.num_kv_heads, g.head_dim, g.block_size, 512
    rng = np.random.default_rng(4001)
    need = -(-lens // bs)
    NB = int(np.ceil(1.25 * need.sum()))
    perm = rng.permutation(NB).astype(np.int32)
    tables = np.full((S, int(need.max())), -1, np.int32)
    i = 0
    for s_, n in enumerate(need):
        tables[s_, :n] = perm[i:i + n]
        i += n
    gen = torch.Generator(device=device).manual_seed(4002)

    def codes():  # uniform E4M3 codes without the two NaN codes
        c = torch.randint(0, 256, (NB, Hkv, bs, D), generator=gen, device=device, dtype=torch.uint8)
        return torch.where((c & 0x7F) == 0x7F, c & 0xBF, c)

    kc, vc = codes(), codes()
    ks = torch.linspace(1 / 448, 2 / 448, Hkv, device=device, dtype=torch.float32)
    vs = torch.linspace(1 / 448, 4 / 448, Hkv, device=device, dtype=torch.float32)
    q = torch.randn((S, Hq, D), generator=gen, device=device, dtype=torch.float32).to(qdt)
    tt = torch.from_numpy(tables).to(device)
    cl = torch.from_numpy(lens.astype(np.int32)).to(device)
    mcl = int(lens.max())
    out = torch.empty_like(q)
    ws = torch.empty(max(1, kvp.decode_workspace_bytes(S, Hq, D, mcl, part)), dtype=torch.uint8,
                     device=device)
    scale = 1 / math.sqrt(D)
    call = lambda: kvp.paged_attention_decode_fp8(q, kc, vc, ks, vs, tt, cl, scale, out,  # noqa: E731
                                                  max_context_len=mcl, partition_size=part,
                                                  workspace=ws)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    clean = torch.ones(256 << 20, dtype=torch.uint8, device=device)

    def timed(fn, n):
        pairs = []
        for _ in range(n):
            flush.fill_(1)
            clean.amax()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            pairs.append((e0, e1))
        torch.cuda.synchronize(device)
        return float(np.median([a.elapsed_time(b) for a, b in pairs]))

    for _ in range(max(3, args.warmup)):
        call()
    kvp.check_device_error(device)
    steps = max(1, args.steps)
    with ClockSampler(device) as clk:
        ms = timed(call, steps)
    # the new token of every sequence, quantised into the cache (one decode step's scatter)
    kn = torch.randn((S, Hkv, D), generator=gen, device=device, dtype=torch.float32).to(qdt)
    vn = torch.randn((S, Hkv, D), generator=gen, device=device, dtype=torch.float32).to(qdt)
    slots = torch.from_numpy((tables[np.arange(S), (lens - 1) // bs].astype(np.int64) * bs
                              + (lens - 1) % bs)).to(device)
    scatter = lambda: kvp.reshape_and_cache_fp8(kn, vn, kc, vc, slots, ks, vs)  # noqa: E731
    for _ in range(3):
        scatter()
    scatter_ms = timed(scatter, steps)
    kvp.check_device_error(device)
    # the 16-bit decode of the same batch (fp16 K/V of the same shape)
    del kc, vc
    k16 = torch.randn((NB, Hkv, bs, D), generator=gen, device=device, dtype=torch.float32).to(qdt)
    v16 = torch.randn((NB, Hkv, bs, D), generator=gen, device=device, dtype=torch.float32).to(qdt)
    call16 = lambda: kvp.paged_attention_decode(q, k16, v16, tt, cl, scale, out,  # noqa: E731
                                                max_context_len=mcl, partition_size=part,
                                                workspace=ws)
    for _ in range(3):
        call16()
    ms16 = timed(call16, steps)
    kvp.check_device_error(device)

    kv = float(lens.sum()) * Hkv * D * 1 * 2
    alg = kv + S * Hq * D * 2 * 2 + 4 * float(need.sum()) + 4 * S
    peak, peak_kind = peaks()
    achieved = alg / (ms * 1e-3) / 1e9
    res = {
        "metric": METRIC, "value": round(achieved, 2), "unit": UNIT, "n_gpus": 1,
        "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"e4m3 (K/V cache), {g.dtype} (q, out), fp32 accumulation",
        "data": "synthetic (uniform E4M3 codes, per-KV-head scales; seeded N(0,1) q)",
        "config": {"workload": (wl.description + ", E4M3 cache with per-KV-head scales"
                                if base != "opt13b" else
                                "OPT-13B geometry, one layer: 64 seqs, 40 heads x 128, block 16, "
                                "ctx U[1,2048], E4M3 cache with per-KV-head scales, partitions of 512"),
                   "name": args.workload,
                   "timed": f"paged_attention_decode_fp8 (median of {steps} calls, L2 flushed "
                            "before each)"},
        "seq_tokens_per_s": round(float(lens.sum()) / (ms * 1e-3), 1),
        "f16_cache_same_batch": {"call_us": round(ms16 * 1e3, 2),
                                 "seq_tokens_per_s": round(float(lens.sum()) / (ms16 * 1e-3), 1),
                                 "speedup_of_e4m3": round(ms16 / ms, 3)},
        "rows": {"reshape_and_cache_fp8_step": {"tokens": S, "us": round(scatter_ms * 1e3, 2)}},
        "roofline": {"kernel": ("paged_attention_decode_fp8: decode_tc (E4M3 tiles widened in shared "
                                "memory) + decode_reduce_kernel" if Hq > Hkv else
                                "paged_attention_decode_fp8: decode_simt (E4M3) + decode_reduce_kernel"),
                     "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "peak_source": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "algorithmic_bytes_per_launch": int(alg), "avg_launch_us": round(ms * 1e3, 2),
                     "traffic": traffic_per_launch("decode_simt_fp8" if Hq == Hkv else "decode_tc_fp8",
                                                   alg)},
        "clocks": clk.summary(),
    }
    return res


def run_reference_sampled(args, world):
    """Reference arm of the prefill and E4M3 workloads: the matching oracle
    (``attention.paged_prefill`` / ``fp8.paged_decode``) on one sequence of the
    workload per step, longest first, inputs drawn before the timed region."""
    from oracle import attention, fp8

    fp8_case = args.workload in FP8_WORKLOADS
    base, T = (args.workload[:-len("_fp8")], 1) if fp8_case else PREFILL_WORKLOADS[args.workload]
    if base == "prompt512":
        g = workloads.Geometry(40, 40, 128, 16, "f16")
        lens = np.full(64, 512, np.int64)
    else:
        wl = workloads.by_name(base)
        g = wl.geometry
        lens = np.asarray(wl.info["context_lens"], np.int64)
    Hq, Hkv, D, bs = g.num_q_heads, g.num_kv_heads, g.head_dim, g.block_size
    rng = np.random.default_rng(6001)
    order = np.argsort(lens)[::-1]
    n = args.warmup + args.steps
    cases = []
    for k in range(n):
        L = int(lens[order[k % len(order)]])
        nb = -(-L // bs)
        table = np.arange(nb, dtype=np.int32)[None]
        if fp8_case:
            kc = rng.integers(0, 256, (nb, Hkv, bs, D), dtype=np.uint8)
            vc = rng.integers(0, 256, (nb, Hkv, bs, D), dtype=np.uint8)
            kc[(kc & 0x7F) == 0x7F] = 0x3F
            vc[(vc & 0x7F) == 0x7F] = 0x3F
            nbytes = L * Hkv * D * 2 + Hq * D * 4 + 4 * nb + 4
        else:
            kc = rng.standard_normal((nb, Hkv, bs, D))
            vc = rng.standard_normal((nb, Hkv, bs, D))
            nbytes = L * Hkv * D * g.elem_bytes * 2 + T * Hq * D * g.elem_bytes * 2 + 4 * nb + 4
        q = rng.standard_normal((1, T, Hq, D) if not fp8_case else (1, Hq, D))
        cases.append((L, table, kc, vc, q, nbytes))
    ks = np.full(Hkv, 1 / 448, np.float32)
    vs = np.full(Hkv, 2 / 448, np.float32)
    scale = 1 / math.sqrt(D)

    def one(c):
        L, table, kc, vc, q, nbytes = c
        if fp8_case:
            fp8.paged_decode(q, kc, vc, table, [L], scale, bs, ks, vs)
        else:
            attention.paged_prefill(q, kc, vc, table, [L], scale, bs)
        return nbytes

    for c in cases[:args.warmup]:
        one(c)
    t0 = time.perf_counter()
    nbytes = sum(one(c) for c in cases[args.warmup:])
    el = time.perf_counter() - t0
    value = nbytes / el / 1e9
    what = "one sequence's E4M3 decode" if fp8_case else f"one sequence's {T}-token prefill"
    res = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / max(1, args.steps), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "name": args.workload},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "kind": "oracle",
                         "cores": len(os.sched_getaffinity(0)), "blas_threads": cpu_threads(),
                         "sample": f"{what} per step (longest contexts first)"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def run_reference(args, world, rank):
    """The oracle as the reference arm: each step is a bounded sample of the workload."""
    if rank != 0:
        return
    if args.workload in FP8_WORKLOADS or args.workload in PREFILL_WORKLOADS:
        run_reference_sampled(args, world)
        return
    from oracle.replay import OracleReplay

    wl = make_workload(args)
    rp = OracleReplay(wl)
    rp.run()
    (i, seqs, tables, lens), = rp.attends[-1:]
    g = wl.geometry
    per_step = max(1, min(len(lens), args.ref_seqs_per_step))
    order = np.argsort(np.asarray(lens))[::-1][: len(lens)].tolist()

    def one(k):
        sel = [order[(k * per_step + j) % len(order)] for j in range(per_step)]
        rp.decode(i, tables, lens, seqs=sel, split=False)
        return algorithmic_bytes([lens[s] for s in sel], g)

    for k in range(args.warmup):
        one(k)
    t0 = time.perf_counter()
    nbytes = sum(one(args.warmup + k) for k in range(args.steps))
    el = time.perf_counter() - t0
    value = nbytes / el / 1e9
    res = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "impl": "reference",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.description, "name": wl.name},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "kind": "oracle",
                         "cores": len(os.sched_getaffinity(0)), "blas_threads": cpu_threads(),
                         "sample": f"{per_step} sequence(s) of one decode step per step"},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="opt13b",
                    choices=["opt13b", "gqa_long_bs16", "gqa_long_bs32", "llama13b_churn",
                             "sharing_A", "sharing_B", "beam"] + list(PREFILL_WORKLOADS)
                    + list(FP8_WORKLOADS) + list(VCACHE_WORKLOADS))
    ap.add_argument("--partition", type=int, default=None)
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="smaller batch of the same workload (profiling small cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seqs-per-step", type=int, default=1)
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the decode window and the other workloads' records of the "
                         "default line")
    ap.add_argument("--decode", choices=["auto", "plain", "grouped", "packed"], default="auto",
                    help="decode entry point of the schedule workloads (auto: grouped for "
                         "the sampling and beam workloads)")
    args = ap.parse_args()
    if args.warmup < 3 and args.workload not in SCHEDULE_WORKLOADS + tuple(PREFILL_WORKLOADS):
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # The oracle needs no GPU and no process group: rank 0 runs, the others exit.
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")),
                      int(os.environ.get("RANK", "0")))
        return
    single_gpu = args.workload in SCHEDULE_WORKLOADS or args.workload in PREFILL_WORKLOADS \
        or args.workload in FP8_WORKLOADS or args.workload in VCACHE_WORKLOADS
    if single_gpu and int(os.environ.get("RANK", "0")) != 0:
        return  # one-GPU workloads: rank 0 runs and prints, the other ranks do nothing
    if args.workload in SCHEDULE_WORKLOADS:
        print(json.dumps(schedule_record(args)), flush=True)
        return
    if args.workload in PREFILL_WORKLOADS:
        print(json.dumps(prefill_record(args)), flush=True)
        return
    if args.workload in FP8_WORKLOADS:
        print(json.dumps(fp8_record(args)), flush=True)
        return
    if args.workload in VCACHE_WORKLOADS:
        import torch

        device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(device)
        print(json.dumps(vcache_record(VCACHE_WORKLOADS[args.workload], device,
                                       calls=max(1, args.steps))), flush=True)
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
