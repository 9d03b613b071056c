"""The five synthetic workloads as seeded operation schedules.

A workload is a geometry, a pool size, the order in which the pool hands out
its physical blocks (a seeded permutation, passed to both block managers as an
input), and a list of operations:

* ``("create", h)``            new empty sequence, handle ``h``
* ``("append", h, n)``         ``n`` new tokens for ``h`` (their K/V values are
                               keyed by the op's index in the list)
* ``("fork", parent, child)``  ``child`` shares every block of ``parent``
* ``("release", h)``           ``h`` finishes
* ``("sync",)``                pending copy-on-write copies, then the K/V of
                               every token appended since the last sync, go to
                               the cache
* ``("attend", [h, ...])``     one decode-attention call over these sequences,
                               in this batch order (q keyed by the op index)

Handles are the generator's own numbering; a driver maps them to the ids its
block manager returns. Seeds: lengths, choices and block placement of workload
``i`` come from ``PCG64(1000 + i)``, values from the value seed ``2000 + i``.

Readings where the configurations leave a detail open:

* ``context_lens`` are lengths after the decode step's append: each sequence
  is prefilled with ``ctx - 1`` tokens, synced, then appends one token, syncs,
  and attends over ``ctx`` tokens.
* Pools are 1.25x the total block need (tiny: 32 blocks; churn: 2x the
  initial need; sharing and beam: 1.25x the no-sharing need of the final
  lengths, an upper bound computed without any allocator).
* Churn: prompt ``round(lognormal(ln 160, 1.0))`` clipped to [1, 2048] plus
  ``U[0, 512]`` already generated tokens; each step ``round(0.1 * 256) = 26``
  live sequences chosen without replacement finish and are replaced by fresh
  prompts.
* Sharing: prompts of 512 tokens have no partly filled last block at block
  size 16, so variant "A" (512) checks that no copy happens and variant "B"
  (prompt ``i`` of ``511 - i`` tokens) makes the shared partial block that
  copy-on-write acts on.
* Beam: 8 prompts (variant B lengths) x width 4; each step every prompt draws
  4 parents with replacement among its beams, forks them, releases the old
  beams and appends one token to each new beam.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Geometry:
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str  # "f16" | "bf16"

    @property
    def elem_bytes(self) -> int:
        return 2


@dataclass
class Workload:
    name: str
    index: int
    geometry: Geometry
    num_blocks: int
    free_order: np.ndarray          # int32 permutation of 0..num_blocks-1
    ops: list
    value_seed: int
    partition_size: int = 0         # 0: one pass over the whole context
    description: str = ""
    info: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.geometry.head_dim)

    def attend_ops(self):
        return [i for i, op in enumerate(self.ops) if op[0] == "attend"]


def _blocks(n: int, bs: int) -> int:
    return -(-n // bs)


def _rng(index: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 + index))


class _Sched:
    def __init__(self):
        self.ops = []
        self.next_h = 0

    def create(self):
        h = self.next_h
        self.next_h += 1
        self.ops.append(("create", h))
        return h

    def append(self, h, n):
        self.ops.append(("append", h, int(n)))

    def fork(self, p):
        c = self.next_h
        self.next_h += 1
        self.ops.append(("fork", p, c))
        return c

    def release(self, h):
        self.ops.append(("release", h))

    def sync(self):
        self.ops.append(("sync",))

    def attend(self, hs):
        self.ops.append(("attend", list(hs)))


def _decode_once(geom, lens, index, name, value_seed, num_blocks, rng, partition_size=0,
                 description=""):
    """Prefill ``ctx - 1`` tokens per sequence, then one decode step over all."""
    sch = _Sched()
    hs = [sch.create() for _ in lens]
    for h, L in zip(hs, lens):
        if L - 1 > 0:
            sch.append(h, L - 1)
    sch.sync()
    for h in hs:
        sch.append(h, 1)
    sch.sync()
    sch.attend(hs)
    order = rng.permutation(num_blocks).astype(np.int32)
    return Workload(name, index, geom, num_blocks, order, sch.ops, value_seed, partition_size,
                    description, {"context_lens": [int(x) for x in lens]})


def tiny() -> Workload:
    geom = Geometry(4, 4, 64, 16, "f16")
    return _decode_once(geom, [1, 15, 16, 37], 0, "tiny", 2000, 32, _rng(0),
                        description="tiny paged decode: 4 seqs, 4 heads x 64, bs 16, "
                                    "ctx {1,15,16,37}, pool 32, fp16")


def opt13b(num_seqs: int = 64, max_len: int = 2048) -> Workload:
    geom = Geometry(40, 40, 128, 16, "f16")
    rng = _rng(1)
    lens = rng.integers(1, max_len + 1, size=num_seqs)
    need = sum(_blocks(int(L), 16) for L in lens)
    nb = math.ceil(1.25 * need)
    return _decode_once(geom, lens, 1, "opt13b", 2001, nb, rng, partition_size=512,
                        description=f"OPT-13B geometry, 1 layer: {num_seqs} seqs, 40 heads x 128, "
                                    f"bs 16, ctx U[1,{max_len}], pool 1.25x need, fp16")


def llama13b_churn(steps: int = 32, num_seqs: int = 256, replace_frac: float = 0.1) -> Workload:
    geom = Geometry(40, 40, 128, 16, "f16")
    rng = _rng(2)

    def prompt():
        return int(min(2048, max(1, round(rng.lognormal(math.log(160.0), 1.0)))))

    sch = _Sched()
    live = []
    init_need = 0
    for _ in range(num_seqs):
        h = sch.create()
        L = prompt() + int(rng.integers(0, 513))
        sch.append(h, L)
        init_need += _blocks(L + 1, 16)
        live.append(h)
    sch.sync()
    n_rep = int(round(replace_frac * num_seqs))
    for _ in range(steps):
        idx = sorted(rng.choice(len(live), size=n_rep, replace=False).tolist())
        done = [live[i] for i in idx]
        for h in done:
            sch.release(h)
        keep = [h for h in live if h not in set(done)]
        fresh = []
        for _ in done:
            h = sch.create()
            sch.append(h, prompt())
            fresh.append(h)
        live = keep + fresh
        for h in live:
            sch.append(h, 1)
        sch.sync()
        sch.attend(live)
    nb = math.ceil(2.0 * init_need)
    order = rng.permutation(nb).astype(np.int32)
    return Workload("llama13b_churn", 2, geom, nb, order, sch.ops, 2002, 512,
                    f"LLaMA-13B geometry, 1 layer: {num_seqs} seqs, prompt lognormal(ln160,1) "
                    f"clipped [1,2048] + U[0,512] generated, {n_rep} replaced per step, "
                    f"{steps} steps, pool 2x initial need, fp16")


def sharing_sampling(variant: str = "B", prompts: int = 8, samples: int = 8,
                     max_suffix: int = 256) -> Workload:
    geom = Geometry(40, 40, 128, 16, "f16")
    rng = _rng(3)
    sch = _Sched()
    groups = []
    lens = []
    for i in range(prompts):
        L = 512 if variant == "A" else 512 - (i + 1)
        lens.append(L)
        p = sch.create()
        sch.append(p, L)
        groups.append([p])
    sch.sync()
    for g in groups:
        for _ in range(samples - 1):
            g.append(sch.fork(g[0]))
    suffix = {h: int(rng.integers(0, max_suffix + 1)) for g in groups for h in g}
    for k in range(1, max(suffix.values()) + 1):
        for g in groups:
            for h in g:
                if suffix[h] >= k:
                    sch.append(h, 1)
        sch.sync()
    allh = [h for g in groups for h in g]
    for h in allh:
        sch.append(h, 1)
    sch.sync()
    sch.attend(allh)
    bound = 0
    for g, L in zip(groups, lens):
        for h in g:
            bound += _blocks(L + suffix[h] + 1, 16)
    nb = math.ceil(1.25 * bound)
    order = rng.permutation(nb).astype(np.int32)
    return Workload(f"sharing_{variant}", 3, geom, nb, order, sch.ops, 2003, 512,
                    f"parallel sampling ({variant}): {prompts} prompts x {samples} samples share "
                    f"prompt blocks, suffix U[0,{max_suffix}], copy-on-write on first write, fp16",
                    {"prompt_lens": lens, "suffix": [suffix[h] for h in allh]})


def beam_search(steps: int = 64, prompts: int = 8, width: int = 4) -> Workload:
    geom = Geometry(40, 40, 128, 16, "f16")
    rng = _rng(3)
    sch = _Sched()
    beams = []
    lens = []
    for i in range(prompts):
        L = 512 - (i + 1)
        lens.append(L)
        p = sch.create()
        sch.append(p, L)
        beams.append([p])
    sch.sync()
    for b in beams:
        for _ in range(width - 1):
            b.append(sch.fork(b[0]))
    for _ in range(steps):
        new_beams = []
        for b in beams:
            parents = rng.integers(0, width, size=width).tolist()
            nb_ = [sch.fork(b[j]) for j in parents]
            for h in b:
                sch.release(h)
            for h in nb_:
                sch.append(h, 1)
            new_beams.append(nb_)
        beams = new_beams
        sch.sync()
    allh = [h for b in beams for h in b]
    sch.attend(allh)
    bound = sum(width * _blocks(L + steps + 1, 16) for L in lens)
    nb = math.ceil(1.25 * bound)
    order = rng.permutation(nb).astype(np.int32)
    return Workload("beam", 3, geom, nb, order, sch.ops, 2013, 512,
                    f"beam search: {prompts} prompts x width {width}, {steps} fork/prune steps, fp16",
                    {"prompt_lens": lens})


def gqa_long(block_size: int = 16, num_seqs: int = 32, lo: int = 16384, hi: int = 32768) -> Workload:
    geom = Geometry(32, 8, 128, block_size, "bf16")
    rng = _rng(4)
    lens = rng.integers(lo, hi + 1, size=num_seqs)
    need = sum(_blocks(int(L), block_size) for L in lens)
    nb = math.ceil(1.25 * need)
    return _decode_once(geom, lens, 4, f"gqa_long_bs{block_size}", 2004, nb, rng,
                        partition_size=512,
                        description=f"long-context GQA: {num_seqs} seqs, 32 q / 8 kv heads x 128, "
                                    f"bs {block_size}, ctx U[{lo},{hi}], partitions of 512, bf16")


def extend_decode_steps(wl: Workload, steps: int) -> list:
    """Ops for ``steps`` more decode steps over the last attended batch."""
    last = [op for op in wl.ops if op[0] == "attend"][-1][1]
    ops = []
    for _ in range(steps):
        for h in last:
            ops.append(("append", h, 1))
        ops.append(("sync",))
        ops.append(("attend", list(last)))
    return ops


ALL_NAMES = ["tiny", "opt13b", "llama13b_churn", "sharing_A", "sharing_B", "beam",
             "gqa_long_bs16", "gqa_long_bs32"]


def by_name(name: str, **kw) -> Workload:
    if name == "tiny":
        return tiny()
    if name == "opt13b":
        return opt13b(**kw)
    if name == "llama13b_churn":
        return llama13b_churn(**kw)
    if name in ("sharing_A", "sharing_B"):
        return sharing_sampling(name[-1], **kw)
    if name == "beam":
        return beam_search(**kw)
    if name.startswith("gqa_long_bs"):
        return gqa_long(int(name[len("gqa_long_bs"):]), **kw)
    raise KeyError(name)
