"""The five workloads end to end on the GPU (host allocator + all kernels) against the oracle.

Every workload runs at its configured size and schedule, in the launch
configuration the bench uses (partitions of 512 tokens). The library and the
oracle replay the schedule in lockstep, one decode step at a time:

* bookkeeping (every slot, copy pair, block table and length) is compared
  bit for bit at every operation;
* the K and V pools are compared at every step through a fingerprint of each
  physical block (the sum of its 16-bit words weighted by 2i + 1, exact in
  int64): the device fingerprints every block, the oracle refreshes the blocks
  it wrote that step (copy destinations, the blocks of the step's slots), so a
  write that lands anywhere else also shows; at the end the pools are compared
  bit for bit;
* attention outputs are compared on every row (every sequence, every head)
  against the fp64 oracle: every attend of the small workloads, the one attend
  of OPT-13B, long-context GQA, sampling and beam search, and the first, every
  fourth and the last of the 32 churn steps.

Both sides take the seeded K/V draws of a step from one computation (the draws
depend only on the workload's value seed and the op index).
"""

import concurrent.futures as cf

import numpy as np
import pytest

from oracle.replay import OracleReplay
from parity import check_close, to_bits
import workloads

pytestmark = pytest.mark.gpu


def fingerprint_host(pool_bits: np.ndarray, blocks) -> np.ndarray:
    """Per block: sum over its 16-bit words w_i of w_i * (2i + 1) (no overflow:
    below 2^16 * n^2 with n words per block)."""
    n = int(np.prod(pool_bits.shape[1:]))
    wts = np.arange(n, dtype=np.uint64) * np.uint64(2) + np.uint64(1)
    out = np.empty(len(blocks), dtype=np.uint64)
    for i, b in enumerate(blocks):
        out[i] = (pool_bits[b].reshape(-1).astype(np.uint64) * wts).sum(dtype=np.uint64)
    return out


def fingerprint_device(cache, chunk=256) -> np.ndarray:
    import torch

    nb = cache.shape[0]
    n = cache[0].numel()
    wts = torch.arange(n, dtype=torch.int64, device=cache.device) * 2 + 1
    flat = cache.reshape(nb, n).view(torch.int16)
    out = torch.empty(nb, dtype=torch.int64, device=cache.device)
    for b0 in range(0, nb, chunk):
        x = (flat[b0:b0 + chunk].to(torch.int32) & 0xFFFF).to(torch.int64)
        out[b0:b0 + chunk] = (x * wts).sum(dim=1)
    return out.cpu().numpy().view(np.uint64)


class Lockstep:
    """Device and oracle replays advanced one step (ops up to a sync) at a time."""

    def __init__(self, wl, grouped=False, check_rows=lambda step: True, packed=False):
        from paged_kv_cache_319_b200.replay import DeviceReplay

        self.wl = wl
        self.dev = DeviceReplay(wl, "cuda", grouped=grouped, packed=packed)
        self.ora = OracleReplay(wl)
        self._values = {}
        draw = self.ora.kv_values  # the seeded draw of op j, before it is shared
        self._draw = draw
        self.dev.kv_values = self.ora.kv_values = lambda j, n: self._values[j]
        nb = wl.num_blocks
        self.fk = np.zeros(nb, np.uint64)   # oracle fingerprints (zero pools: all 0)
        self.fv = np.zeros(nb, np.uint64)
        self.check_rows = check_rows
        self.refs = {}                      # attend op index -> fp64 reference
        self.steps = 0
        self.attend_count = 0

    def _on_attend(self, i, seqs, tables, lens):
        if self.check_rows(self.attend_count):
            self.refs[i] = self.ora.decode(i, tables, lens.tolist())
        self.attend_count += 1

    def run(self):
        import paged_kv_cache_319_b200 as kvp

        ops = self.wl.ops
        bs = self.wl.geometry.block_size
        i = 0
        with cf.ThreadPoolExecutor(16) as ex:
            while i < len(ops):
                j = i
                while j < len(ops) and ops[j][0] != "sync":
                    j += 1
                step = ops[i:j + 1]
                apps = [(i + k, op[2]) for k, op in enumerate(step) if op[0] == "append" and op[2]]
                for (idx, _), kv in zip(apps, ex.map(lambda a: self._draw(*a), apps)):
                    self._values[idx] = kv
                ev0 = len(self.ora.events)
                self.dev.run(step, start_index=i)
                self.ora.run(step, attend=self._on_attend, start_index=i)
                self._values.clear()
                if step[-1][0] == "sync":
                    self._check_pools(ev0, bs)
                i = j + 1
        kvp.check_device_error()

    def _check_pools(self, ev0, bs):
        touched = set()
        for (_, kind, payload) in self.ora.events[ev0:]:
            if kind == "append":
                touched.update(int(s) // bs for s in payload)
            elif kind == "sync":
                touched.update(int(d) for _, d in payload)
        blocks = sorted(touched)
        if blocks:
            self.fk[blocks] = fingerprint_host(self.ora.k_cache, blocks)
            self.fv[blocks] = fingerprint_host(self.ora.v_cache, blocks)
        assert np.array_equal(fingerprint_device(self.dev.k_cache), self.fk), f"K pool, step {self.steps}"
        assert np.array_equal(fingerprint_device(self.dev.v_cache), self.fv), f"V pool, step {self.steps}"
        self.steps += 1


def replay_pair(wl, grouped=False, packed=False):
    """Both sides replayed in lockstep, every attend compared in full."""
    ls = Lockstep(wl, grouped=grouped, packed=packed)
    ls.run()
    return ls.dev, ls.ora, ls.refs


def bookkeeping_equal(dev, ora):
    assert len(dev.events) == len(ora.events)
    for (i, k, a), (j, k2, b) in zip(dev.events, ora.events):
        assert (i, k) == (j, k2)
        if k in ("append", "sync"):
            assert [tuple(x) if isinstance(x, tuple) else x for x in a] == \
                   [tuple(x) if isinstance(x, tuple) else x for x in b], (i, k)
    for (i, s, t, l), (j, s2, t2, l2) in zip(dev.attends, ora.attends):
        assert i == j and s == s2 and np.array_equal(t, np.asarray(t2)) and l.tolist() == l2


def pools_equal(dev, ora):
    assert np.array_equal(to_bits(dev.k_cache), ora.k_cache)
    assert np.array_equal(to_bits(dev.v_cache), ora.v_cache)


def test_pool_fingerprint_sees_a_swap_inside_a_block():
    # the fingerprint is position-weighted: two words exchanged within a block change it
    rng = np.random.default_rng(5)
    pool = rng.integers(0, 1 << 16, size=(3, 2, 16, 8), dtype=np.uint16)
    f0 = fingerprint_host(pool, [0, 1, 2])
    pool[1, 0, 3, 2], pool[1, 1, 7, 5] = pool[1, 1, 7, 5], pool[1, 0, 3, 2]
    if pool[1, 0, 3, 2] != pool[1, 1, 7, 5]:
        f1 = fingerprint_host(pool, [0, 1, 2])
        assert f1[0] == f0[0] and f1[2] == f0[2] and f1[1] != f0[1]


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("sharing_A", {}), ("sharing_B", {}),
                                     ("beam", {})])
def test_small_workloads_every_output(name, kw):
    wl = workloads.by_name(name, **kw)
    dev, ora, refs = replay_pair(wl)
    bookkeeping_equal(dev, ora)
    pools_equal(dev, ora)
    assert refs
    for i, ref in refs.items():
        check_close(to_bits(dev.outputs[i]), ref, wl.geometry.dtype)


@pytest.mark.parametrize("decode", ["grouped", "packed"])
@pytest.mark.parametrize("name", ["sharing_A", "sharing_B", "beam"])
def test_shared_workloads_grouped_every_output(name, decode):
    # forked sequences through the entry points that read shared blocks once per group
    wl = workloads.by_name(name)
    dev, ora, refs = replay_pair(wl, grouped=decode == "grouped", packed=decode == "packed")
    bookkeeping_equal(dev, ora)
    pools_equal(dev, ora)
    assert refs
    for i, ref in refs.items():
        check_close(to_bits(dev.outputs[i]), ref, wl.geometry.dtype)


def test_sharing_b_made_the_expected_copies():
    wl = workloads.sharing_sampling("B")
    dev, _, _ = replay_pair(wl)
    copies = [p for (_, k, payload) in dev.events if k == "sync" for p in payload]
    assert len(copies) == 8 * 7
    st = dev.pool.stats()
    assert st["cow_copies_total"] == 56 and st["num_shared"] >= 8 * 31


def test_opt13b_full_size_every_row():
    wl = workloads.opt13b()
    dev, ora, refs = replay_pair(wl)
    bookkeeping_equal(dev, ora)
    pools_equal(dev, ora)
    (i, ref), = refs.items()
    err, rel = check_close(to_bits(dev.outputs[i]), ref, "f16")
    assert err < 2e-3


def test_llama13b_churn_32_steps():
    wl = workloads.llama13b_churn()  # the configured 32 steps
    n_att = sum(1 for op in wl.ops if op[0] == "attend")
    assert n_att == 32
    ls = Lockstep(wl, check_rows=lambda k: k % 4 == 0 or k == n_att - 1)
    ls.run()
    assert ls.steps >= 32
    bookkeeping_equal(ls.dev, ls.ora)
    pools_equal(ls.dev, ls.ora)
    assert len(ls.refs) == 9
    for i, ref in ls.refs.items():
        check_close(to_bits(ls.dev.outputs[i]), ref, "f16")


@pytest.mark.parametrize("bs", [16, 32])
def test_gqa_long_full_size_every_row(bs):
    wl = workloads.gqa_long(bs)
    dev, ora, refs = replay_pair(wl)
    bookkeeping_equal(dev, ora)
    pools_equal(dev, ora)
    (i, ref), = refs.items()
    err, rel = check_close(to_bits(dev.outputs[i]), ref, "bf16")
    assert err < 2e-3
