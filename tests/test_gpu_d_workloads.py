"""The five workloads end to end on the GPU (host allocator + all kernels) against the oracle.

Small workloads are compared on every attention output and the final K/V
pools bit for bit. Full-size workloads run in the launch configuration the
bench uses (partitions of 512 tokens) and are compared on sampled sequences
(every head of each), plus the pools bit for bit.
"""

import numpy as np
import pytest

from oracle.replay import OracleReplay
from parity import check_close, to_bits
import workloads

pytestmark = pytest.mark.gpu


def replay_pair(wl, rows_of=None):
    """Runs both sides. The oracle decodes each attend op when it happens (later
    steps may reuse released blocks), on the rows ``rows_of(lens)`` (default: all);
    the references are returned by op index."""
    from paged_kv_cache_319_b200.replay import DeviceReplay
    import paged_kv_cache_319_b200 as kvp

    dev = DeviceReplay(wl, "cuda")
    dev.run()
    kvp.check_device_error()
    ora = OracleReplay(wl)
    refs = {}

    def on_attend(i, seqs, tables, lens):
        rows = None if rows_of is None else rows_of(lens)
        refs[i] = (rows, ora.decode(i, tables, lens.tolist(), seqs=rows))

    ora.run(attend=on_attend)
    return dev, ora, refs


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


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("sharing_A", {}), ("sharing_B", {}),
                                     ("beam", {"steps": 16})])
def test_small_workloads_every_output(name, kw):
    wl = workloads.by_name(name, **kw)
    dev, ora, refs = replay_pair(wl)
    bookkeeping_equal(dev, ora)
    pools_equal(dev, ora)
    assert refs
    for i, (rows, ref) in refs.items():
        check_close(to_bits(dev.outputs[i]), ref, wl.geometry.dtype)


def test_sharing_b_made_the_expected_copies():
    wl = workloads.sharing_sampling("B")
    dev, _, _ = replay_pair(wl)
    copies = [p for (_, k, payload) in dev.events if k == "sync" for p in payload]
    assert len(copies) == 8 * 7
    st = dev.pool.stats()
    assert st["cow_copies_total"] == 56 and st["num_shared"] >= 8 * 31


def sampled(lens, n=6):
    lens = np.asarray(lens)
    order = np.argsort(lens)
    pick = {int(order[0]), int(order[-1])}
    rng = np.random.default_rng(0)
    pick |= set(rng.choice(len(lens), size=min(n, len(lens)), replace=False).tolist())
    return sorted(pick)


def test_opt13b_full_size():
    wl = workloads.opt13b()
    dev, ora, refs = replay_pair(wl, lambda l: sampled(l, 8))
    bookkeeping_equal(dev, ora)
    pools_equal(dev, ora)
    (i, (rows, ref)), = refs.items()
    err, rel = check_close(to_bits(dev.outputs[i]), ref, "f16", rows=rows)
    assert err < 2e-3


def test_llama13b_churn():
    wl = workloads.llama13b_churn(steps=4)
    dev, ora, refs = replay_pair(wl, lambda l: sampled(l, 6))
    bookkeeping_equal(dev, ora)
    pools_equal(dev, ora)
    assert len(refs) == 4
    for i, (rows, ref) in refs.items():
        check_close(to_bits(dev.outputs[i]), ref, "f16", rows=rows)


@pytest.mark.parametrize("bs", [16, 32])
def test_gqa_long_full_size(bs):
    wl = workloads.gqa_long(bs)
    dev, ora, refs = replay_pair(wl, lambda l: sampled(l, 2))
    bookkeeping_equal(dev, ora)
    (i, (rows, ref)), = refs.items()
    err, rel = check_close(to_bits(dev.outputs[i]), ref, "bf16", rows=rows)
    assert err < 2e-3
