"""The seeded workload generators: shapes, ranges, determinism, no OOM under the oracle."""

import numpy as np
import pytest

from oracle.replay import OracleReplay
import workloads


def test_values_are_seeded_and_typed():
    a = workloads.normal_bits([1, 2, 3], (4, 5), "f16")
    b = workloads.normal_bits([1, 2, 3], (4, 5), "f16")
    c = workloads.normal_bits([1, 2, 4], (4, 5), "f16")
    assert a.dtype == np.uint16 and np.array_equal(a, b) and not np.array_equal(a, c)
    x = workloads.normal_bits([7], (20000,), "bf16")
    f = (x.astype(np.uint32) << 16).view(np.float32)
    assert abs(f.mean()) < 0.05 and abs(f.std() - 1) < 0.05


def test_tiny_and_opt13b_shapes():
    t = workloads.tiny()
    assert t.info["context_lens"] == [1, 15, 16, 37] and t.num_blocks == 32
    assert sorted(t.free_order.tolist()) == list(range(32))
    o = workloads.opt13b()
    lens = o.info["context_lens"]
    assert len(lens) == 64 and min(lens) >= 1 and max(lens) <= 2048
    need = sum(-(-L // 16) for L in lens)
    assert o.num_blocks == int(np.ceil(1.25 * need))


def test_gqa_long_lengths():
    for bs in (16, 32):
        w = workloads.gqa_long(bs)
        lens = w.info["context_lens"]
        assert len(lens) == 32 and min(lens) >= 16384 and max(lens) <= 32768
        assert w.geometry.num_q_heads == 32 and w.geometry.num_kv_heads == 8
        assert w.partition_size == 512 and w.geometry.dtype == "bf16"


@pytest.mark.parametrize("name", ["llama13b_churn", "sharing_A", "sharing_B", "beam"])
def test_schedules_run_without_oom(name):
    kw = {"steps": 4} if name in ("llama13b_churn", "beam") else {}
    wl = workloads.by_name(name, **kw)
    rp = OracleReplay(wl, with_cache=False)
    rp.run()
    for (_, seqs, tables, lens) in rp.attends:
        assert len(seqs) == {"llama13b_churn": 256, "beam": 32}.get(name, 64)
        assert min(lens) >= 1


def test_churn_replaces_ten_percent():
    wl = workloads.llama13b_churn(steps=2)
    rel = sum(1 for op in wl.ops if op[0] == "release")
    assert rel == 2 * 26
