"""paged_attention_prefill: a chunk of T new tokens per sequence, causal within the chunk, against the oracle.

The cases cover chunks that fit one launch (T * G <= 16 columns) and chunks cut
into several launches (a whole prompt), sequences holding fewer tokens than
the chunk (their first queries see nothing), a whole prompt (ctx == T),
grouped-query heads (G = 4 and 16), block sizes 16 and 32, split and unsplit
partitions, launches that stop at the last token their queries see, and T = 1
(the decode path). Chunks of at least 64 query rows (T x G, G a power of two)
run on the prompt-shaped kernel (128 query rows per tensor-core tile): whole
512-token prompts, grouped heads filling the rows (G = 2, 8, 16), a query
tile cut short (inside a warp's 32 rows too), long contexts split or not, and
rows that see nothing.
"""

import math

import numpy as np
import pytest

from oracle import attention
from oracle.numerics import to_f64
from parity import check_close, from_bits, random_paged_batch, to_bits
import workloads

pytestmark = pytest.mark.gpu


def run(q, k, v, tables, lens, dtype, scale, partition):
    import torch
    import paged_kv_cache_319_b200 as kvp

    out = kvp.paged_attention_prefill(
        from_bits(q, dtype), from_bits(k, dtype), from_bits(v, dtype),
        torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda(), scale,
        max_context_len=int(max(lens.max(), 1)), partition_size=partition)
    kvp.check_device_error()
    return to_bits(out)


CASES = [
    # (Hq, Hkv, bs, lens, T, dtype, partition)
    (8, 8, 16, [16, 100, 530, 1100], 16, "f16", 512),    # one launch of 16 columns
    (8, 8, 16, [20, 40, 700, 1500], 40, "f16", 512),     # 16 + 16 + 8 queries; ctx 20 < T
    (4, 4, 32, [100, 100, 333], 100, "bf16", 128),       # whole prompts (ctx == T) and one longer
    (16, 4, 16, [64, 300, 2000], 4, "bf16", 512),        # G = 4: 4 queries per launch
    (16, 4, 16, [9, 300, 1200], 10, "bf16", 0),          # 4 + 4 + 2, unsplit, ctx 9 < T
    (16, 1, 32, [50, 700], 3, "bf16", 256),              # G = 16: one query per launch
    (8, 8, 16, [1, 33, 900], 1, "f16", 512),             # T = 1: decode
    # 13 launches; each reads only the tokens its last query sees, and the
    # reduce merges each row's visible partitions: ctx 150 < T with two
    # partitions (the first 50 rows see nothing), partition boundaries inside
    # the launches' ranges
    (4, 4, 16, [150, 300, 700], 200, "f16", 128),
    (16, 4, 32, [90, 520, 1000], 24, "bf16", 128),       # G = 4: 6 launches of 4 queries
    # prompt-shaped chunks (T x G >= 64 rows): 128 query rows per tensor-core tile
    (8, 8, 16, [512, 512, 512], 512, "f16", 512),        # whole 512-token prompts, 4 tiles each
    (8, 8, 16, [512, 512, 512], 512, "bf16", 512),
    (64, 8, 16, [16, 200, 1000], 16, "bf16", 256),       # G = 8: 16 tokens x 8 heads
    (32, 2, 32, [8, 50, 700], 8, "f16", 0),              # G = 16: 8 tokens x 16 heads, unsplit
    (8, 8, 32, [130, 1000, 2500], 130, "bf16", 512),     # a tile of 128 and one of 2 tokens
    (16, 8, 16, [64, 1500, 3000], 64, "f16", 0),         # G = 2, long contexts unsplit
    (8, 8, 16, [40, 300], 100, "f16", 128),              # ctx 40 < T: 60 rows see nothing
    (4, 4, 16, [1, 129, 1000], 300, "bf16", 128),        # ctx 1 < T; partitions cut the tiles
    # unsplit, last tile cut inside a warp's rows: whole warps store through
    # TMA, the rest row by row
    (8, 8, 16, [200, 900], 200, "f16", 0),               # last tile: 72 tokens
    (16, 4, 16, [72, 1000], 72, "bf16", 0),              # G = 4: last tile 8 tokens x 4 heads
]


@pytest.mark.parametrize("Hq,Hkv,bs,lens,T,dtype,partition", CASES)
def test_prefill_matches_oracle(Hq, Hkv, bs, lens, T, dtype, partition):
    seed = Hq * 1000 + T * 10 + bs
    _, k, v, t, l = random_paged_batch(seed, len(lens), Hq, Hkv, 128, bs, lens, dtype)
    q = workloads.normal_bits([seed, 21], (len(lens), T, Hq, 128), dtype)
    scale = 1 / math.sqrt(128)
    got = run(q, k, v, t, l, dtype, scale, partition)
    ref = attention.paged_prefill(to_f64(q, dtype), k, v, t, l, scale, bs, dtype=dtype)
    check_close(got, ref, dtype, allow_ulp=(dtype == "bf16"))


def test_last_query_of_a_chunk_equals_decode():
    """The chunk's last query sees the whole context: the same row as a decode step."""
    import torch
    import paged_kv_cache_319_b200 as kvp

    lens = [300, 1024, 2000]
    _, k, v, t, l = random_paged_batch(5, 3, 8, 8, 128, 16, lens, "f16")
    q = workloads.normal_bits([5, 22], (3, 8, 8, 128), "f16")
    pre = to_f64(run(q, k, v, t, l, "f16", 0.09, 512), "f16")
    dec = kvp.paged_attention_decode(
        from_bits(q[:, -1].copy(), "f16"), from_bits(k, "f16"), from_bits(v, "f16"),
        torch.from_numpy(t).cuda(), torch.from_numpy(l).cuda(), 0.09,
        max_context_len=int(l.max()), partition_size=512)
    assert np.abs(pre[:, -1] - to_f64(to_bits(dec), "f16")).max() <= 2e-3
