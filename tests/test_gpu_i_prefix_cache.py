"""Prefix caching end to end on the GPU. Requests share three system prompts; each is
created with kv_seq_create_prefixed, so its leading full blocks are ones an earlier
request wrote (some of those requests already released, their blocks waiting as
evictable), and only its own tokens are scattered with reshape_and_cache. The decode
over the resulting tables - per sequence and grouped - must equal the oracle's
attention over each request's own token history.

Keys and values of a token are a function of (token id, position) - a stand-in for a
model, under which identical prefixes have identical keys and values, which is what
makes reuse valid.
"""

import math

import numpy as np
import pytest

from oracle.attention import attend
from parity import check_close, from_bits, to_bits

pytestmark = pytest.mark.gpu


def test_decode_over_prefixes_reused_across_requests():
    import torch
    import paged_kv_cache_319_b200 as kvp

    Hq = Hkv = 8
    D, bs, NB, vocab, max_pos = 128, 16, 420, 64, 1024
    rng = np.random.default_rng(9)
    kt = rng.standard_normal((vocab, Hkv, D)) * 0.7
    kp = rng.standard_normal((max_pos, Hkv, D)) * 0.7
    vt = rng.standard_normal((vocab, Hkv, D))
    vp = rng.standard_normal((max_pos, Hkv, D)) * 0.5

    def rows(tokens, pos0):  # [T, Hkv, D] fp16 keys and values of tokens at pos0..
        p = np.arange(pos0, pos0 + len(tokens))
        t = np.asarray(tokens)
        return (kt[t] + kp[p]).astype(np.float16), (vt[t] + vp[p]).astype(np.float16)

    pool = kvp.BlockPool(NB, bs, Hkv, D, free_order=rng.permutation(NB))
    pool.set_prefix_caching(True)
    k_cache = torch.zeros((NB, Hkv, bs, D), dtype=torch.float16, device="cuda")
    v_cache = torch.zeros_like(k_cache)
    systems = [rng.integers(0, vocab, size=n).tolist() for n in (100, 250, 530)]
    hist = {}
    for r in range(16):
        prompt = systems[r % 3] + rng.integers(0, vocab, size=int(rng.integers(5, 60))).tolist()
        s, cached = pool.create_prefixed(prompt)
        slots = pool.append_tokens(s, prompt[cached:])
        k_new, v_new = rows(prompt[cached:], cached)
        kvp.reshape_and_cache(torch.from_numpy(k_new).cuda(), torch.from_numpy(v_new).cuda(),
                              k_cache, v_cache, torch.tensor(slots, dtype=torch.int64, device="cuda"))
        hist[s] = prompt
        if r in (2, 4, 7):  # finished requests: their registered blocks become evictable
            pool.release(s)
            del hist[s]
    assert pool.take_copies() == []
    st = pool.prefix_stats()
    assert st["hit_tokens"] > 2000 and st["registered"] > 0
    seqs = sorted(hist)
    mb = max(-(-len(h) // bs) for h in hist.values())
    tables, lens = pool.build_batch(seqs, mb)
    # requests 0 and 3 (the first system prompt) share their leading blocks
    assert tables[seqs.index(0), 0] == tables[seqs.index(3), 0]
    q = rng.standard_normal((len(seqs), Hq, D)).astype(np.float16)
    qb = q.view(np.uint16)
    scale = 1 / math.sqrt(D)
    ref = np.zeros((len(seqs), Hq, D))
    for i, s in enumerate(seqs):
        K, V = rows(hist[s], 0)
        for g in range(Hkv):
            ref[i, g] = attend(q[i, g].astype(np.float64), K[:, g].astype(np.float64),
                               V[:, g].astype(np.float64), scale)
    tt, ll = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    for grouped in (False, True):
        out = kvp.paged_attention_decode(from_bits(qb, "f16"), k_cache, v_cache, tt, ll, scale,
                                         max_context_len=int(lens.max()), partition_size=512,
                                         grouped=grouped,
                                         host_plan=kvp.group_plan(tables, lens, block_size=bs,
                                                                  partition_size=512,
                                                                  num_q_heads=Hq, num_kv_heads=Hkv,
                                                                  num_blocks=NB,
                                                                  max_context_len=int(lens.max()))
                                         if grouped else None)
        kvp.check_device_error()
        check_close(to_bits(out), ref, "f16")
