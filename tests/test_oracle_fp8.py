"""Pins of the FP8 KV-cache oracle (oracle/fp8.py) against facts it does not derive
itself: the E4M3 values torch's float8_e4m3fn type decodes, torch's own fp32 -> E4M3
cast on in-range values, hand-worked codes (unit, largest, smallest normal and
subnormal, a division by 3), ties to even at every midpoint, saturation, and
attention identities (a key scale acts like a query scale; a value scale scales the
output; the result equals torch fp64 SDPA on the dequantised cache).
"""

import numpy as np
import pytest

from oracle import attention, fp8

torch = pytest.importorskip("torch")


def torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_decode_matches_torch_e4m3fn_for_all_codes():
    c = np.arange(256, dtype=np.uint8)
    ours, ref = fp8.decode(c), torch_decode(c)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(ref[fin]))


def test_hand_worked_codes():
    d = fp8.decode(np.array([0x00, 0x80, 0x01, 0x07, 0x08, 0x38, 0x3F, 0x40, 0x7E, 0xFE, 0x7F, 0xFF],
                            np.uint8))
    assert d[0] == 0 and not np.signbit(d[0]) and d[1] == 0 and np.signbit(d[1])
    assert d[2] == 2.0**-9 and d[3] == 7 * 2.0**-9 and d[4] == 2.0**-6
    assert d[5] == 1.0 and d[6] == 1.875 and d[7] == 2.0
    assert d[8] == 448.0 and d[9] == -448.0
    assert np.isnan(d[10]) and np.isnan(d[11])
    assert int(np.isnan(fp8.decode(np.arange(256, dtype=np.uint8))).sum()) == 2
    # 1/3 in fp32 is 0.3333333433; the E4M3 neighbours are 0.3125 and 0.34375
    assert fp8.quantize(np.float32(1.0), np.float32(3.0)) == 0x2B
    assert fp8.decode(0x2B) == 0.34375


def test_every_finite_value_round_trips():
    c = np.arange(256, dtype=np.uint8)
    v = fp8.decode(c)
    fin = ~np.isnan(v)
    assert np.array_equal(fp8.encode(v[fin]), c[fin])


def test_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(100_000) * np.exp2(rng.uniform(-14, 9, 100_000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.encode(x), ref)


def test_ties_go_to_the_even_code():
    c = np.arange(0x00, 0x7E, dtype=np.uint8)  # positive finite codes but the largest
    lo, hi = fp8.decode(c), fp8.decode(c + 1)
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # midpoints are exact in fp32
    want = np.where(c % 2 == 0, c, c + 1).astype(np.uint8)
    assert np.array_equal(fp8.encode(mid), want)
    assert np.array_equal(fp8.encode(-mid), want | 0x80)
    # just off the midpoint the nearer code wins
    up = np.nextafter(mid, np.float32(np.inf))
    assert np.array_equal(fp8.encode(up), (c + 1).astype(np.uint8))


def test_saturation_signs_and_nan():
    v = np.array([448, 460, 464, 479.9, 1e6, np.inf, -np.inf, -1e30, np.nan, -0.0, 2.0**-11],
                 np.float32)
    assert fp8.encode(v).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x80, 0x00]
    # subnormal edges: 2^-10 ties to 0, 3 * 2^-10 ties to 2 * 2^-9, 15 * 2^-10 ties up to 2^-6
    assert fp8.encode(np.float32([2.0**-10, 3 * 2.0**-10, 15 * 2.0**-10])).tolist() == [0x00, 0x02, 0x08]


def test_reshape_and_cache_writes_each_head_with_its_scale():
    rng = np.random.default_rng(3)
    T, Hkv, D, bs, NB = 5, 3, 16, 4, 6
    k_new = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    v_new = rng.standard_normal((T, Hkv, D)).astype(np.float32)
    ks, vs = np.float32([0.5, 1.0, 3.0]), np.float32([2.0, 0.25, 1.0])
    slots = [7, -1, 0, 23, 12]
    kc = np.zeros((NB, Hkv, bs, D), np.uint8)
    vc = np.zeros_like(kc)
    fp8.reshape_and_cache(kc, vc, k_new, v_new, slots, bs, ks, vs)
    for t, s in enumerate(slots):
        if s < 0:
            continue
        for g in range(Hkv):
            assert np.array_equal(kc[s // bs, g, s % bs], fp8.encode(k_new[t, g] / ks[g]))
            assert np.array_equal(vc[s // bs, g, s % bs], fp8.encode(v_new[t, g] / vs[g]))
    # slots 7, 0, 23, 12 are blocks 1, 0, 5, 3: blocks 2 and 4 stay untouched
    assert not kc[2].any() and not kc[4].any() and not vc[2].any() and not vc[4].any()


def _fp8_batch(seed, lens, Hq=4, Hkv=2, D=16, bs=4):
    rng = np.random.default_rng(seed)
    need = [-(-L // bs) for L in lens]
    NB = sum(need) + 2
    perm = rng.permutation(NB)
    tables = np.full((len(lens), max(need)), -1, np.int32)
    i = 0
    for s, n in enumerate(need):
        tables[s, :n] = perm[i:i + n]
        i += n
    kc = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
    vc = rng.integers(0, 256, (NB, Hkv, bs, D), dtype=np.uint8)
    # no NaN codes in a cache that quantisation wrote
    kc[(kc & 0x7F) == 0x7F] = 0x3F
    vc[(vc & 0x7F) == 0x7F] = 0x3F
    q = rng.standard_normal((len(lens), Hq, D))
    return q, kc, vc, tables, np.asarray(lens, np.int32)


def test_decode_equals_sdpa_on_the_dequantised_cache():
    q, kc, vc, t, l = _fp8_batch(11, [1, 6, 13])
    ks, vs = np.float32([0.01, 0.02]), np.float32([0.5, 0.125])
    out = fp8.paged_decode(q, kc, vc, t, l, 0.3, 4, ks, vs)
    for s, L in enumerate(l):
        for g in range(2):
            K = torch.from_numpy(fp8.decode(attention.gather(kc, t[s], L, g, 4)) * float(ks[g]))
            V = torch.from_numpy(fp8.decode(attention.gather(vc, t[s], L, g, 4)) * float(vs[g]))
            Q = torch.from_numpy(q[s, 2 * g:2 * g + 2])
            ref = torch.nn.functional.scaled_dot_product_attention(Q[None], K[None], V[None],
                                                                   scale=0.3)[0].numpy()
            assert np.allclose(out[s, 2 * g:2 * g + 2], ref, atol=1e-12, rtol=0)


def test_scales_act_as_the_math_says():
    q, kc, vc, t, l = _fp8_batch(12, [5, 9])
    ks, vs = np.float32([0.01, 0.02]), np.float32([0.5, 0.125])
    base = fp8.paged_decode(q, kc, vc, t, l, 0.3, 4, ks, vs)
    # doubling a key scale is doubling the queries of that KV head's group
    q2 = q.copy()
    q2[:, 0:2] *= 2
    assert np.allclose(fp8.paged_decode(q, kc, vc, t, l, 0.3, 4, ks * np.float32([2, 1]), vs),
                       fp8.paged_decode(q2, kc, vc, t, l, 0.3, 4, ks, vs), atol=1e-12, rtol=0)
    # a value scale multiplies its group's output
    o4 = fp8.paged_decode(q, kc, vc, t, l, 0.3, 4, ks, vs * np.float32([1, 4]))
    assert np.allclose(o4[:, 2:4], 4 * base[:, 2:4], atol=1e-12, rtol=0)
    assert np.array_equal(o4[:, 0:2], base[:, 0:2])
