"""Pins of oracle/numerics.py: bit decoding and the half-ulp tolerance widening.

``half_ulp`` widens the tolerance of the small bf16 edge cases by half a unit
in the last place of the reference. It is pinned here against what the
formats fix, not against its own formula: hand-worked values, and, for every
positive finite bit pattern, half the gap to the next representable value
(found by incrementing the pattern, as IEEE 754 orders positive floats by
their bits). A slip such as the wrong mantissa width or a whole ulp instead of
half fails these.
"""

import numpy as np
import pytest

from oracle.numerics import half_ulp, to_f64


@pytest.mark.parametrize("dtype,x,want", [
    ("bf16", 1.0, 2.0**-8),      # 7 stored mantissa bits: ulp 2^-7 on [1, 2)
    ("bf16", 1.5, 2.0**-8),
    ("bf16", 3.0, 2.0**-7),      # [2, 4): ulp 2^-6
    ("bf16", 0.25, 2.0**-10),    # [2^-2, 2^-1): ulp 2^-9
    ("bf16", -1.0, 2.0**-8),     # by magnitude
    ("bf16", 448.0, 2.0**0),     # [256, 512): ulp 2
    ("f16", 1.0, 2.0**-11),      # 10 stored mantissa bits: ulp 2^-10 on [1, 2)
    ("f16", 3.0, 2.0**-10),      # [2, 4): ulp 2^-9
    ("f16", 0.5, 2.0**-12),
    ("f16", 1000.0, 2.0**-2),    # [512, 1024): ulp 2^-1
    ("f16", 2.0**-14, 2.0**-25), # smallest normal: ulp 2^-24
    ("f16", 1e-6, 2.0**-25),     # subnormals share the spacing 2^-24
])
def test_half_ulp_hand_values(dtype, x, want):
    assert float(half_ulp(np.array([x]), dtype)[0]) == want


def _neighbour_half_gaps(dtype, lo_exp):
    """(values, half gaps to the next value above) for every positive finite
    pattern with exponent field >= lo_exp, the largest finite excluded."""
    if dtype == "f16":
        exp_bits, mant = 5, 10
    else:
        exp_bits, mant = 8, 7
    max_exp = (1 << exp_bits) - 1
    bits = np.arange(1, 1 << 15, dtype=np.uint32)
    e = bits >> mant
    keep = (e >= lo_exp) & (e < max_exp)
    bits = bits[keep]
    nxt = bits + 1
    keep = (nxt >> mant) < max_exp          # the next pattern must be finite too
    bits, nxt = bits[keep], nxt[keep]
    x = to_f64(bits.astype(np.uint16), dtype)
    y = to_f64(nxt.astype(np.uint16), dtype)
    return x, (y - x) / 2


def test_half_ulp_equals_half_the_gap_to_the_next_fp16_value_everywhere():
    x, gap = _neighbour_half_gaps("f16", 0)  # subnormals included
    assert len(x) > 30000
    assert np.array_equal(half_ulp(x, "f16"), gap)


def test_half_ulp_equals_half_the_gap_to_the_next_bf16_value_in_its_range():
    # the stated domain: magnitudes from 2^-14 (exponent field 127 - 14) up
    x, gap = _neighbour_half_gaps("bf16", 127 - 14)
    assert len(x) > 10000
    assert np.array_equal(half_ulp(x, "bf16"), gap)
    # below it the widening is clamped: still at least the true half gap
    x2, gap2 = _neighbour_half_gaps("bf16", 1)
    small = x2 < 2.0**-14
    assert small.any()
    assert np.all(half_ulp(x2[small], "bf16") >= gap2[small])


def test_half_ulp_is_the_rounding_radius_of_a_cast():
    # a value less than half an ulp above a representable x rounds back to x;
    # one just above x + half ulp rounds away (fp16 by NumPy's own cast)
    x, gap = _neighbour_half_gaps("f16", 1)
    h = half_ulp(x, "f16")
    inside = (x + 0.999 * h).astype(np.float16).astype(np.float64)
    outside = (x + 1.001 * h).astype(np.float16).astype(np.float64)
    assert np.array_equal(inside, x)
    assert np.all(outside > x)


def test_to_f64_decodes_hand_patterns():
    assert to_f64(np.array([0x3C00, 0xC000, 0x0001, 0x7BFF], np.uint16), "f16").tolist() == \
        [1.0, -2.0, 2.0**-24, 65504.0]
    assert to_f64(np.array([0x3F80, 0xC040, 0x0080, 0x3EAB], np.uint16), "bf16").tolist() == \
        [1.0, -3.0, 2.0**-126, 0.333984375]
