"""Pins of the capacity / waste model against the numbers the pages print."""

import json
import os

from oracle import capacity

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_size_worked_example.json")


def load():
    with open(GOLDEN) as f:
        return json.load(f)


def test_opt13b_per_token_bytes_is_800_kib():
    g = load()["opt13b"]
    b = capacity.kv_bytes_per_token(g["hidden"], g["layers"], g["bytes_per_value"])
    assert b == g["per_token_bytes"] == 800 * 1024
    # "800 KB" as printed is this figure in KiB.
    assert round(b / 1024) == 800


def test_per_sequence_figures_round_to_printed_values():
    g = load()
    o, l = g["opt13b"], g["llama13b"]
    b_opt = capacity.kv_bytes_per_sequence(o["sequence_tokens"], o["hidden"], o["layers"],
                                           o["bytes_per_value"])
    assert round(b_opt / 1e9, 1) == o["sequence_gb_approx"]
    b_llama = capacity.kv_bytes_per_sequence(l["sequence_tokens_reading"], l["hidden"], l["layers"],
                                             l["bytes_per_value"])
    assert round(b_llama / 1e9, 1) == l["sequence_gb_approx"]


def test_paged_waste_bound_is_block_size_minus_one():
    g = load()["paging"]
    bs = g["block_size"]
    wastes = [capacity.paged_waste_slots(n, bs) for n in range(1, 5000)]
    assert min(wastes) == 0
    assert max(wastes) == g["max_waste_slots_printed"] == bs - 1
    # A full block wastes nothing; one token into a new block wastes bs-1.
    assert capacity.paged_waste_slots(32, bs) == 0
    assert capacity.paged_waste_slots(33, bs) == bs - 1


def test_slab_waste_worked_example():
    g = load()["slab"]
    frac = capacity.slab_waste_fraction(g["output_tokens"], g["reserved_tokens"])
    assert int(frac * 100) == round(g["waste_fraction_approx"] * 100)


def test_block_bytes_and_resident_sequences():
    # One OPT-13B layer block (40 heads x 16 slots x 128 dims, K and V, fp16): 320 KiB.
    assert capacity.block_bytes(40, 16, 128, 2) == 320 * 1024
    # With the per-token figure over all 40 layers, a 12 GB budget holds
    # floor(12e9 / (ceil(2000/16) * 16 * 819200)) sequences of 2,000 tokens.
    per_tok = capacity.kv_bytes_per_token(5120, 40, 2)
    n = capacity.max_resident_sequences(12 * 10**9, 2000, 16, per_tok)
    assert n == 12 * 10**9 // (125 * 16 * per_tok) == 7
    # Rounding up to whole blocks matters: 2,001 tokens need one more block.
    assert capacity.blocks_for(2001, 16) == 126
