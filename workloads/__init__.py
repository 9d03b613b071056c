"""Seeded synthetic workloads shared by the tests and the bench.

This package holds input generation only: sequence-length draws, operation
schedules (create / append / fork / release / sync / attend) and random
q/K/V values as fp16 or bf16 bit patterns. It contains none of the method's
arithmetic - no block allocation, no slot computation, no attention - so
both the fp64 oracle and the CUDA library can be fed from it without sharing
code with each other.

Workload shapes follow the geometries the pages discuss (OPT-13B and
LLaMA-13B: hidden 5120 = 40 heads x 128, block size 16, lengths up to 2,048,
parallel sampling and beam search over shared prompts) plus a long-context
grouped-query case; the datasets the pages measure on are not used, their
length distributions are replaced by the seeded draws documented in
:mod:`workloads.configs`.
"""

from .values import normal_bits, value_seed_words
from .configs import (Geometry, Workload, tiny, opt13b, llama13b_churn, sharing_sampling,
                      beam_search, gqa_long, by_name, ALL_NAMES, extend_decode_steps)

__all__ = [
    "normal_bits", "value_seed_words", "Geometry", "Workload", "tiny", "opt13b",
    "llama13b_churn", "sharing_sampling", "beam_search", "gqa_long", "by_name", "ALL_NAMES",
    "extend_decode_steps",
]
