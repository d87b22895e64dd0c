"""Seeded synthetic inputs for the lightning-indexer scoring path.

This package only draws random numbers and lays them out: it holds none of the
indexer's arithmetic (no scoring, no Top-k, no bounds).  Both the CUDA path and
the CPU oracle read the arrays it produces, so that they see identical bits.
"""

from .inputs import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_from_f64,
    bf16_bits_to_f32,
    make_decode,
    make_integer_prefill,
    make_prefill,
    make_prefill_fp8,
    quantize_e4m3_rows,
    random_distinct_keys,
)
