"""Seeded synthetic inputs for paged decode attention.

This package builds the inputs that both the CUDA path and the CPU oracle
consume: sequence lengths, block tables, slot mappings, copy-on-write pairs,
and the 16-bit bit patterns of q, the K/V block pools and the new tokens.
It holds none of the attention arithmetic; the same bits feed both sides.
"""

from .generate import (  # noqa: F401
    DTYPES,
    NAN_BITS,
    PAD_ENTRY,
    PagedLayout,
    PagedValues,
    f32_to_bits,
    bits_to_torch,
    config_tiny,
    config_llama7b,
    config_llama3_8b,
    config_llama3_8b_prefill,
    config_llama2_70b_shared,
    config_opt13b_long,
    random_layout,
    restrict_layout,
    fill_values_numpy,
    fill_values_torch,
    CONFIGS,
)
