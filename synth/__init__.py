"""Seeded synthetic inputs for cross-model attention-map reuse.

This package holds random draws, bf16 rounding of those draws, and shapes. It holds none of the
method's arithmetic (no logits, no softmax, no block statistics, no mixing): both the float64
oracle and the CUDA path take their inputs from here, and nothing here depends on either.
"""

from .workloads import (  # noqa: F401
    bf16_bits,
    bf16_bits_to_f32,
    bf16_bits_to_f64,
    PrefillWorkload,
    HeadMatchWorkload,
    DecodeWorkload,
    make_prefill,
    make_head_match,
    make_decode,
    PREFILL_CONFIGS,
    prefill_config,
    head_match_config,
    decode_config,
    PrefixWorkload,
    make_prefix_requests,
    prefix_config,
    ChunkWorkload,
    chunk_of,
    make_sender_values,
    select_sequences,
)
