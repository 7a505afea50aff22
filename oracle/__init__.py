"""fp64 CPU oracle for fused QK RoPE + paged KV cache + ragged GQA attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product package. See rpk_oracle.c
for the definitions and the passages of the pages each one follows.
"""

from .oracle import (  # noqa: F401
    F32, BF16, attention, band, bf16_bits_to_f64, cache_image, f64_to_bf16_bits,
    flash_step, freqs_cis, freqs_cis_proportional, rope, round_to, visible, widen, lib,
)
