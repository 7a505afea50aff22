"""fp64 CPU oracle for fused QK RoPE + paged KV cache + ragged GQA attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product package. See rpk_oracle.c
for the definitions and the passages of the pages each one follows.
"""

from .oracle import (  # noqa: F401
    BF16, E4M3, F32, attention, attention_backward, band, bf16_bits_to_f64, cache_image, e4m3_to_f64,
    f64_to_bf16_bits, f64_to_e4m3, flash_step, freqs_cis, freqs_cis_proportional, lib, rope,
    round_to, visible, widen,
)
