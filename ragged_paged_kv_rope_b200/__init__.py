"""Fused QK RoPE into a paged KV cache + ragged causal GQA attention on B200.

The compute path is the C-ABI library ``librpk.so`` (hand-written sm_100a
CUDA kernels, declared in ``include/rpk.h``). This package is the thin Python
binding over it (argument marshalling only) plus host-side helpers:

* ``binding``   -- ctypes binding with the same entry-point names as the C ABI
* ``workloads`` -- seeded synthetic inputs (no method arithmetic)
* ``metrics``   -- algorithmic bytes / FLOPs for roofline accounting
* ``build``     -- nvcc build of the library for sm_100a

There is no CPU fallback: calling an entry point without the built library or
without a CUDA device raises.
"""

from .binding import (  # noqa: F401
    PagedKVCache,
    RpkError,
    freqs_cis,
    freqs_cis_proportional,
    lib,
    ragged_paged_attention,
    ragged_paged_attention_backward,
    ragged_paged_attention_workspace_size,
    rope_qk_paged_ragged,
    set_wait_limit_ns,
    wait_limit_ns,
)
