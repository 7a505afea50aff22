"""Algorithmic work of one call: bytes and FLOPs that the roofline counts.

Host-side accounting only (numpy over the per-sequence lengths); nothing here
runs on the data path.
"""

from __future__ import annotations

import numpy as np


def kv_cache_bytes(layers: int, heads: int, head_dim: int, seq_len: int, batch: int,
                   bytes_per_elt: int) -> int:
    """K and V footprint of a dense cache: 2 * layers * heads * d * seq * batch * elt.

    The formula of algenta's kv_cache_memory_bytes ("Attention variant kernels",
    transformer_attention module); 32 layers, 32 heads, d 128, 4096 tokens,
    batch 1 and 2-byte elements give 2147483648 bytes.
    """
    return 2 * layers * heads * head_dim * seq_len * batch * bytes_per_elt


def _bands(q_len: int, kv_len: int, window: int):
    """(lo, hi) arrays of the visible keys of each row (hi < lo: none).

    Row r sits at p = r + kv_len - q_len and sees keys [p - (w - 1), p] under a
    window w > 0, else [0, p] (NumKong "Attention with a Pre-Packed KV-Cache").
    """
    r = np.arange(q_len, dtype=np.int64)
    p = r + kv_len - q_len
    lo = np.maximum(p - (window - 1), 0) if window > 0 else np.zeros_like(p)
    hi = np.minimum(p, kv_len - 1)
    return lo, hi


def visible_pairs(q_lens, kv_lens, window: int) -> int:
    """Number of (query row, key) pairs inside the band, summed over sequences."""
    total = 0
    for ql, kl in zip(np.asarray(q_lens), np.asarray(kv_lens)):
        if ql <= 0:
            continue
        lo, hi = _bands(int(ql), int(kl), window)
        total += int(np.maximum(hi - lo + 1, 0).sum())
    return total


def keys_read(q_lens, kv_lens, window: int) -> int:
    """Keys of each sequence that any of its rows sees (each counted once)."""
    total = 0
    for ql, kl in zip(np.asarray(q_lens), np.asarray(kv_lens)):
        if ql <= 0:
            continue
        lo, hi = _bands(int(ql), int(kl), window)
        ok = hi >= lo
        if ok.any():
            total += int(hi[ok].max() - lo[ok].min() + 1)
    return total


def attention_kv_bytes(q_lens, kv_lens, window: int, n_kv_heads: int, head_dim: int,
                       elt_bytes: int) -> int:
    """K and V bytes attention must read: every visible key once per KV head."""
    return keys_read(q_lens, kv_lens, window) * n_kv_heads * head_dim * 2 * elt_bytes


def attention_flops(q_lens, kv_lens, window: int, n_heads: int, head_dim: int) -> int:
    """2 * d FLOPs for q.k and 2 * d for p * v, per visible pair and query head."""
    return 4 * n_heads * head_dim * visible_pairs(q_lens, kv_lens, window)


def rope_bytes(total_tokens: int, n_heads: int, n_kv_heads: int, head_dim: int,
               rotary_dim: int, elt_bytes: int) -> int:
    """Bytes the RoPE + scatter step moves: read q, k_new, v_new; write out_q and
    the K and V cache rows; one fp32 (cos, sin) table row per token."""
    per_token = (2 * n_heads * head_dim + 4 * n_kv_heads * head_dim) * elt_bytes
    return total_tokens * (per_token + rotary_dim * 4)
