"""The roofline accounting (ragged_paged_kv_rope_b200.metrics) against brute force.

The benchmark divides these counts by kernel time, so they are product claims:
visible (row, key) pairs and the keys attention must read are counted here
key by key with the oracle's visibility rule (NumKong "Attention with a
Pre-Packed KV-Cache": row r of a sequence with q_len rows and k_len keys sits
at p = r + k_len - q_len and sees keys [p - (w - 1), p] under a window w,
else [0, p]), on small ragged cases that include empty sequences, rows that
see no key and windows wider than the context.
"""

import numpy as np
import pytest

import oracle as O
from ragged_paged_kv_rope_b200 import metrics as M

CASES = [
    ([1, 1, 1], [5, 1, 40], 0),
    ([7, 3], [7, 10], 0),
    ([12, 4], [5, 30], 0),          # the first sequence's first rows see no key
    ([9, 0, 6], [20, 3, 6], 4),
    ([5, 8], [60, 8], 100),          # window wider than the context
    ([16], [16], 1),
    ([3, 2, 1], [50, 17, 9], 7),
]


def _brute(q_lens, kv_lens, window):
    pairs, keys = 0, 0
    for ql, kl in zip(q_lens, kv_lens):
        seen = set()
        for r in range(ql):
            for j in range(kl):
                if O.visible(r, ql, kl, window, 0, j):
                    pairs += 1
                    seen.add(j)
        keys += len(seen)
    return pairs, keys


@pytest.mark.parametrize("q_lens,kv_lens,window", CASES)
def test_visible_pairs_and_keys_read_match_brute_force(q_lens, kv_lens, window):
    pairs, keys = _brute(q_lens, kv_lens, window)
    assert M.visible_pairs(q_lens, kv_lens, window) == pairs
    assert M.keys_read(q_lens, kv_lens, window) == keys


def test_random_cases_match_brute_force():
    rng = np.random.default_rng(7)
    for _ in range(20):
        B = int(rng.integers(1, 4))
        q = rng.integers(0, 9, size=B)
        k = q + rng.integers(0, 12, size=B)
        w = int(rng.choice([0, 1, 3, 8, 30]))
        pairs, keys = _brute(list(q), list(k), w)
        assert M.visible_pairs(q, k, w) == pairs
        assert M.keys_read(q, k, w) == keys


def test_flops_and_bytes_scale_the_counts():
    q, k, w = [7, 3], [7, 10], 0
    pairs, keys = _brute(q, k, w)
    assert M.attention_flops(q, k, w, n_heads=8, head_dim=64) == 4 * 8 * 64 * pairs
    assert M.attention_kv_bytes(q, k, w, n_kv_heads=2, head_dim=64, elt_bytes=2) == \
        keys * 2 * 64 * 2 * 2


def test_decode_reads_every_cached_key_once():
    # one new token per sequence, no window: every key of every sequence, once
    kv = [512, 8192, 1000]
    assert M.keys_read([1, 1, 1], kv, 0) == sum(kv)
    assert M.visible_pairs([1, 1, 1], kv, 0) == sum(kv)


def test_rope_bytes_hand_count():
    # one token, H 4, Hk 2, d 8, R 8, bf16: read q (64 B), k and v (32 B each);
    # write out_q (64 B), K and V rows (32 B each); one fp32 table row (32 B)
    assert M.rope_bytes(1, 4, 2, 8, 8, 2) == 64 + 32 + 32 + 64 + 32 + 32 + 32
