"""The oracle's paged attention against a dense numpy brute force on tiny inputs.

The brute force builds, per sequence, the full score matrix and a dense mask
from NumKong's band rule ("Attention with a Pre-Packed KV-Cache": row r of q
rows over k keys sits at r + k - q and sees keys_before keys before it and
keys_after = 0 after), applies a masked softmax and returns zeros for rows with
no visible key. The paged pools are built here from dense K/V with a shuffled
page assignment, independently of the oracle.
"""

import numpy as np
import pytest

import oracle as O
from test_oracle_pins import paged


def dense_reference(q, k_dense, v_dense, q_lens, scale, window, sinks=0):
    H = q.shape[1]
    Hk = k_dense[0].shape[1]
    G = H // Hk
    out = np.zeros(q.shape, dtype=np.float64)
    lse = np.full(q.shape[:2], -np.inf)
    t0 = 0
    for b, ql in enumerate(q_lens):
        kl = k_dense[b].shape[0]
        rows = np.arange(ql)[:, None]
        keys = np.arange(kl)[None, :]
        pos = rows + kl - ql
        mask = keys <= pos
        if window > 0:
            # the recent window, plus the first `sinks` keys (StreamingLLM)
            mask &= (keys >= pos - (window - 1)) | (keys < sinks)
        for h in range(H):
            qq = q[t0:t0 + ql, h].astype(np.float64)
            kk = k_dense[b][:, h // G].astype(np.float64)
            vv = v_dense[b][:, h // G].astype(np.float64)
            s = scale * (qq @ kk.T)
            s = np.where(mask, s, -np.inf)
            m = s.max(axis=1, keepdims=True) if kl else np.full((ql, 1), -np.inf)
            has = np.isfinite(m[:, 0])
            w = np.zeros_like(s)
            w[has] = np.exp(s[has] - m[has])
            w[has] /= w[has].sum(axis=1, keepdims=True)
            out[t0:t0 + ql, h] = w @ vv if kl else 0.0
            # log-sum-exp straight from its definition (the scores are small)
            with np.errstate(divide="ignore"):
                lse[t0:t0 + ql, h] = np.log(np.where(mask, np.exp(s), 0.0).sum(axis=1))
        t0 += ql
    return out, lse


CASES = [
    # (q_lens, kv_lens, H, Hk, d, page, window, sinks)
    ([5, 11], [5, 11], 4, 2, 16, 4, 0, 0),
    ([1, 1, 1], [7, 1, 19], 4, 1, 8, 4, 0, 0),
    ([3, 8, 2], [10, 8, 20], 6, 3, 8, 3, 0, 0),
    ([6, 9], [6, 20], 2, 2, 8, 4, 4, 0),
    ([4, 1], [2, 3], 2, 1, 4, 2, 0, 0),          # rows with no key
    ([12], [12], 8, 2, 16, 5, 1, 0),             # window 1: only itself
    ([7, 0, 5], [7, 4, 15], 4, 4, 8, 4, 3, 0),   # an empty sequence
    ([6, 9], [6, 20], 2, 2, 8, 4, 4, 2),         # window 4 with 2 sinks
    ([12, 1], [12, 30], 4, 2, 8, 5, 1, 3),       # window 1 with 3 sinks
    ([3, 2], [3, 25], 2, 1, 8, 4, 5, 0),
    ([2, 5], [40, 9], 2, 1, 8, 4, 5, 7),         # sinks reaching into the window
]


@pytest.mark.parametrize("idx", range(len(CASES)))
def test_oracle_matches_dense_bruteforce(idx):
    q_lens, kv_lens, H, Hk, d, P, w, sinks = CASES[idx]
    rng = np.random.default_rng(100 + idx)
    k = [rng.normal(size=(n, Hk, d)).astype(np.float32) for n in kv_lens]
    v = [rng.normal(size=(n, Hk, d)).astype(np.float32) for n in kv_lens]
    T = sum(q_lens)
    q = rng.normal(size=(T, H, d)).astype(np.float32)
    kp, vp, bt = paged(k, v, page_size=P, seed=len(q_lens))
    offs = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    scale = 1.0 / np.sqrt(d)
    got, got_lse = O.attention(q, offs, kv_lens, kp, vp, bt, Hk, scale, w, n_threads=2,
                               with_lse=True, sinks=sinks)
    want, want_lse = dense_reference(q, k, v, q_lens, scale, w, sinks)
    assert np.max(np.abs(got - want)) < 1e-12
    assert np.array_equal(np.isinf(got_lse), np.isinf(want_lse))
    fin = np.isfinite(want_lse)
    assert np.max(np.abs(got_lse[fin] - want_lse[fin]), initial=0.0) < 1e-12
