"""Full-size parity: the launches the benchmark times, checked against the oracle.

* Ragged causal prefill (16 sequences, 34069 tokens, 32 query heads): every one
  of its 1 090 208 (token, query head) rows and their log-sum-exp.
* Mixed chunked M-RoPE prefill (32 sequences, 64 query heads over 8 KV heads):
  every token of one query head per KV head (the head moves through the group
  with the KV head, so all eight positions of a group are covered), which
  reaches every 128-row query tile of every (sequence, KV head).
* The same mixed workload end to end at full size: GPU table, RoPE with the
  M-RoPE sections and position gaps, the paged scatter and attention, against
  the oracle's chain; RoPE on every Q row, the cache image bit for bit where
  the method fixes it, attention on one row of every 128-row query tile of
  every (sequence, KV head) plus the last row of each.
* The attention backward on the full ragged prefill batch: the query, key and
  value gradients of its two shortest sequences in full, and the query
  gradients of 256 tokens of its longest sequence (each token's gradient is
  computed by the oracle as a one-token sequence with the same keys, since a
  row's query gradient depends only on that row and its visible keys).

Tolerances are those of every other parity test (bf16 attention max-abs 2e-2,
mean-abs 2e-3; gradients relative to their largest magnitude).
"""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import (check_attention, check_lse, check_rope, gather_logical, new_token_slots,
                    oracle_rope, oracle_table, raw_bits, to_device)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _gpu_attention(wl, dev, q, lse=None):
    sp = wl.spec
    out = torch.empty_like(q)
    R.ragged_paged_attention(q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads, sp.n_kv_heads,
                             sp.head_dim, sp.softmax_scale, sp.window, out,
                             max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len, log_sum_exp=lse)
    return out


def test_ragged_prefill_every_row():
    sp = W.SPECS["ragged_prefill"]
    src = W.make(sp, seed=0)
    wl = W.attention_only(sp, 0, src.q_lens, src.kv_lens)
    dev = to_device(wl)
    lse = torch.full((wl.total_tokens, sp.n_heads), float("nan"), device="cuda")
    out = _gpu_attention(wl, dev, dev.q, lse)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    got, got_lse = out.cpu(), lse.cpu()
    del out, lse, dev
    ref, ref_lse = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages,
                               wl.block_table, sp.n_kv_heads, sp.softmax_scale, sp.window,
                               with_lse=True)
    check_lse(got_lse, ref_lse, "ragged_prefill full size")
    check_attention(got, ref, "bf16", "ragged_prefill full size, every row")


def _one_head_per_kv_head(wl):
    sp = wl.spec
    G = sp.n_heads // sp.n_kv_heads
    heads = [kvh * G + kvh % G for kvh in range(sp.n_kv_heads)]
    return np.array([[t, h] for t in range(wl.total_tokens) for h in heads], np.int32)


def test_mixed_chunked_one_head_per_kv_head_every_token():
    sp = W.SPECS["mixed_chunked_mrope"]
    src = W.make(sp, seed=0)
    wl = W.attention_only(sp, 0, src.q_lens, src.kv_lens)
    dev = to_device(wl)
    lse = torch.full((wl.total_tokens, sp.n_heads), float("nan"), device="cuda")
    out = _gpu_attention(wl, dev, dev.q, lse)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    rows = _one_head_per_kv_head(wl)
    ti, hi = torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 1]).long()
    got, got_lse = out.cpu()[ti, hi], lse.cpu()[ti, hi]
    ref, ref_lse = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages,
                               wl.block_table, sp.n_kv_heads, sp.softmax_scale, sp.window,
                               rows=rows, with_lse=True)
    check_lse(got_lse, ref_lse, "mixed_chunked_mrope full size")
    check_attention(got, ref, "bf16", "mixed_chunked_mrope full size, one head per KV head")


def _tile_rows(wl):
    """One (token, head) row inside every 128-row query tile of every (sequence,
    KV head), plus the last token of each: a tile holds 128 / G consecutive
    tokens of the group's G heads."""
    sp = wl.spec
    G = sp.n_heads // sp.n_kv_heads
    tpt = 128 // G
    rows = []
    for b in range(sp.batch):
        lo, hi = int(wl.q_offsets[b]), int(wl.q_offsets[b + 1])
        for kvh in range(sp.n_kv_heads):
            for j, t0 in enumerate(range(lo, hi, tpt)):
                n = min(tpt, hi - t0)
                rows.append((t0 + (5 * j + kvh) % n, kvh * G + (j + kvh) % G))
            if hi > lo:
                rows.append((hi - 1, kvh * G + (b + kvh) % G))
    return np.array(rows, np.int32)


def test_mixed_chunked_end_to_end_full_size():
    sp = W.SPECS["mixed_chunked_mrope"]
    wl = W.make(sp, seed=0)
    dev = to_device(wl)
    tab = R.freqs_cis(wl.max_position, sp.rotary_dim, sp.theta)
    q_rot = torch.empty_like(dev.q)
    R.rope_qk_paged_ragged(dev.q, dev.offsets, dev.k_new, dev.v_new, dev.cache, tab,
                           dev.position_ids, sp.interleaved, sp.rotary_dim, q_rot,
                           mrope_section=sp.mrope_section)
    out = _gpu_attention(wl, dev, q_rot)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0

    tab_np = oracle_table(wl)
    # the GPU table is the oracle's to within one fp32 rounding of cos / sin
    assert np.allclose(tab.cpu().numpy(), tab_np, rtol=0, atol=2.0 ** -23)
    q_ref, k_ref = oracle_rope(wl, tab_np)
    check_rope(q_rot, q_ref, wl.q, sp.rotary_dim, sp.interleaved, sp.dtype, "out_q full size")
    k_img, v_img = O.cache_image(k_ref, wl.v_new, wl.q_offsets, wl.cache_lens, wl.block_table,
                                 wl.k_pages, wl.v_pages)
    kp, vp = raw_bits(dev.cache.k_pages), raw_bits(dev.cache.v_pages)
    assert np.array_equal(vp, v_img.view(vp.dtype)), "V pool differs from the oracle image"
    k_in = raw_bits(wl.k_pages)
    touched = np.any(k_img.view(kp.dtype) != k_in, axis=(2, 3))
    assert np.array_equal(kp[~touched], k_in[~touched]), "untouched K slots changed"
    k_got = gather_logical(dev.cache.k_pages.cpu(), wl, new_token_slots(wl))
    check_rope(k_got, k_ref, wl.k_new, sp.rotary_dim, sp.interleaved, sp.dtype, "K cache")

    rows = _tile_rows(wl)
    ref = O.attention(O.round_to(q_ref, O.BF16), wl.q_offsets, wl.kv_lens, k_img, v_img,
                      wl.block_table, sp.n_kv_heads, sp.softmax_scale, sp.window, rows=rows)
    ti, hi = torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 1]).long()
    check_attention(out.cpu()[ti, hi], ref, "bf16", "mixed_chunked_mrope end to end, tile rows")


GRAD_TOL = (2e-2, 2e-3)  # bf16: max and mean error relative to the largest |reference|


def _check_grad(got: np.ndarray, ref: np.ndarray, what: str):
    assert np.all(np.isfinite(got)), f"{what}: non-finite gradient"
    scale = float(np.max(np.abs(ref)))
    assert scale > 0.0, f"{what}: reference is identically zero"
    diff = np.abs(got - ref)
    assert diff.max() <= GRAD_TOL[0] * scale, f"{what}: max error {diff.max():.3g} / {scale:.3g}"
    assert diff.mean() <= GRAD_TOL[1] * scale, f"{what}: mean error {diff.mean():.3g}"


def test_backward_full_size_sampled():
    sp = W.SPECS["ragged_prefill"]
    src = W.make(sp, seed=0)
    wl = W.attention_only(sp, 0, src.q_lens, src.kv_lens)
    dev = to_device(wl)
    T, H, d = wl.q.shape
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    out = _gpu_attention(wl, dev, dev.q, lse)
    rng = np.random.default_rng(7)
    d_out_h = torch.from_numpy(rng.standard_normal((T, H, d), dtype=np.float32)).to(wl.q.dtype)
    d_out = d_out_h.cuda()
    d_q = torch.full((T, H, d), float("nan"), device="cuda")
    pool = tuple(dev.cache.k_pages.shape)
    d_k = torch.zeros(pool, dtype=torch.float32, device="cuda")
    d_v = torch.zeros(pool, dtype=torch.float32, device="cuda")
    R.ragged_paged_attention_backward(dev.q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads,
                                      sp.n_kv_heads, sp.head_dim, sp.softmax_scale, sp.window,
                                      out, d_out, lse, d_q, d_k, d_v, max_q_len=wl.max_q_len,
                                      max_kv_len=wl.max_kv_len)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    gq = d_q.cpu().double().numpy()
    gk, gv = d_k.cpu(), d_v.cpu()

    # (1) the two shortest sequences in full: a sub-batch with the same pools
    order = np.argsort(wl.q_lens)
    for b in sorted(order[:2].tolist()):
        lo, hi = int(wl.q_offsets[b]), int(wl.q_offsets[b + 1])
        offs = np.array([0, hi - lo], np.int64)
        rq, rk, rv = O.attention_backward(wl.q[lo:hi], d_out_h[lo:hi], offs, wl.kv_lens[b:b + 1],
                                          wl.k_pages, wl.v_pages, wl.block_table[b:b + 1],
                                          sp.n_kv_heads, sp.softmax_scale, sp.window)
        _check_grad(gq[lo:hi], rq, f"d_q of sequence {b}")
        slots = [(b, list(range(int(wl.kv_lens[b]))))]
        ref_k = gather_logical(torch.from_numpy(rk), wl, slots).numpy()
        ref_v = gather_logical(torch.from_numpy(rv), wl, slots).numpy()
        _check_grad(gather_logical(gk, wl, slots).double().numpy(), ref_k, f"d_k of sequence {b}")
        _check_grad(gather_logical(gv, wl, slots).double().numpy(), ref_v, f"d_v of sequence {b}")

    # (2) 256 tokens of the longest sequence, each as a one-token sequence
    b = int(order[-1])
    lo, hi = int(wl.q_offsets[b]), int(wl.q_offsets[b + 1])
    toks = np.sort(np.random.default_rng(8).choice(np.arange(lo, hi), 256, replace=False))
    toks[0], toks[-1] = lo, hi - 1
    pos = toks - lo + int(wl.kv_lens[b]) - (hi - lo)
    n = len(toks)
    rq, _, _ = O.attention_backward(wl.q[toks], d_out_h[toks], np.arange(n + 1), pos + 1,
                                    wl.k_pages, wl.v_pages, np.repeat(wl.block_table[b:b + 1],
                                                                      n, axis=0),
                                    sp.n_kv_heads, sp.softmax_scale, sp.window)
    _check_grad(gq[toks], rq, f"d_q of 256 tokens of sequence {b}")
