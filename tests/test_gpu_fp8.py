"""GPU parity of the e4m3 KV cache against the fp64 oracle.

rope_qk_paged_ragged writes code = e4m3(x / scale) into an e4m3 cache (one
fp32 scale per KV head for K and one for V), and ragged_paged_attention reads
key = code * k_scale, value = code * v_scale (the decode kernel in f16 after an
exact widening, the CUDA-core kernel in fp32).

Cache codes: the kernel divides in fp32 and rounds that quotient once, the
oracle divides in fp64 and rounds once. The codes must be equal, except that
two adjacent codes are accepted where the exact quotient lies within the fp32
error of the value (V: the division, 2^-23 relative; rotated K: the RoPE
evaluation bound 2^-22 (|a| + |b|) of its pair, divided by the scale) of the
midpoint between them. Slots the call does not write stay bit for bit.
Attention: the tolerances of the other attention tests, against the oracle
run on the same e4m3 pools.
"""

import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import (REDUCED, check_attention, check_lse, check_rope, gpu_attention, gpu_rope,
                    new_token_slots, oracle_rope, oracle_table, pair_abs_sum, sample_rows,
                    to_device)

pytestmark = pytest.mark.gpu

E4M3 = {name: dataclasses.replace(sp, cache_dtype="e4m3") for name, sp in REDUCED.items()}

_DEC = np.array([O.e4m3_to_f64(c) for c in range(256)])


def _codes(pool: torch.Tensor) -> np.ndarray:
    return pool.detach().cpu().contiguous().view(torch.uint8).numpy()


def _check_codes(got, want, exact_q, slack, what):
    """got / want: uint8 codes; exact_q: the fp64 quotients; slack: allowed distance of
    the quotient from the midpoint of two adjacent codes."""
    bad = np.nonzero(got != want)
    if bad[0].size == 0:
        return 0
    g, w, q, s = got[bad], want[bad], exact_q[bad], slack[bad]
    gv, wv = _DEC[g], _DEC[w]
    # adjacent codes of the same sign (or across zero)
    lo, hi = np.minimum(gv, wv), np.maximum(gv, wv)
    adjacent = np.array([_next_up(a) == b for a, b in zip(lo, hi)])
    near_tie = np.abs(q - 0.5 * (gv + wv)) <= s
    ok = adjacent & near_tie
    assert np.all(ok), (f"{what}: {int((~ok).sum())} cache codes differ beyond a near-tie, "
                        f"first quotient {q[~ok][0]!r}: got {gv[~ok][0]!r} want {wv[~ok][0]!r}")
    return int(bad[0].size)


_FINITE = np.unique(_DEC[~np.isnan(_DEC)])


def _next_up(a: float) -> float:
    i = np.searchsorted(_FINITE, a, side="right")
    return _FINITE[i] if i < len(_FINITE) else np.inf


@pytest.mark.parametrize("name", ["llama3_8b_decode", "gemma_swa_decode",
                                  "mixed_chunked_mrope", "tiny_prefill_f32"])
def test_rope_writes_e4m3_cache(name):
    sp = E4M3[name]
    wl = W.make(sp, seed=2)
    dev = to_device(wl)
    table = R.freqs_cis(wl.max_position, sp.rotary_dim, sp.theta)
    before_k, before_v = _codes(dev.cache.k_pages), _codes(dev.cache.v_pages)
    out_q = gpu_rope(wl, dev, table)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    q_ref, k_ref = oracle_rope(wl, oracle_table(wl))
    check_rope(out_q.cpu(), q_ref, wl.q, sp.rotary_dim, sp.interleaved, sp.dtype, name)

    gk, gv = _codes(dev.cache.k_pages), _codes(dev.cache.v_pages)
    wk, wv = O.cache_image(k_ref, wl.v_new, wl.q_offsets, wl.cache_lens, wl.block_table,
                           wl.k_pages, wl.v_pages, k_scale=wl.k_scale, v_scale=wl.v_scale)
    # the written slots, token by token
    P = sp.page_size
    written = np.zeros(gk.shape[:2], dtype=bool)
    n_tie = 0
    ks, vs = wl.k_scale.astype(np.float64), wl.v_scale.astype(np.float64)
    ps = pair_abs_sum(O.widen(wl.k_new), sp.rotary_dim, sp.interleaved)
    v64 = O.widen(wl.v_new)
    for b, slots in new_token_slots(wl):
        for i, slot in enumerate(slots):
            t = int(wl.q_offsets[b]) + i
            page, row = int(wl.block_table[b, slot // P]), slot % P
            written[page, row] = True
            qk = k_ref[t] / ks[:, None]
            sk = 2.0 ** -22 * ps[t] / ks[:, None] + 2.0 ** -22 * np.abs(qk)
            n_tie += _check_codes(gk[page, row], wk[page, row], qk, sk, f"{name} K slot {slot}")
            qv = v64[t] / vs[:, None]
            n_tie += _check_codes(gv[page, row], wv[page, row], qv, 2.0 ** -22 * np.abs(qv),
                                  f"{name} V slot {slot}")
    assert np.array_equal(gk[~written], before_k[~written]), f"{name}: untouched K slots changed"
    assert np.array_equal(gv[~written], before_v[~written]), f"{name}: untouched V slots changed"
    assert n_tie <= max(4, gk[written].size // 1000), f"{name}: {n_tie} near-tie differences"


@pytest.mark.parametrize("name", ["llama3_8b_decode", "gemma_swa_decode", "ragged_prefill",
                                  "mixed_chunked_mrope", "tiny_prefill_f32"])
def test_attention_over_e4m3_cache(name):
    sp = E4M3[name]
    ref_wl = W.make(sp, seed=0)
    wl = W.attention_only(sp, 1, ref_wl.q_lens, ref_wl.kv_lens)
    dev = to_device(wl)
    lse = torch.full((wl.total_tokens, sp.n_heads), float("nan"), device="cuda")
    rows = None if wl.total_tokens * sp.n_heads <= 20000 else sample_rows(wl, 600)
    out = gpu_attention(wl, dev, dev.q, lse=lse)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    ref, ref_lse = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages,
                               wl.block_table, sp.n_kv_heads, sp.softmax_scale, sp.window,
                               rows=rows, with_lse=True, k_scale=wl.k_scale, v_scale=wl.v_scale)
    got, got_lse = out.cpu(), lse.cpu()
    if rows is not None:
        ti, hi = torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 1]).long()
        got, got_lse = got[ti, hi], got_lse[ti, hi]
    check_lse(got_lse, ref_lse, f"{name} e4m3")
    check_attention(got, ref, sp.dtype, f"{name} e4m3")


@pytest.mark.parametrize("d", [64, 256])
def test_decode_over_e4m3_cache_head_dims(d):
    sp = W.spec("llama3_8b_decode", cache_dtype="e4m3", head_dim=d, rotary_dim=d, batch=5,
                cache_tokens=("uniform", 30, 900))
    wl = W.attention_only(sp, 4, [1, 1, 1, 1, 1], [31, 64, 65, 513, 901])
    dev = to_device(wl)
    out = gpu_attention(wl, dev, dev.q)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    ref = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages, wl.block_table,
                      sp.n_kv_heads, sp.softmax_scale, 0, k_scale=wl.k_scale, v_scale=wl.v_scale)
    check_attention(out.cpu(), ref, "bf16", f"d={d} e4m3")


@pytest.mark.parametrize("d", [128, 256])
def test_decode_over_e4m3_cache_more_rows(d):
    # 3 and 4 tokens of a group of 4: 12 and 16 rows per KV head (two n-tiles)
    sp = W.spec("llama3_8b_decode", cache_dtype="e4m3", head_dim=d, rotary_dim=d, batch=3)
    wl = W.attention_only(sp, 6, [3, 4, 1], [200, 700, 64])
    dev = to_device(wl)
    out = gpu_attention(wl, dev, dev.q)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    ref = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages, wl.block_table,
                      sp.n_kv_heads, sp.softmax_scale, 0, k_scale=wl.k_scale, v_scale=wl.v_scale)
    check_attention(out.cpu(), ref, "bf16", f"d={d} e4m3, 12 and 16 rows")


def test_decode_e4m3_large_and_small_queries():
    # Q far outside f16's range in both directions: the kernel's power-of-two
    # pre-scale keeps the scores right.
    sp = W.spec("llama3_8b_decode", cache_dtype="e4m3", batch=3)
    wl = W.attention_only(sp, 5, [1, 1, 1], [200, 700, 64])
    big = wl.q.float() * 1e6
    big[1] = wl.q[1].float() * 1e-7
    wl.q = big.to(torch.bfloat16)
    dev = to_device(wl)
    scale = 1e-6
    out = torch.empty_like(dev.q)
    R.ragged_paged_attention(dev.q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads,
                             sp.n_kv_heads, sp.head_dim, scale, 0, out, max_q_len=1,
                             max_kv_len=wl.max_kv_len)
    torch.cuda.synchronize()
    ref = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages, wl.block_table,
                      sp.n_kv_heads, scale, 0, k_scale=wl.k_scale, v_scale=wl.v_scale)
    check_attention(out.cpu(), ref, "bf16", "large / small q, e4m3")


def test_end_to_end_decode_step_e4m3():
    # RoPE writes the new token into the e4m3 cache, attention reads it back;
    # the oracle attends over the pools the GPU wrote (stage-isolated).
    sp = E4M3["llama3_8b_decode"]
    wl = W.make(sp, seed=7)
    dev = to_device(wl)
    table = R.freqs_cis(wl.max_position, sp.rotary_dim, sp.theta)
    q_rot = gpu_rope(wl, dev, table)
    out = gpu_attention(wl, dev, q_rot)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    ref = O.attention(q_rot.cpu(), wl.q_offsets, wl.kv_lens, dev.cache.k_pages.cpu(),
                      dev.cache.v_pages.cpu(), wl.block_table, sp.n_kv_heads, sp.softmax_scale,
                      sp.window, k_scale=wl.k_scale, v_scale=wl.v_scale)
    check_attention(out.cpu(), ref, "bf16", "decode step e4m3")


# ------------------------------------------- prefill shapes over an e4m3 cache
# The tcgen05 prefill kernel widens each key tile's codes to f16 on chip (exact)
# and narrows each Q row to f16 under a power-of-two scale, so the products are
# those of the bf16 path up to f16's extra mantissa bits.

def _e4m3_case(sp, q_lens, kv_lens, seed, window=0, sinks=0, q_mul=None):
    wl = W.attention_only(sp, seed, q_lens, kv_lens)
    if q_mul is not None:
        wl.q = (wl.q.float() * q_mul).to(torch.bfloat16)
    dev = to_device(wl)
    lse = torch.full((wl.total_tokens, sp.n_heads), float("nan"), device="cuda")
    out = gpu_attention(wl, dev, dev.q, window=window, lse=lse, sinks=sinks)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    ref, ref_lse = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages,
                               wl.block_table, sp.n_kv_heads, sp.softmax_scale, window,
                               with_lse=True, sinks=sinks, k_scale=wl.k_scale,
                               v_scale=wl.v_scale)
    what = f"e4m3 d={sp.head_dim} q={list(q_lens)} window={window} sinks={sinks}"
    check_lse(lse.cpu(), ref_lse, what)
    check_attention(out.cpu(), ref, "bf16", what)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("window,sinks", [(0, 0), (150, 0), (129, 70)])
def test_prefill_over_e4m3_cache(d, window, sinks):
    # two query tiles per item, several key tiles, ragged tails, a chunk whose
    # first token sits deep in its sequence and a one-token sequence
    sp = W.spec("ragged_prefill", cache_dtype="e4m3", head_dim=d, rotary_dim=d, batch=4,
                n_heads=8, n_kv_heads=2)
    _e4m3_case(sp, [300, 129, 1, 77], [300, 700, 64, 77], seed=21, window=window,
                       sinks=sinks)


def test_prefill_over_e4m3_cache_page_16_group_8():
    # pages of 16 tokens (a key tile spans four pages) and eight query heads per
    # KV head (16 tokens per query tile)
    sp = W.spec("llama3_8b_decode", cache_dtype="e4m3", batch=3, n_heads=16, n_kv_heads=2,
                page_size=16)
    _e4m3_case(sp, [100, 33, 250], [400, 33, 250], seed=22)


def test_prefill_e4m3_large_and_small_queries():
    # Q rows far outside f16's range in both directions: each row's
    # power-of-two pre-scale keeps its scores right.
    sp = W.spec("ragged_prefill", cache_dtype="e4m3", batch=3, n_heads=8, n_kv_heads=2)
    wl = W.attention_only(sp, 23, [200, 70, 130], [200, 300, 130])
    mul = torch.ones(wl.total_tokens, 1, 1)
    mul[:200] = 1e6
    mul[200:270] = 1e-7
    _e4m3_case(sp, [200, 70, 130], [200, 300, 130], seed=23, q_mul=mul)


@pytest.mark.parametrize("d", [128, 256])
def test_decode_over_e4m3_cache_window_and_sinks(d):
    # decode rows (one and two tokens) under a window with attention sinks: the
    # sink tile and the band's tiles, a band whose first tile is partial and a
    # sequence shorter than the window
    sp = W.spec("llama3_8b_decode", cache_dtype="e4m3", head_dim=d, rotary_dim=d, batch=4)
    _e4m3_case(sp, [1, 1, 1, 2], [5000, 300, 70, 2000], seed=24, window=1000, sinks=4)
