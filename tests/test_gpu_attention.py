"""GPU parity of ragged_paged_attention against the fp64 oracle.

Inputs are drawn once and handed to both sides: q (as if rotated) and a fully
populated paged cache with sentinel NaNs in every unused slot, so a kernel
that reads a key or value outside the band shows up as a non-finite or wrong
row. Tolerances: bf16 max-abs 2e-2 and mean-abs 2e-3, fp32 max-abs 1e-4.
"""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import REDUCED, check_attention, check_lse, gpu_attention, sample_rows, to_device

pytestmark = pytest.mark.gpu


def _attn_case(sp: W.Spec, q_lens, kv_lens, seed=0, rows=None, window=None, sinks=0):
    wl = W.attention_only(sp, seed, q_lens, kv_lens)
    dev = to_device(wl)
    w = sp.window if window is None else window
    # every case also checks the log-sum-exp output against the oracle's
    lse = torch.full((wl.total_tokens, sp.n_heads), float("nan"), device="cuda")
    out = gpu_attention(wl, dev, dev.q, window=w, lse=lse, sinks=sinks)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    ref, ref_lse = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages,
                               wl.block_table, sp.n_kv_heads, sp.softmax_scale, w, rows=rows,
                               with_lse=True, sinks=sinks)
    got, got_lse = out.cpu(), lse.cpu()
    if rows is not None:
        ti, hi = torch.from_numpy(rows[:, 0]).long(), torch.from_numpy(rows[:, 1]).long()
        got, got_lse = got[ti, hi], got_lse[ti, hi]
    what = f"{sp.name} q={list(q_lens)[:4]}"
    check_lse(got_lse, ref_lse, what)
    return check_attention(got, ref, sp.dtype, what)


def _lens_from(wl_spec, seed):
    wl = W.make(wl_spec, seed=seed)
    return wl.q_lens, wl.kv_lens


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_attention_reduced_configs(name):
    sp = REDUCED[name]
    q_lens, kv_lens = _lens_from(sp, 0)
    _attn_case(sp, q_lens, kv_lens)


def test_attention_decode_full_size():
    # Llama-3-8B-shaped decode at its full size: every row checked.
    sp = W.SPECS["llama3_8b_decode"]
    q_lens, kv_lens = _lens_from(sp, 0)
    _attn_case(sp, q_lens, kv_lens)


@pytest.mark.slow
def test_attention_swa_decode_full_size():
    sp = W.SPECS["gemma_swa_decode"]
    _attn_case(sp, [1] * sp.batch, [32769] * sp.batch)


@pytest.mark.parametrize("name", ["ragged_prefill", "mixed_chunked_mrope"])
def test_attention_prefill_full_size_sampled(name):
    sp = W.SPECS[name]
    wl = W.make(sp, seed=0)
    _attn_case(sp, wl.q_lens, wl.kv_lens, rows=sample_rows(wl, 400))


# ---------------------------------------------------------------- edge cases

EDGE = [
    # (description, spec overrides, q_lens, kv_lens, window)
    ("single token", {}, [1], [1], 0),
    ("rows without keys", {}, [5, 3], [2, 3], 0),
    ("empty sequence in batch", {}, [4, 0, 3], [9, 5, 3], 0),
    ("window 1", {}, [6, 1], [6, 40], 1),
    ("window longer than context", {}, [3, 1], [10, 30], 100),
    ("page boundaries", {"page_size": 16}, [17, 1, 33], [33, 16, 64], 0),
    ("tail inside a tile", {"page_size": 64}, [1, 1, 1], [65, 127, 129], 0),
    ("MHA group 1", {"n_heads": 4, "n_kv_heads": 4}, [7, 1], [20, 9], 0),
    ("group 16", {"n_heads": 16, "n_kv_heads": 1}, [1, 1], [300, 7], 0),
    ("long decode", {}, [1, 1], [20000, 3], 0),
    ("long decode window", {"page_size": 128}, [1], [20000], 333),
    ("head_dim 64", {"head_dim": 64, "rotary_dim": 64}, [1, 9], [70, 30], 0),
    ("head_dim 256", {"head_dim": 256, "rotary_dim": 128}, [1, 2], [513, 200], 0),
    ("chunked prefill rows", {}, [3, 2], [100, 5], 0),
    ("head_dim 256, 12 rows", {"head_dim": 256, "rotary_dim": 128}, [3, 2], [300, 77], 0),
]


@pytest.mark.parametrize("idx", range(len(EDGE)))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_attention_edge_cases(idx, dtype):
    desc, over, q_lens, kv_lens, window = EDGE[idx]
    base = dict(n_heads=8, n_kv_heads=2, head_dim=128, page_size=32, dtype=dtype)
    base.update(over)
    sp = W.spec("ragged_prefill", **base)
    _attn_case(sp, q_lens, kv_lens, seed=idx, window=window)


# ------------------------------------------------ attention sinks + window

SINKS = [
    # (description, spec overrides, q_lens, kv_lens, window, sinks)
    ("decode, 4 sinks", {}, [1, 1, 1], [5000, 300, 70], 1000, 4),
    ("decode, sinks over several tiles", {}, [1, 1], [9000, 2000], 700, 150),
    ("decode, sinks reach the window", {}, [1, 1], [400, 90], 300, 200),
    ("decode, group 8 two tokens", {"n_heads": 16, "n_kv_heads": 2}, [2, 1], [3000, 129], 64, 3),
    ("prefill, 4 sinks", {}, [300, 200], [300, 900], 100, 4),
    ("prefill, sinks over two tiles", {}, [260, 40], [700, 260], 129, 200),
    ("prefill head_dim 64", {"head_dim": 64, "rotary_dim": 64}, [150, 90], [600, 90], 64, 17),
    ("head_dim 256", {"head_dim": 256, "rotary_dim": 128}, [1, 40], [3000, 500], 256, 8),
    ("window 1 with sinks", {}, [50, 1], [50, 1000], 1, 5),
]


@pytest.mark.parametrize("idx", range(len(SINKS)))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_attention_sinks(idx, dtype):
    desc, over, q_lens, kv_lens, window, sinks = SINKS[idx]
    base = dict(n_heads=8, n_kv_heads=2, head_dim=128, page_size=32, dtype=dtype)
    base.update(over)
    sp = W.spec("ragged_prefill", **base)
    _attn_case(sp, q_lens, kv_lens, seed=40 + idx, window=window, sinks=sinks)


def test_attention_sinks_ignored_without_window():
    sp = W.spec("ragged_prefill", n_heads=8, n_kv_heads=2, batch=2)
    wl = W.attention_only(sp, 50, [70, 1], [70, 500])
    dev = to_device(wl)
    a = gpu_attention(wl, dev, dev.q, window=0, sinks=0).cpu()
    b = gpu_attention(wl, dev, dev.q, window=0, sinks=9).cpu()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_attention_window_covering_every_key_is_unbounded():
    # a window of at least max_kv_len keys bounds nothing (sinks included), up to
    # the largest int32 window: the result equals the unbounded one bit for bit
    sp = W.spec("ragged_prefill", n_heads=8, n_kv_heads=2, batch=2)
    wl = W.attention_only(sp, 52, [70, 1], [70, 500])
    dev = to_device(wl)
    a = gpu_attention(wl, dev, dev.q, window=0).cpu()
    for w in (wl.max_kv_len, 2**31 - 1):
        b = gpu_attention(wl, dev, dev.q, window=w, sinks=3).cpu()
        torch.cuda.synchronize()
        assert int(dev.error_word.item()) == 0
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), w


@pytest.mark.slow
def test_attention_gemma_window_with_sinks_sampled():
    # the Gemma-like sliding-window decode at full context, with 4 sink tokens
    sp = W.SPECS["gemma_swa_decode"]
    rng_rows = np.array([[t, h] for t in range(sp.batch) for h in range(sp.n_heads)], np.int32)
    _attn_case(sp, [1] * sp.batch, [32769] * sp.batch, seed=51, rows=rng_rows, sinks=4)


@pytest.mark.parametrize("window", [0, 200])
def test_attention_prefill_head_dim_256(window):
    # Gemma-like layout (16 query heads over 8 KV heads, head_dim 256): one
    # query tile per work item, several 64-key tiles, ragged tails, a chunked
    # row block and a short sequence
    sp = W.spec("gemma_swa_decode", batch=3, page_size=64)
    _attn_case(sp, [300, 129, 7], [300, 700, 7], seed=16, window=window)


def test_attention_prefill_shapes_bf16():
    sp = W.spec("ragged_prefill", n_heads=8, n_kv_heads=2)
    _attn_case(sp, [130, 64, 1, 257], [130, 64, 400, 300], seed=11)
    _attn_case(sp, [200, 77], [200, 500], seed=12, window=50)


def test_attention_decode_equals_last_prefill_row():
    sp = W.spec("llama3_8b_decode", batch=2)
    wl = W.attention_only(sp, 13, [40, 1], [40, 40])
    dev = to_device(wl)
    out = gpu_attention(wl, dev, dev.q).cpu()
    ref = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages, wl.block_table,
                      sp.n_kv_heads, sp.softmax_scale, 0)
    check_attention(out, ref, "bf16", "mixed prefill/decode")


def test_attention_bad_page_sets_error_bit():
    sp = W.spec("llama3_8b_decode", batch=3)
    wl = W.attention_only(sp, 14, [1, 1, 1], [300, 200, 100])
    wl.block_table[1, 1] = -3
    dev = to_device(wl)
    out = gpu_attention(wl, dev, dev.q)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) & R.binding.DEVERR_PAGE
    ref = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages,
                      np.where(wl.block_table < 0, 0, wl.block_table), sp.n_kv_heads,
                      sp.softmax_scale, 0, rows=np.array([[0, h] for h in range(32)] +
                                                         [[2, h] for h in range(32)]))
    got = out.cpu()[[0] * 32 + [2] * 32, list(range(32)) * 2]
    check_attention(got, ref, "bf16", "rows of intact sequences")


def test_attention_length_over_bound_sets_error_bit():
    sp = W.spec("llama3_8b_decode", batch=2)
    wl = W.attention_only(sp, 15, [1, 1], [100, 50])
    dev = to_device(wl)
    out = torch.empty_like(dev.q)
    R.ragged_paged_attention(dev.q, dev.offsets, dev.kv_lens, dev.cache, 32, 8, 128, None, 0, out,
                             max_q_len=1, max_kv_len=60)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) & R.binding.DEVERR_LENGTH
