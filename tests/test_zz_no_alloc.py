"""ragged_paged_attention_noalloc against the oracle and the workspace entry point.

Some callers cannot allocate device memory when they run attention: a serving
engine that reserved all free HBM for its KV cache at start-up, a plugin that
runs inside a framework owning every allocator, or a decode loop that cannot
pay for cudaMalloc's implicit synchronisation. For them the library has an
entry point that takes no workspace and keeps its scratch in a fixed 32 MiB
array of its own. These tests call it through the C ABI and check its rows
against the fp64 oracle and against the workspace entry point, within the
attention tolerance used everywhere else (bf16: max-abs 2e-2, mean-abs 2e-3).

Two calls in a row, on different batches, check that the shared array, which
keeps whatever the previous call left in it, does not leak into the next
result. Further cases: a short context that runs as one split (no scratch
used), a window of 2^31 - 1 keys with rows that see no key, and a check that
the call changes neither the device's free memory nor torch's allocator.
This file is collected last so that a stop at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import binding as B
from ragged_paged_kv_rope_b200 import workloads as W
from parity import check_attention, to_device

pytestmark = pytest.mark.gpu


def _args(sp: W.Spec, wl: W.Workload, dev, window):
    return (dev.q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads, sp.n_kv_heads, sp.head_dim,
            sp.softmax_scale, window)


def _both(sp: W.Spec, q_lens, kv_lens, seed: int, window=None):
    """(no-alloc rows, workspace-entry rows, oracle rows), all fp64."""
    wl = W.attention_only(sp, seed, q_lens, kv_lens)
    dev = to_device(wl)
    w = sp.window if window is None else window
    args = _args(sp, wl, dev, w)
    kw = dict(max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len)
    ref = torch.empty_like(dev.q)
    R.ragged_paged_attention(*args, ref, **kw)
    got = torch.full_like(dev.q, float("nan"))
    B.ragged_paged_attention_noalloc(*args, got, **kw)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    oracle = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages, wl.block_table,
                         sp.n_kv_heads, sp.softmax_scale, w)
    return O.widen(got.cpu()), O.widen(ref.cpu()), oracle


def _check(sp, q_lens, kv_lens, seed, what, window=None):
    got, ref, oracle = _both(sp, q_lens, kv_lens, seed, window)
    check_attention(got, oracle, "bf16", f"{what} vs oracle")
    check_attention(got, ref, "bf16", f"{what} vs workspace entry point")
    return got


def test_noalloc_matches_oracle_on_two_calls_in_a_row():
    # call 1: the Llama-3-8B-shaped decode batch (64 sequences, contexts up to 8192)
    sp1 = W.SPECS["llama3_8b_decode"]
    wl1 = W.make(sp1, seed=0)
    _check(sp1, wl1.q_lens, wl1.kv_lens, 21, "no-alloc call 1")
    # call 2: a different shape (d 256, window, two query rows per sequence) that
    # uses less of the array, so stale partials of call 1 would show
    sp2 = W.spec("gemma_swa_decode", batch=5, window=900, page_size=64)
    _check(sp2, [1, 2, 1, 2, 1], [3000, 1200, 64, 5000, 700], 22, "no-alloc call 2")


def test_noalloc_single_split_short_contexts():
    # contexts of at most 512 keys run as one split per sequence: the kernel
    # writes the rows itself and the array is not touched
    sp = W.spec("llama3_8b_decode", batch=6)
    _check(sp, [1] * 6, [512, 1, 63, 64, 65, 300], 23, "single split")


def test_noalloc_window_of_int32_max_with_rows_that_see_no_key():
    # kv_len < q_len: the first rows of the first sequence sit before key 0 and
    # see no key (zeros). A window of 2^31 - 1 keys covers every key, so the
    # result is the unbounded one; the window arithmetic must not overflow.
    sp = W.spec("llama3_8b_decode", batch=3)
    q_lens, kv_lens = [3, 1, 2], [1, 700, 2000]
    got = _check(sp, q_lens, kv_lens, 24, "window 2^31 - 1", window=2**31 - 1)
    assert np.all(got[0:2] == 0.0), "rows before the first key must be zeros"
    unbounded, _, _ = _both(sp, q_lens, kv_lens, 24, window=0)
    assert np.array_equal(got, unbounded)


def test_noalloc_call_does_not_allocate():
    sp = W.spec("llama3_8b_decode", batch=8)
    wl = W.attention_only(sp, 25, [1] * 8, [4000, 100, 2500, 8000, 7000, 640, 1, 3333])
    dev = to_device(wl)
    args = _args(sp, wl, dev, 0)
    kw = dict(max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len)
    out = torch.empty_like(dev.q)
    # a first call loads the library's device code and looks up the array's address
    B.ragged_paged_attention_noalloc(*args, out, **kw)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    reserved0 = torch.cuda.memory_reserved()
    for _ in range(3):
        B.ragged_paged_attention_noalloc(*args, out, **kw)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    assert int(dev.error_word.item()) == 0


def test_noalloc_refuses_what_it_cannot_run():
    dev = torch.device("cuda")
    H, Hk, d, P = 32, 8, 128, 64
    k = torch.zeros(8, P, Hk, d, dtype=torch.bfloat16, device=dev)
    cache = R.PagedKVCache(k, k.clone(), torch.zeros(64, 640, dtype=torch.int32, device=dev))
    q = torch.zeros(64, H, d, dtype=torch.bfloat16, device=dev)
    out = torch.empty_like(q)
    offs = torch.arange(65, dtype=torch.int32, device=dev)
    kvl = torch.ones(64, dtype=torch.int32, device=dev)
    # partials of 64 rows x 32 heads over a 40000-key bound exceed the 32 MiB array
    assert R.ragged_paged_attention_workspace_size(64, H, d, 64, 40000, P) > B.NOALLOC_SCRATCH_BYTES
    with pytest.raises(R.RpkError) as e:
        B.ragged_paged_attention_noalloc(q, offs, kvl, cache, H, Hk, d, None, 0, out,
                                         max_q_len=1, max_kv_len=40000)
    assert e.value.status == 6
    # prefill shapes do not use the split-KV path
    with pytest.raises(R.RpkError) as e:
        B.ragged_paged_attention_noalloc(q, offs, kvl, cache, H, Hk, d, None, 0, out,
                                         max_q_len=64, max_kv_len=64)
    assert e.value.status == 4
