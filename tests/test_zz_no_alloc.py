"""ragged_paged_attention_noalloc against ragged_paged_attention.

Some callers cannot allocate device memory when they run attention: a serving
engine that reserved all free HBM for its KV cache at start-up, a plugin that
runs inside a framework owning every allocator, or a decode loop that cannot
pay for cudaMalloc's implicit synchronisation. For them the library has an
entry point that takes no workspace and keeps its scratch in a fixed 32 MiB
array of its own. These tests call it through the C ABI and check that it
returns the same rows as the workspace entry point, within the attention
tolerance used everywhere else (bf16: max-abs 2e-2, mean-abs 2e-3).

Two calls in a row, on different batches, check that the shared array, which
keeps whatever the previous call left in it, does not leak into the next
result. This file is collected last so that a stop at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""

import numpy as np
import pytest
import torch

import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import binding as B
from ragged_paged_kv_rope_b200 import workloads as W
from parity import check_attention, to_device

pytestmark = pytest.mark.gpu


def _both(sp: W.Spec, q_lens, kv_lens, seed: int):
    wl = W.attention_only(sp, seed, q_lens, kv_lens)
    dev = to_device(wl)
    args = (dev.q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads, sp.n_kv_heads, sp.head_dim,
            sp.softmax_scale, sp.window)
    kw = dict(max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len)
    ref = torch.empty_like(dev.q)
    R.ragged_paged_attention(*args, ref, **kw)
    got = torch.full_like(dev.q, float("nan"))
    B.ragged_paged_attention_noalloc(*args, got, **kw)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    return got.float().cpu().numpy().astype(np.float64), ref.float().cpu().numpy().astype(np.float64)


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    # call 1: the Llama-3-8B-shaped decode batch (64 sequences, contexts up to 8192)
    sp1 = W.SPECS["llama3_8b_decode"]
    wl1 = W.make(sp1, seed=0)
    got1, ref1 = _both(sp1, wl1.q_lens, wl1.kv_lens, seed=21)
    check_attention(got1, ref1, "bf16", "no-alloc call 1")
    # call 2: a different shape (d 256, window, two query rows per sequence) that
    # uses less of the array, so stale partials of call 1 would show
    sp2 = W.spec("gemma_swa_decode", batch=5, window=900, page_size=64)
    got2, ref2 = _both(sp2, [1, 2, 1, 2, 1], [3000, 1200, 64, 5000, 700], seed=22)
    check_attention(got2, ref2, "bf16", "no-alloc call 2")


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
