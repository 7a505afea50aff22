"""Device-side bounded waits that run out, on the GPU.

Every wait of the attention kernels (a K/V stage, a score tile, a work item)
is bounded. rpk_set_wait_limit_ns shortens that bound for later launches; at
a few nanoseconds every wait whose phase is not already complete gives up,
which happens at once in any real launch (the first K/V tiles come from HBM).
A CTA that gives up ORs RPK_DEVERR_TIMEOUT into the error word, lets the
copies and tensor-core operations it issued finish, frees its tensor memory
and returns. Each test checks that bit, then restores the default bound,
clears the error word and runs the same call again on the same stream: it
must match the oracle, which shows the context and the GPU stayed usable.

Cases: the split-KV decode kernel with several splits (so the combine kernel
runs after the decode kernel gave up), and the tcgen05 prefill kernel.
Nothing here faults, traps or spins without a bound.
"""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import check_attention, gpu_attention, to_device

pytestmark = pytest.mark.gpu

SHORT_NS = 20  # under the timer resolution: waits give up at their first incomplete test


def _timeout_then_healthy(sp: W.Spec, q_lens, kv_lens, seed: int):
    wl = W.attention_only(sp, seed, q_lens, kv_lens)
    dev = to_device(wl)
    stream = torch.cuda.current_stream()
    try:
        R.set_wait_limit_ns(SHORT_NS)
        assert R.wait_limit_ns() == SHORT_NS
        gpu_attention(wl, dev, dev.q)
        torch.cuda.synchronize()
        word = int(dev.error_word.item())
    finally:
        R.set_wait_limit_ns(0)
    assert R.wait_limit_ns() == 2_000_000_000
    assert word & R.binding.DEVERR_TIMEOUT, f"no timeout reported (error word {word:#x})"
    assert word & ~R.binding.DEVERR_TIMEOUT == 0, f"unexpected error bits {word:#x}"

    # the same call again on the same stream, with the default bound
    dev.error_word.zero_()
    out = gpu_attention(wl, dev, dev.q)
    stream.synchronize()
    assert int(dev.error_word.item()) == 0
    ref = O.attention(wl.q, wl.q_offsets, wl.kv_lens, wl.k_pages, wl.v_pages, wl.block_table,
                      sp.n_kv_heads, sp.softmax_scale, sp.window)
    check_attention(out.cpu(), ref, sp.dtype, f"{sp.name} after a timed-out launch")


def test_decode_and_combine_wait_limit_runs_out():
    # contexts of 2000-6000 keys: 32 (sequence, KV head) units take splits of
    # 11 key tiles (9 splits for the longest), so the combine kernel runs, and
    # every split holds more tiles than the stage ring: the producer's wait for
    # a free stage cannot already be complete
    sp = W.spec("llama3_8b_decode", batch=4)
    _timeout_then_healthy(sp, [1, 1, 1, 1], [6000, 2000, 4100, 3000], seed=61)


def test_prefill_wait_limit_runs_out():
    sp = W.spec("ragged_prefill", batch=3, n_heads=8, n_kv_heads=2)
    _timeout_then_healthy(sp, [300, 129, 64], [300, 129, 700], seed=62)

