"""The whole path on the GPU -- table, RoPE + scatter, attention -- against the
oracle's chain (oracle table, oracle RoPE, oracle cache image, oracle
attention) on the same seeded inputs."""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import REDUCED, check_attention, oracle_rope, oracle_table, to_device

pytestmark = pytest.mark.gpu


def _chain(wl: W.Workload, use_gpu_table: bool):
    sp = wl.spec
    dev = to_device(wl)
    tab_np = oracle_table(wl)
    tab = (R.freqs_cis(wl.max_position, sp.rotary_dim, sp.theta) if use_gpu_table
           else torch.from_numpy(tab_np).cuda())
    q_rot = torch.empty_like(dev.q)
    R.rope_qk_paged_ragged(dev.q, dev.offsets, dev.k_new, dev.v_new, dev.cache, tab,
                           dev.position_ids, sp.interleaved, sp.rotary_dim, q_rot,
                           mrope_section=sp.mrope_section)
    out = torch.empty_like(q_rot)
    R.ragged_paged_attention(q_rot, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads,
                             sp.n_kv_heads, sp.head_dim, sp.softmax_scale, sp.window, out,
                             max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0

    q_ref, k_ref = oracle_rope(wl, tab_np)
    code = O.BF16 if sp.dtype == "bf16" else O.F32
    q_rounded = O.round_to(q_ref, code)
    k_img, v_img = O.cache_image(k_ref, wl.v_new, wl.q_offsets, wl.cache_lens, wl.block_table,
                                 wl.k_pages, wl.v_pages)
    ref = O.attention(q_rounded, wl.q_offsets, wl.kv_lens, k_img, v_img, wl.block_table,
                      sp.n_kv_heads, sp.softmax_scale, sp.window)
    check_attention(out.cpu(), ref, sp.dtype, f"end to end {sp.name}")


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_end_to_end_reduced(name):
    _chain(W.make(REDUCED[name], seed=0), use_gpu_table=False)


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_end_to_end_gpu_table(name):
    _chain(W.make(REDUCED[name], seed=1), use_gpu_table=True)
