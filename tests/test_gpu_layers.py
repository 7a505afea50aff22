"""Multi-layer cache collections on the GPU (Mojo's layer_idx: "index of the
layer whose keys are updated in the cache").

The pools hold several layers, layer-major; a call with layer_idx = l must
write and read layer l exactly as a single-layer call on that layer's pools
would, and leave every other layer bit for bit as it was.
"""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import (check_attention, check_lse, check_rope, gather_logical, new_token_slots,
                    oracle_rope, oracle_table, raw_bits)

pytestmark = pytest.mark.gpu


def _layered(wl: W.Workload, n_layers: int, seed: int):
    """n_layers pools: the workload's own pools as every layer, each other layer's
    used slots redrawn so that the layers differ."""
    rng = np.random.default_rng(seed)
    ks, vs = [], []
    for layer in range(n_layers):
        k, v = wl.k_pages.clone(), wl.v_pages.clone()
        if layer:
            noise = torch.from_numpy(rng.normal(size=tuple(k.shape)).astype(np.float32))
            keep = torch.isnan(k.float())
            k = torch.where(keep, k, noise.to(k.dtype))
            noise = torch.from_numpy(rng.normal(size=tuple(v.shape)).astype(np.float32))
            v = torch.where(torch.isnan(v.float()), v, noise.to(v.dtype))
        ks.append(k)
        vs.append(v)
    return torch.stack(ks), torch.stack(vs)


@pytest.mark.parametrize("layer", [0, 2])
def test_rope_writes_only_its_layer(layer):
    sp = W.spec("mixed_chunked_mrope", batch=3, new_tokens=("uniform", 1, 40),
                cache_tokens=("uniform", 0, 200))
    wl = W.make(sp, seed=31)
    kl, vl = _layered(wl, 3, seed=32)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = R.PagedKVCache(k_pages=kl.cuda(), v_pages=vl.cuda(), block_table=i32(wl.block_table),
                           cache_lens=i32(wl.cache_lens), error_word=err, layer_idx=layer)
    tab_np = oracle_table(wl)
    out = torch.empty_like(wl.q).cuda()
    R.rope_qk_paged_ragged(wl.q.cuda(), i32(wl.q_offsets), wl.k_new.cuda(), wl.v_new.cuda(),
                           cache, torch.from_numpy(tab_np).cuda(), i32(wl.position_ids),
                           sp.interleaved, sp.rotary_dim, out, mrope_section=sp.mrope_section)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    q_ref, k_ref = oracle_rope(wl, tab_np)
    check_rope(out, q_ref, wl.q, sp.rotary_dim, sp.interleaved, sp.dtype, "out_q")
    kp, vp = cache.k_pages.cpu(), cache.v_pages.cpu()
    for other in range(3):
        if other != layer:
            assert np.array_equal(raw_bits(kp[other]), raw_bits(kl[other])), f"K layer {other}"
            assert np.array_equal(raw_bits(vp[other]), raw_bits(vl[other])), f"V layer {other}"
    k_img, v_img = O.cache_image(k_ref, wl.v_new, wl.q_offsets, wl.cache_lens, wl.block_table,
                                 kl[layer], vl[layer])
    vb = raw_bits(vp[layer])
    assert np.array_equal(vb, v_img.view(vb.dtype))
    k_got = gather_logical(kp[layer], wl, new_token_slots(wl))
    check_rope(k_got, k_ref, wl.k_new, sp.rotary_dim, sp.interleaved, sp.dtype, "K layer")


@pytest.mark.parametrize("name,q_lens,kv_lens", [
    ("llama3_8b_decode", [1, 1, 1], [700, 65, 1500]),      # split-KV decode
    ("ragged_prefill", [130, 70], [130, 300]),             # tcgen05 prefill
])
@pytest.mark.parametrize("layer", [1, 3])
def test_attention_reads_only_its_layer(name, q_lens, kv_lens, layer):
    sp = W.spec(name, batch=len(q_lens))
    wl = W.attention_only(sp, 33, q_lens, kv_lens)
    kl, vl = _layered(wl, 4, seed=34)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = R.PagedKVCache(k_pages=kl.cuda(), v_pages=vl.cuda(), block_table=i32(wl.block_table),
                           error_word=err, layer_idx=layer)
    q = wl.q.cuda()
    out = torch.empty_like(q)
    lse = torch.empty((wl.total_tokens, sp.n_heads), device="cuda")
    R.ragged_paged_attention(q, i32(wl.q_offsets), i32(wl.kv_lens), cache, sp.n_heads,
                             sp.n_kv_heads, sp.head_dim, sp.softmax_scale, sp.window, out,
                             max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len, log_sum_exp=lse)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, ref_lse = O.attention(wl.q, wl.q_offsets, wl.kv_lens, kl[layer], vl[layer],
                               wl.block_table, sp.n_kv_heads, sp.softmax_scale, sp.window,
                               with_lse=True)
    check_attention(out.cpu(), ref, sp.dtype, f"layer {layer}")
    check_lse(lse.cpu(), ref_lse, f"layer {layer}")
