"""GPU parity of rope_qk_paged_ragged (and of the table builder) against the oracle.

Both sides receive the same seeded inputs and the same fp32 (cos, sin) table
(built by the oracle), so the comparison isolates the rotation and the
scatter. The GPU table builder is compared with the oracle's table separately.
"""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import (REDUCED, check_rope, gather_logical, gpu_rope, new_token_slots,
                    oracle_rope, oracle_table, raw_bits, to_device)

pytestmark = pytest.mark.gpu


def _run_and_check(wl: W.Workload, in_place: bool = False, tab_np=None):
    sp = wl.spec
    dev = to_device(wl)
    tab_np = oracle_table(wl) if tab_np is None else tab_np
    tab = torch.from_numpy(tab_np).cuda()
    out = gpu_rope(wl, dev, tab, out_q=dev.q if in_place else None)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    q_ref, k_ref = oracle_rope(wl, tab_np)
    check_rope(out, q_ref, wl.q, sp.rotary_dim, sp.interleaved, sp.dtype, "out_q")

    # Cache image: placement, V bytes and untouched slots bit-exact.
    k_img, v_img = O.cache_image(k_ref, wl.v_new, wl.q_offsets, wl.cache_lens, wl.block_table,
                                 wl.k_pages, wl.v_pages)
    kp, vp = raw_bits(dev.cache.k_pages), raw_bits(dev.cache.v_pages)
    assert np.array_equal(vp, v_img.view(vp.dtype)), "V pool differs from the oracle image"
    k_in = raw_bits(wl.k_pages)
    touched = np.any(k_img.view(kp.dtype) != k_in, axis=(2, 3))
    assert np.array_equal(kp[~touched], k_in[~touched]), "untouched K slots changed"
    # Rotated K read back in logical order, within the RoPE tolerance.
    slots = new_token_slots(wl)
    k_got = gather_logical(dev.cache.k_pages.cpu(), wl, slots)
    if k_got.shape[0]:
        check_rope(k_got, k_ref, wl.k_new, sp.rotary_dim, sp.interleaved, sp.dtype, "K cache")
    # Tokens at position 0 are rotated by the identity: bit-exact.
    pos0 = []
    for b, ss in slots:
        for i, s in enumerate(ss):
            t = int(wl.q_offsets[b]) + i
            p = s if wl.position_ids is None else wl.position_ids.reshape(-1, wl.total_tokens)[:, t]
            if np.all(np.asarray(p) == 0):
                pos0.append(t)
    if pos0:
        assert np.array_equal(raw_bits(out)[pos0], raw_bits(wl.q)[pos0])


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_rope_reduced_configs(name):
    _run_and_check(W.make(REDUCED[name], seed=0))


@pytest.mark.parametrize("name", sorted(REDUCED))
def test_rope_other_seeds(name):
    for seed in (1, 2):
        _run_and_check(W.make(REDUCED[name], seed=seed))


@pytest.mark.parametrize("name", ["llama3_8b_decode", "ragged_prefill", "mixed_chunked_mrope",
                                  "tiny_prefill_f32"])
def test_rope_full_size(name):
    _run_and_check(W.make(name, seed=0))


@pytest.mark.slow
def test_rope_full_size_gemma():
    _run_and_check(W.make("gemma_swa_decode", seed=0))


def test_rope_in_place():
    _run_and_check(W.make(REDUCED["mixed_chunked_mrope"], seed=3), in_place=True)


@pytest.mark.parametrize("interleaved", [False, True])
@pytest.mark.parametrize("rotary_dim,head_dim", [(64, 64), (32, 128), (128, 256), (256, 256)])
def test_rope_layouts_and_partial(interleaved, rotary_dim, head_dim):
    sp = W.spec("ragged_prefill", batch=3, new_tokens=("uniform", 1, 70),
                cache_tokens=("uniform", 0, 90), head_dim=head_dim, rotary_dim=rotary_dim,
                interleaved=interleaved, n_heads=6, n_kv_heads=3, page_size=16)
    _run_and_check(W.make(sp, seed=5))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_rope_mrope_and_gaps(dtype):
    sp = W.spec("mixed_chunked_mrope", batch=5, new_tokens=("uniform", 1, 40),
                cache_tokens=("uniform", 0, 100), dtype=dtype, n_heads=8, n_kv_heads=2,
                mrope_section=(8, 28, 28))
    _run_and_check(W.make(sp, seed=6))


def test_freqs_table_matches_oracle():
    for (maxp, R_, theta) in [(40000, 128, 500000.0), (4096, 64, 10000.0), (100, 2, 10000.0)]:
        got = R.freqs_cis(maxp, R_, theta).cpu().numpy()
        want = O.freqs_cis(maxp, R_, theta)
        # both round cos/sin computed in fp64 once to fp32: at most 1 ulp apart
        gi, wi = got.view(np.int32).astype(np.int64), want.view(np.int32).astype(np.int64)
        assert np.max(np.abs(gi - wi)) <= 1
        assert np.mean(gi != wi) < 1e-3


@pytest.mark.parametrize("maxp,d,rot,theta", [(40000, 256, 32, 1e6), (3000, 128, 64, 1e4),
                                              (100, 64, 0, 1e4), (100, 64, 32, 1e4)])
def test_p_rope_table_matches_oracle(maxp, d, rot, theta):
    got = R.freqs_cis_proportional(maxp, d, rot * 2 / d, theta).cpu().numpy()
    want = O.freqs_cis_proportional(maxp, d, rot, theta)
    gi, wi = got.view(np.int32).astype(np.int64), want.view(np.int32).astype(np.int64)
    assert np.max(np.abs(gi - wi)) <= 1
    assert np.array_equal(got[:, 2 * rot:], want[:, 2 * rot:])  # identity pairs exact


@pytest.mark.parametrize("d,rot", [(256, 32), (128, 16)])
def test_p_rope_rotation(d, rot):
    # p-RoPE through the same kernel: half layout, rotary_dim = head_dim and the
    # proportional table; the identity pairs come back bit for bit.
    sp = W.spec("ragged_prefill", batch=3, new_tokens=("uniform", 1, 60),
                cache_tokens=("uniform", 0, 500), head_dim=d, rotary_dim=d, interleaved=False,
                n_heads=8, n_kv_heads=4, page_size=32, theta=1e6)
    wl = W.make(sp, seed=9)
    tab = O.freqs_cis_proportional(wl.max_position, d, rot, sp.theta)
    _run_and_check(wl, tab_np=tab)
    dev = to_device(wl)
    out = gpu_rope(wl, dev, torch.from_numpy(tab).cuda())
    keep = np.r_[rot:d // 2, d // 2 + rot:d]
    assert np.array_equal(raw_bits(out)[..., keep], raw_bits(wl.q)[..., keep])


def test_rope_bad_page_sets_error_bit():
    wl = W.make(REDUCED["llama3_8b_decode"], seed=7)
    wl.block_table[2, :] = wl.num_pages + 5     # sequence 2 points outside the pool
    dev = to_device(wl)
    tab = torch.from_numpy(oracle_table(wl)).cuda()
    out = gpu_rope(wl, dev, tab)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) & R.binding.DEVERR_PAGE
    # the other sequences are unaffected
    q_ref, _ = oracle_rope(wl, oracle_table(wl))
    check_rope(out, q_ref, wl.q, wl.spec.rotary_dim, wl.spec.interleaved, wl.spec.dtype, "out_q")


def test_rope_bad_position_sets_error_bit():
    sp = W.spec("mixed_chunked_mrope", batch=2, new_tokens=("const", 4), cache_tokens=("const", 3),
                n_heads=8, n_kv_heads=2)
    wl = W.make(sp, seed=8)
    wl.position_ids[1, 2] = wl.max_position + 10
    dev = to_device(wl)
    tab = torch.from_numpy(oracle_table(wl)).cuda()
    gpu_rope(wl, dev, tab)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) & R.binding.DEVERR_POSITION
