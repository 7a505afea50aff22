"""GPU parity of ragged_paged_attention_backward against the fp64 oracle.

The GPU forward runs first (output and log-sum-exp), then the backward with a
seeded N(0, 1) output gradient; the oracle computes the gradients from the same
q, output gradient and pools by the definition (exact D_i and P_ij). The
kernel takes D_i = d_out_i . out_i from the forward's rounded output and P_ij
from its fp32 log-sum-exp, as the API defines, so the comparison is relative
to each gradient's scale: for bf16, max |got - ref| <= 2e-2 max|ref| and
mean |got - ref| <= 2e-3 max|ref| (the output's bf16 rounding, 2^-9, enters
D_i and so every dS_ij; the tensor-core kernels also round P_ij and dS_ij to
bf16, relative 2^-9, as operands of their second products); for fp32,
1e-4 max|ref|.

bf16 shapes run on the tensor-core kernels: tcgen05 for head_dim 64 / 128
with groups of up to 64 query heads, warp-level mma.sync for head_dim 256
with groups of up to 16. The others (fp32, an e4m3 cache, larger groups)
run on the CUDA-core ones. The cases cover all three, several key tiles and
row blocks with ragged tails, windows with sinks across tiles, groups that
do not divide 64, and rows that see no key.
"""

import numpy as np
import pytest
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W
from parity import to_device

pytestmark = pytest.mark.gpu

TOL = {"bf16": (2e-2, 2e-3), "f32": (1e-4, 1e-5)}


def _check(got: torch.Tensor, ref: np.ndarray, dtype: str, what: str):
    g = got.detach().cpu().double().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    assert scale > 0.0, f"{what}: reference is identically zero"
    diff = np.abs(g - ref)
    mx_tol, mean_tol = TOL[dtype]
    assert diff.max() <= mx_tol * scale, f"{what}: max error {diff.max():.3g} vs scale {scale:.3g}"
    assert diff.mean() <= mean_tol * scale, f"{what}: mean error {diff.mean():.3g}"


CASES = [
    # (description, spec name, overrides, q_lens, kv_lens, window, sinks)
    ("prefill bf16", "ragged_prefill", dict(n_heads=8, n_kv_heads=2, page_size=32),
     [37, 5, 70], [37, 60, 70], 0, 0),
    ("decode bf16", "llama3_8b_decode", dict(n_heads=8, n_kv_heads=2), [1, 1, 1],
     [300, 64, 1000], 0, 0),
    ("window and sinks", "ragged_prefill", dict(n_heads=4, n_kv_heads=2, page_size=16),
     [40, 20], [90, 20], 17, 3),
    ("head_dim 256 window", "gemma_swa_decode", dict(n_heads=4, n_kv_heads=2), [2, 1],
     [600, 300], 128, 0),
    ("head_dim 64", "ragged_prefill", dict(n_heads=4, n_kv_heads=1, head_dim=64, rotary_dim=64),
     [33, 9], [33, 40], 0, 0),
    ("fp32", "tiny_prefill_f32", {}, [5, 11], [5, 11], 0, 0),
    ("e4m3 cache", "llama3_8b_decode", dict(n_heads=8, n_kv_heads=2, cache_dtype="e4m3"),
     [3, 1], [200, 90], 0, 0),
    ("tiles and ragged tails", "ragged_prefill", dict(n_heads=8, n_kv_heads=2, page_size=64),
     [200, 64, 1], [330, 64, 129], 0, 0),
    ("window and sinks across tiles", "ragged_prefill",
     dict(n_heads=8, n_kv_heads=2, page_size=32), [150, 30], [400, 100], 70, 5),
    ("group of 3", "ragged_prefill", dict(n_heads=6, n_kv_heads=2), [50, 7], [120, 7], 0, 0),
    ("group of 16", "ragged_prefill",
     dict(n_heads=16, n_kv_heads=1, head_dim=64, rotary_dim=64), [9, 20], [70, 20], 0, 0),
    ("group of 32", "ragged_prefill",
     dict(n_heads=32, n_kv_heads=1, head_dim=64, rotary_dim=64), [3, 5], [50, 5], 0, 0),
    ("rows without keys", "ragged_prefill", dict(n_heads=4, n_kv_heads=2), [12, 3], [5, 40],
     0, 0),
    ("head_dim 256 prefill, window and sinks", "gemma_swa_decode",
     dict(n_heads=4, n_kv_heads=2), [100, 1], [300, 77], 128, 4),
    ("many 128-key and 128-row blocks", "ragged_prefill",
     dict(n_heads=8, n_kv_heads=2, page_size=64), [700, 129, 3], [900, 129, 260], 0, 0),
    ("group of 8, chunked rows, window", "mixed_chunked_mrope",
     dict(n_heads=16, n_kv_heads=2, mrope_section=None), [150, 1, 40], [1000, 300, 41], 300, 0),
    ("group of 128 (CUDA cores), one token per row block", "ragged_prefill",
     dict(n_heads=128, n_kv_heads=1, head_dim=64, rotary_dim=64, page_size=128), [5, 2],
     [300, 2], 0, 0),
]


@pytest.mark.parametrize("idx", range(len(CASES)))
def test_backward_matches_oracle(idx):
    desc, name, over, q_lens, kv_lens, window, sinks = CASES[idx]
    sp = W.spec(name, **over)
    wl = W.attention_only(sp, 10 + idx, q_lens, kv_lens)
    dev = to_device(wl)
    T, H, d = wl.q.shape
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    out = torch.empty_like(dev.q)
    R.ragged_paged_attention(dev.q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads,
                             sp.n_kv_heads, sp.head_dim, sp.softmax_scale, window, out,
                             max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len, log_sum_exp=lse,
                             sink_tokens=sinks)
    rng = np.random.default_rng(idx)
    d_out = torch.from_numpy(rng.standard_normal((T, H, d), dtype=np.float32)).to(
        wl.q.dtype).cuda()
    d_q = torch.full((T, H, d), float("nan"), device="cuda")
    pool = tuple(dev.cache.k_pages.shape)
    d_k = torch.zeros(pool, dtype=torch.float32, device="cuda")
    d_v = torch.zeros(pool, dtype=torch.float32, device="cuda")
    R.ragged_paged_attention_backward(dev.q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads,
                                      sp.n_kv_heads, sp.head_dim, sp.softmax_scale, window, out,
                                      d_out, lse, d_q, d_k, d_v, max_q_len=wl.max_q_len,
                                      max_kv_len=wl.max_kv_len, sink_tokens=sinks)
    torch.cuda.synchronize()
    assert int(dev.error_word.item()) == 0
    rq, rk, rv = O.attention_backward(wl.q, d_out.cpu(), wl.q_offsets, wl.kv_lens, wl.k_pages,
                                      wl.v_pages, wl.block_table, sp.n_kv_heads,
                                      sp.softmax_scale, window, sinks, k_scale=wl.k_scale,
                                      v_scale=wl.v_scale)
    _check(d_q, rq, sp.dtype, f"{desc}: d_q")
    _check(d_k, rk, sp.dtype, f"{desc}: d_k")
    _check(d_v, rv, sp.dtype, f"{desc}: d_v")
