"""Shared helpers of the GPU parity tests: move a workload to the device, run
the library and the oracle on the same inputs, and compare with the stated
tolerances.

Tolerances (written here once, used by every test):

* RoPE, bf16: an output passes if |got - ref| <= 2 bf16 ulp of |ref|, or
  |got - ref| <= 2^-22 (|a| + |b|) for its pair (a, b) -- twice the fp32
  evaluation bound 2^-23 (|a| + |b|) of a*c - b*s, which governs when the
  result cancels. fp32 mode: 1e-5 relative, with the same cancellation floor
  2^-22 (|a| + |b|).
* Attention: bf16 max-abs 2e-2 and mean-abs 2e-3; fp32 max-abs 1e-4, against
  the oracle's fp64 rows before rounding.
* Log-sum-exp: |got - ref| <= 2e-3 + 1e-4 |ref|, and -inf exactly where the
  row sees no key. It is a smooth maximum of the scores, so its error is at
  most the largest score error plus the relative error of the sum: an fp32
  dot product of d <= 256 terms errs by at most d 2^-24 sum|q_i k_i| (under
  2.5e-3 at scale 1 for the N(0,1)-scale inputs here, far less at
  1/sqrt(d)), and the sum of n fp32 terms with ex2.approx by about
  (n + 2) 2^-23 relative, i.e. 1e-4 |lse| covers it with margin.
* Cache placement, V bytes, untouched slots, channels >= rotary_dim and rows
  at position 0: bit-exact.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

import oracle as O
import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import workloads as W

ATTN_TOL = {"bf16": (2e-2, 2e-3), "f32": (1e-4, 1e-4)}
LSE_TOL = (2e-3, 1e-4)  # absolute, relative


@dataclass
class Dev:
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    offsets: torch.Tensor
    cache_lens: torch.Tensor
    kv_lens: torch.Tensor
    position_ids: torch.Tensor | None
    cache: R.PagedKVCache
    error_word: torch.Tensor


def to_device(wl: W.Workload, device="cuda") -> Dev:
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    f32 = lambda a: None if a is None else torch.from_numpy(
        np.ascontiguousarray(a, dtype=np.float32)).to(device)
    cache = R.PagedKVCache(
        k_pages=wl.k_pages.to(device), v_pages=wl.v_pages.to(device),
        block_table=i32(wl.block_table), cache_lens=i32(wl.cache_lens), error_word=err,
        k_scale=f32(wl.k_scale), v_scale=f32(wl.v_scale))
    return Dev(
        q=wl.q.to(device), k_new=wl.k_new.to(device), v_new=wl.v_new.to(device),
        offsets=i32(wl.q_offsets), cache_lens=i32(wl.cache_lens), kv_lens=i32(wl.kv_lens),
        position_ids=None if wl.position_ids is None else i32(wl.position_ids),
        cache=cache, error_word=err)


def oracle_table(wl: W.Workload) -> np.ndarray:
    sp = wl.spec
    return O.freqs_cis(wl.max_position, sp.rotary_dim, sp.theta)


def gpu_rope(wl: W.Workload, dev: Dev, table: torch.Tensor, out_q=None) -> torch.Tensor:
    sp = wl.spec
    out = torch.empty_like(dev.q) if out_q is None else out_q
    R.rope_qk_paged_ragged(dev.q, dev.offsets, dev.k_new, dev.v_new, dev.cache, table,
                           dev.position_ids, sp.interleaved, sp.rotary_dim, out,
                           mrope_section=sp.mrope_section)
    return out


def oracle_rope(wl: W.Workload, table: np.ndarray):
    sp = wl.spec
    args = (wl.q_offsets, wl.cache_lens, wl.position_ids, sp.mrope_section, table,
            sp.interleaved, sp.rotary_dim)
    return O.rope(wl.q, *args), O.rope(wl.k_new, *args)


def gpu_attention(wl: W.Workload, dev: Dev, q: torch.Tensor, window=None, lse=None, sinks=0):
    sp = wl.spec
    out = torch.empty_like(q)
    R.ragged_paged_attention(q, dev.offsets, dev.kv_lens, dev.cache, sp.n_heads, sp.n_kv_heads,
                             sp.head_dim, sp.softmax_scale, sp.window if window is None else window,
                             out, max_q_len=wl.max_q_len, max_kv_len=wl.max_kv_len,
                             log_sum_exp=lse, sink_tokens=sinks)
    return out


def pair_abs_sum(x: np.ndarray, rotary_dim: int, interleaved: bool) -> np.ndarray:
    """|a| + |b| of the pair each channel belongs to (0 for pass-through channels)."""
    a = np.abs(x)
    out = np.zeros_like(a)
    R_ = rotary_dim
    if interleaved:
        s = a[..., 0:R_:2] + a[..., 1:R_:2]
        out[..., 0:R_:2] = s
        out[..., 1:R_:2] = s
    else:
        s = a[..., :R_ // 2] + a[..., R_ // 2:R_]
        out[..., :R_ // 2] = s
        out[..., R_ // 2:R_] = s
    return out


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return np.exp2(e - 7)


def check_rope(got: torch.Tensor, ref: np.ndarray, x_in, rotary_dim: int, interleaved: bool,
               dtype: str, what: str):
    g = O.widen(got)
    xin = O.widen(x_in)
    ps = pair_abs_sum(xin, rotary_dim, interleaved)
    diff = np.abs(g - ref)
    if dtype == "bf16":
        ok = (diff <= 2 * bf16_ulp(ref)) | (diff <= 2.0 ** -22 * ps)
    else:
        ok = diff <= np.maximum(1e-5 * np.abs(ref), 2.0 ** -22 * ps)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    bad = np.argwhere(~ok)
    assert bad.size == 0, (f"{what}: {len(bad)} outputs outside the RoPE tolerance, first at "
                           f"{bad[0].tolist()}: got {g[tuple(bad[0])]!r} ref {ref[tuple(bad[0])]!r}")
    # channels >= rotary_dim are copies
    assert np.array_equal(g[..., rotary_dim:], xin[..., rotary_dim:]), f"{what}: pass-through"


def check_attention(got: torch.Tensor | np.ndarray, ref: np.ndarray, dtype: str, what: str):
    g = O.widen(got) if isinstance(got, torch.Tensor) else got
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    diff = np.abs(g - ref)
    max_tol, mean_tol = ATTN_TOL[dtype]
    mx, mean = float(diff.max()) if diff.size else 0.0, float(diff.mean()) if diff.size else 0.0
    assert mx <= max_tol, f"{what}: max abs error {mx:.3g} > {max_tol}"
    assert mean <= mean_tol, f"{what}: mean abs error {mean:.3g} > {mean_tol}"
    return mx, mean


def check_lse(got: torch.Tensor | np.ndarray, ref: np.ndarray, what: str):
    g = got.detach().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), empty), f"{what}: -inf rows differ"
    assert np.all(np.isfinite(g[~empty])), f"{what}: non-finite log-sum-exp"
    diff = np.abs(g[~empty] - ref[~empty])
    tol = LSE_TOL[0] + LSE_TOL[1] * np.abs(ref[~empty])
    bad = np.argwhere(diff > tol)
    assert bad.size == 0, (f"{what}: {len(bad)} log-sum-exp values outside tolerance, worst "
                           f"{float((diff - tol).max()):.3g} over")
    return float(diff.max()) if diff.size else 0.0


def gather_logical(pool: torch.Tensor, wl: W.Workload, slots_of) -> torch.Tensor:
    """Rows of a (CPU) pool read in logical order through the block table."""
    P = wl.spec.page_size
    pages, rows = [], []
    for b, t_slots in slots_of:
        for slot in t_slots:
            pages.append(int(wl.block_table[b, slot // P]))
            rows.append(slot % P)
    return pool[torch.tensor(pages, dtype=torch.long), torch.tensor(rows, dtype=torch.long)]


def new_token_slots(wl: W.Workload):
    return [(b, [int(wl.cache_lens[b]) + i for i in range(int(wl.q_lens[b]))])
            for b in range(wl.spec.batch)]


def raw_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.view(torch.int32).numpy()


def sample_rows(wl: W.Workload, n: int, seed: int = 0) -> np.ndarray:
    """(token, head) rows: the first and last row of every sequence for a few heads,
    plus uniformly drawn rows."""
    rng = np.random.default_rng(seed)
    H = wl.spec.n_heads
    rows = []
    for b in range(wl.spec.batch):
        lo, hi = int(wl.q_offsets[b]), int(wl.q_offsets[b + 1])
        if hi > lo:
            for t in {lo, hi - 1, (lo + hi) // 2}:
                rows.append((t, int(rng.integers(0, H))))
                rows.append((t, H - 1))
    T = wl.total_tokens
    extra = max(0, n - len(rows))
    if T:
        rows += list(zip(rng.integers(0, T, extra).tolist(), rng.integers(0, H, extra).tolist()))
    return np.array(rows, dtype=np.int32)


def reduced(name: str, **kw) -> W.Spec:
    return W.spec(name, **kw)


# Reduced versions of the five workloads: same head layouts, dtypes, page
# sizes, RoPE variants and windows; fewer / shorter sequences so that the
# oracle finishes in seconds while still spanning several tiles, pages and
# ragged tails.
REDUCED = {
    "tiny_prefill_f32": W.spec("tiny_prefill_f32"),
    "llama3_8b_decode": W.spec("llama3_8b_decode", batch=6, cache_tokens=("uniform", 40, 700)),
    "ragged_prefill": W.spec("ragged_prefill", batch=3, new_tokens=("uniform", 60, 400)),
    "gemma_swa_decode": W.spec("gemma_swa_decode", batch=3, cache_tokens=("uniform", 900, 2500),
                               window=700),
    "mixed_chunked_mrope": W.spec("mixed_chunked_mrope", batch=4, new_tokens=("uniform", 1, 48),
                                  cache_tokens=("uniform", 0, 300)),
}
