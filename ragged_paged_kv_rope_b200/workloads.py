"""Seeded synthetic inputs for the RoPE + paged-KV + ragged-attention path.

This module only draws inputs: lengths, page tables, position ids and N(0, 1)
values. It holds none of the method's arithmetic (no rotation, no table of
angles, no softmax), so that the fp64 oracle and the CUDA path can both be fed
from it without sharing any code that computes a result.

Layout conventions of the arrays it returns:

* ``q``, ``out_q``           ``[T, n_heads, head_dim]``
* ``k_new``, ``v_new``       ``[T, n_kv_heads, head_dim]``
* ``k_pages``, ``v_pages``   ``[num_pages, page_size, n_kv_heads, head_dim]``
* ``block_table``            ``[batch, max_pages_per_seq]`` int32, -1 where a
  sequence owns no page (never read by a correct kernel)
* ``q_offsets``              ``[batch + 1]`` int32 cumulative row offsets
  (the ``input_row_offsets`` of Mojo's fused QK RoPE kernel and the
  ``query_offsets`` of NumKong's ``attention_packed``)
* ``position_ids``           ``None``, ``[T]``, or ``[3, T]`` with M-RoPE

Values are drawn as float32 N(0, 1) with numpy's PCG64 and narrowed to
bfloat16 by torch's own conversion (round to nearest, ties to even) where the
workload is bf16. Slots of the page pool that hold no token are filled with a
NaN sentinel so that any read of them by a kernel shows up in the result.

With ``cache_dtype="e4m3"`` the pools hold e4m3 codes: one fp32 scale per KV
head for K and one for V, drawn uniformly in [1/64, 1/32] from a separate
seeded stream, and the tokens already in the cache are stored as torch's
float8_e4m3fn conversion of value / scale (the new tokens are q's dtype and
reach the cache through the kernels).
"""

from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field

import numpy as np
import torch

BF16_SENTINEL_BITS = 0x7FC1          # a quiet NaN with a payload
F32_SENTINEL_BITS = 0x7FC01234       # a quiet NaN with a payload
E4M3_SENTINEL_BITS = 0x7F            # the e4m3 NaN code


@dataclass(frozen=True)
class Spec:
    """Shape and distribution of one synthetic workload."""

    name: str
    dtype: str                       # "f32" or "bf16": q/k/v/out and cache dtype
    batch: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    page_size: int
    rotary_dim: int
    theta: float
    interleaved: bool
    window: int                      # <= 0: unbounded
    scale: float | None              # None: 1/sqrt(head_dim)
    new_tokens: tuple                # ("fixed", [..]) | ("const", n) | ("uniform", lo, hi)
    cache_tokens: tuple              # same forms
    position_gaps: int | None = None # max random gap between consecutive positions
    mrope_section: tuple | None = None
    rms_norm: bool = False           # RMS-normalise q, k_new and cached K per head
    spare_pages: int = 8
    cache_dtype: str | None = None   # None: dtype; "e4m3": codes of value / per-head scale
    description: str = ""

    @property
    def softmax_scale(self) -> float:
        return (1.0 / math.sqrt(self.head_dim)) if self.scale is None else float(self.scale)


# The five workloads, named by what they are.
SPECS: dict[str, Spec] = {
    "tiny_prefill_f32": Spec(
        name="tiny_prefill_f32", dtype="f32", batch=2, n_heads=4, n_kv_heads=2,
        head_dim=64, page_size=16, rotary_dim=64, theta=10000.0, interleaved=False,
        window=0, scale=None, new_tokens=("fixed", [5, 11]), cache_tokens=("const", 0),
        description="2 sequences of 5 and 11 tokens, 4 q heads, 2 kv heads, d=64, "
                    "page 16, half RoPE theta 1e4, causal, fp32"),
    "llama3_8b_decode": Spec(
        name="llama3_8b_decode", dtype="bf16", batch=64, n_heads=32, n_kv_heads=8,
        head_dim=128, page_size=64, rotary_dim=128, theta=500000.0, interleaved=False,
        window=0, scale=None, new_tokens=("const", 1), cache_tokens=("uniform", 512, 8192),
        description="batch 64 decode, 32 q heads, 8 kv heads, d=128, cached context "
                    "U[512, 8192], page 64, half RoPE theta 5e5, bf16"),
    "ragged_prefill": Spec(
        name="ragged_prefill", dtype="bf16", batch=16, n_heads=32, n_kv_heads=8,
        head_dim=128, page_size=64, rotary_dim=128, theta=500000.0, interleaved=False,
        window=0, scale=None, new_tokens=("uniform", 128, 4096), cache_tokens=("const", 0),
        description="16 sequences of U[128, 4096] tokens into an empty cache, 32 q heads, "
                    "8 kv heads, d=128, page 64, half RoPE theta 5e5, causal, bf16"),
    "gemma_swa_decode": Spec(
        name="gemma_swa_decode", dtype="bf16", batch=8, n_heads=16, n_kv_heads=8,
        head_dim=256, page_size=128, rotary_dim=128, theta=10000.0, interleaved=True,
        window=4096, scale=1.0, new_tokens=("const", 1), cache_tokens=("const", 32768),
        rms_norm=True,
        description="batch 8 decode over 32768 cached tokens, window 4096, 16 q heads, "
                    "8 kv heads, d=256, interleaved partial RoPE R=128 theta 1e4, "
                    "scale 1.0 with RMS-normalised q/k, page 128, bf16"),
    "mixed_chunked_mrope": Spec(
        name="mixed_chunked_mrope", dtype="bf16", batch=32, n_heads=64, n_kv_heads=8,
        head_dim=128, page_size=64, rotary_dim=128, theta=10000.0, interleaved=False,
        window=0, scale=None, new_tokens=("uniform", 1, 512), cache_tokens=("uniform", 0, 16384),
        position_gaps=3, mrope_section=(16, 24, 24),
        description="batch 32, U[1, 512] new tokens onto U[0, 16384] cached, 64 q heads, "
                    "8 kv heads, d=128, M-RoPE sections [16, 24, 24] pairs with position "
                    "gaps of 0-3, page 64, causal, bf16"),
}


def spec(name: str, **overrides) -> Spec:
    """A named spec, optionally with some fields replaced (for reduced sizes)."""
    return dataclasses.replace(SPECS[name], **overrides)


@dataclass
class Workload:
    spec: Spec
    seed: int
    q_lens: np.ndarray
    cache_lens: np.ndarray
    kv_lens: np.ndarray
    q_offsets: np.ndarray
    block_table: np.ndarray
    num_pages: int
    position_ids: np.ndarray | None
    max_position: int
    q: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    k_pages: torch.Tensor
    v_pages: torch.Tensor
    extra: dict = field(default_factory=dict)
    k_scale: np.ndarray | None = None   # fp32 [n_kv_heads] of an e4m3 cache
    v_scale: np.ndarray | None = None

    @property
    def total_tokens(self) -> int:
        return int(self.q_offsets[-1])

    @property
    def max_q_len(self) -> int:
        return int(self.q_lens.max()) if len(self.q_lens) else 0

    @property
    def max_kv_len(self) -> int:
        return int(self.kv_lens.max()) if len(self.kv_lens) else 0

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.block_table.shape[1])


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _draw(rng: np.random.Generator, form: tuple, n: int) -> np.ndarray:
    kind = form[0]
    if kind == "fixed":
        vals = np.asarray(form[1], dtype=np.int64)
        assert len(vals) == n, (form, n)
        return vals
    if kind == "const":
        return np.full(n, int(form[1]), dtype=np.int64)
    if kind == "uniform":
        return rng.integers(int(form[1]), int(form[2]), size=n, endpoint=True)
    raise ValueError(form)


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _rms_normalise(x: np.ndarray) -> np.ndarray:
    # Input shaping only (unit-weight RMSNorm per head row, eps 1e-6): the
    # values the attention sees are then of unit RMS, as after a QK-norm.
    ms = np.mean(np.square(x, dtype=np.float32), axis=-1, keepdims=True, dtype=np.float32)
    return (x / np.sqrt(ms + np.float32(1e-6))).astype(np.float32)


def _narrow(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch_dtype(dtype))


def sentinel_pool(num_pages: int, page_size: int, n_kv_heads: int, head_dim: int,
                  dtype: str) -> torch.Tensor:
    """A pool whose every slot holds the NaN sentinel."""
    shape = (num_pages, page_size, n_kv_heads, head_dim)
    if dtype == "e4m3":
        return torch.full(shape, E4M3_SENTINEL_BITS, dtype=torch.uint8).view(torch.float8_e4m3fn)
    if dtype == "bf16":
        bits = torch.full(shape, BF16_SENTINEL_BITS, dtype=torch.int16)
        return bits.view(torch.bfloat16)
    bits = torch.full(shape, F32_SENTINEL_BITS, dtype=torch.int32)
    return bits.view(torch.float32)


def _cache_scales(sp: Spec, seed: int):
    """Per-KV-head (k_scale, v_scale) of an e4m3 cache, else (None, None)."""
    if sp.cache_dtype != "e4m3":
        return None, None
    srng = np.random.default_rng([seed, 0xE4])
    ks = srng.uniform(1.0 / 64, 1.0 / 32, size=sp.n_kv_heads).astype(np.float32)
    vs = srng.uniform(1.0 / 64, 1.0 / 32, size=sp.n_kv_heads).astype(np.float32)
    return ks, vs


def _cache_rows(x: np.ndarray, sp: Spec, scale: np.ndarray | None) -> torch.Tensor:
    """Rows [n, Hk, d] as stored in the cache: q's dtype, or e4m3 codes of x / scale."""
    if scale is None:
        return _narrow(x, sp.dtype)
    q = (x / scale[None, :, None]).astype(np.float32)
    return torch.from_numpy(np.ascontiguousarray(q)).to(torch.float8_e4m3fn)


def make(spec_or_name, seed: int = 0, **overrides) -> Workload:
    """Draw one workload. Same (spec, seed) gives the same arrays bit for bit."""
    sp = spec(spec_or_name, **overrides) if isinstance(spec_or_name, str) else \
        dataclasses.replace(spec_or_name, **overrides)
    rng = np.random.default_rng(seed)
    B = sp.batch
    q_lens = _draw(rng, sp.new_tokens, B)
    cache_lens = _draw(rng, sp.cache_tokens, B)
    kv_lens = cache_lens + q_lens
    q_offsets = np.zeros(B + 1, dtype=np.int64)
    q_offsets[1:] = np.cumsum(q_lens)
    T = int(q_offsets[-1])
    P = sp.page_size

    # Page table: each sequence owns ceil(kv_len / P) pages of a shuffled pool.
    pages_per_seq = (kv_lens + P - 1) // P
    num_pages = int(pages_per_seq.sum()) + sp.spare_pages
    perm = rng.permutation(num_pages)
    max_pages = max(1, int(pages_per_seq.max()) if B else 1)
    block_table = np.full((B, max_pages), -1, dtype=np.int64)
    cursor = 0
    for b in range(B):
        n = int(pages_per_seq[b])
        block_table[b, :n] = perm[cursor:cursor + n]
        cursor += n

    # Positions: implicit (cache_len + i) unless random gaps are asked for; with
    # M-RoPE each of the three sections draws its own gaps.
    position_ids = None
    max_position = int(kv_lens.max()) if B else 1
    if sp.position_gaps is not None:
        n_sec = 3 if sp.mrope_section is not None else 1
        pos = np.zeros((n_sec, T), dtype=np.int64)
        for s in range(n_sec):
            for b in range(B):
                lo, n = int(q_offsets[b]), int(q_lens[b])
                if n == 0:
                    continue
                gaps = rng.integers(0, sp.position_gaps, size=n - 1, endpoint=True)
                steps = np.concatenate([[0], np.cumsum(1 + gaps)])
                pos[s, lo:lo + n] = int(cache_lens[b]) + steps
        position_ids = pos if n_sec == 3 else pos[0]
        if T:
            max_position = max(max_position, int(pos.max()) + 1)

    H, Hk, d = sp.n_heads, sp.n_kv_heads, sp.head_dim
    q = _normal(rng, (T, H, d))
    k_new = _normal(rng, (T, Hk, d))
    v_new = _normal(rng, (T, Hk, d))
    if sp.rms_norm:
        q = _rms_normalise(q)
        k_new = _rms_normalise(k_new)

    ks, vs = _cache_scales(sp, seed)
    k_pages = sentinel_pool(num_pages, P, Hk, d, sp.cache_dtype or sp.dtype)
    v_pages = sentinel_pool(num_pages, P, Hk, d, sp.cache_dtype or sp.dtype)
    # Tokens already in the cache: N(0, 1) in slots [0, cache_len) of each sequence.
    for b in range(B):
        n = int(cache_lens[b])
        if n == 0:
            continue
        kc = _normal(rng, (n, Hk, d))
        vc = _normal(rng, (n, Hk, d))
        if sp.rms_norm:
            kc = _rms_normalise(kc)
        kc_t = _cache_rows(kc, sp, ks)
        vc_t = _cache_rows(vc, sp, vs)
        for pg in range((n + P - 1) // P):
            page = int(block_table[b, pg])
            rows = min(P, n - pg * P)
            k_pages[page, :rows] = kc_t[pg * P: pg * P + rows]
            v_pages[page, :rows] = vc_t[pg * P: pg * P + rows]

    return Workload(
        spec=sp, seed=seed,
        q_lens=q_lens.astype(np.int32), cache_lens=cache_lens.astype(np.int32),
        kv_lens=kv_lens.astype(np.int32), q_offsets=q_offsets.astype(np.int32),
        block_table=block_table.astype(np.int32), num_pages=num_pages,
        position_ids=None if position_ids is None else position_ids.astype(np.int32),
        max_position=max_position,
        q=_narrow(q, sp.dtype), k_new=_narrow(k_new, sp.dtype), v_new=_narrow(v_new, sp.dtype),
        k_pages=k_pages, v_pages=v_pages, k_scale=ks, v_scale=vs)


def attention_only(sp: Spec, seed: int, q_lens, kv_lens) -> Workload:
    """A workload for attention alone: q and a fully populated cache.

    Every slot below kv_len holds an N(0, 1) key and value; q is drawn as if
    already rotated. Used to test attention without going through RoPE.
    """
    rng = np.random.default_rng(seed)
    q_lens = np.asarray(q_lens, dtype=np.int64)
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    B = len(q_lens)
    sp = dataclasses.replace(sp, batch=B)
    q_offsets = np.zeros(B + 1, dtype=np.int64)
    q_offsets[1:] = np.cumsum(q_lens)
    T = int(q_offsets[-1])
    P = sp.page_size
    pages_per_seq = (kv_lens + P - 1) // P
    num_pages = int(pages_per_seq.sum()) + sp.spare_pages
    perm = rng.permutation(num_pages)
    max_pages = max(1, int(pages_per_seq.max()) if B else 1)
    block_table = np.full((B, max_pages), -1, dtype=np.int64)
    cursor = 0
    for b in range(B):
        n = int(pages_per_seq[b])
        block_table[b, :n] = perm[cursor:cursor + n]
        cursor += n
    H, Hk, d = sp.n_heads, sp.n_kv_heads, sp.head_dim
    q = _normal(rng, (T, H, d))
    if sp.rms_norm:
        q = _rms_normalise(q)
    ks, vs = _cache_scales(sp, seed)
    k_pages = sentinel_pool(num_pages, P, Hk, d, sp.cache_dtype or sp.dtype)
    v_pages = sentinel_pool(num_pages, P, Hk, d, sp.cache_dtype or sp.dtype)
    for b in range(B):
        n = int(kv_lens[b])
        if n == 0:
            continue
        kc = _normal(rng, (n, Hk, d))
        vc = _normal(rng, (n, Hk, d))
        if sp.rms_norm:
            kc = _rms_normalise(kc)
        kc_t, vc_t = _cache_rows(kc, sp, ks), _cache_rows(vc, sp, vs)
        for pg in range((n + P - 1) // P):
            page = int(block_table[b, pg])
            rows = min(P, n - pg * P)
            k_pages[page, :rows] = kc_t[pg * P: pg * P + rows]
            v_pages[page, :rows] = vc_t[pg * P: pg * P + rows]
    empty = torch.zeros((0,))
    return Workload(
        spec=sp, seed=seed,
        q_lens=q_lens.astype(np.int32), cache_lens=(kv_lens - q_lens).astype(np.int32),
        kv_lens=kv_lens.astype(np.int32), q_offsets=q_offsets.astype(np.int32),
        block_table=block_table.astype(np.int32), num_pages=num_pages,
        position_ids=None, max_position=int(kv_lens.max()) if B else 1,
        q=_narrow(q, sp.dtype), k_new=empty, v_new=empty,
        k_pages=k_pages, v_pages=v_pages, k_scale=ks, v_scale=vs)
