"""ctypes binding of librpk.so (declared in include/rpk.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, turned into raw pointers and sizes, and handed to the C ABI, whose
CUDA kernels do every step of the path. There is no CPU fallback: a missing
library, a CPU tensor or a non-zero status raises.

Entry points keep the C names:

* ``rope_qk_paged_ragged``  fused RoPE on Q and new K, K/V written into the cache
* ``ragged_paged_attention`` ragged causal GQA attention over the paged cache
* ``ragged_paged_attention_backward`` its query, key and value gradients
* ``ragged_paged_attention_workspace_size``
* ``freqs_cis``             builds the fp32 (cos, sin) table with ``rope_freqs_cis``
* ``freqs_cis_proportional`` builds the p-RoPE table with ``rope_freqs_cis_proportional``
* ``ragged_paged_attention_noalloc`` the decode path with library-owned scratch
* ``set_wait_limit_ns`` / ``wait_limit_ns`` the bound of the kernels' device-side waits
"""

from __future__ import annotations

import ctypes as C
import math
import os
import re
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librpk.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "rpk.h")

RPK_F32, RPK_BF16, RPK_E4M3 = 0, 1, 2
STATUS = {0: "RPK_OK", 1: "RPK_ERR_NULL", 2: "RPK_ERR_SHAPE", 3: "RPK_ERR_DTYPE",
          4: "RPK_ERR_UNSUPPORTED", 5: "RPK_ERR_CUDA", 6: "RPK_ERR_WORKSPACE"}
DEVERR_PAGE, DEVERR_POSITION, DEVERR_LENGTH, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8


class RpkError(RuntimeError):
    """A non-zero status from the C ABI (``.status`` holds the code)."""

    def __init__(self, msg: str, status: int | None = None):
        super().__init__(msg)
        self.status = status


class PagedKV(C.Structure):
    """Mirror of rpk_paged_kv."""

    _fields_ = [
        ("k_pages", C.c_void_p), ("v_pages", C.c_void_p),
        ("num_pages", C.c_int32), ("page_size", C.c_int32),
        ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32),
        ("cache_dtype", C.c_int),
        ("block_table", C.c_void_p), ("max_pages_per_seq", C.c_int32), ("batch", C.c_int32),
        ("cache_lens", C.c_void_p), ("error_word", C.c_void_p),
        ("num_layers", C.c_int32), ("layer_idx", C.c_int32),
        ("k_scale", C.c_void_p), ("v_scale", C.c_void_p),
    ]


_lib = None


def lib():
    """The loaded librpk.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RpkError(f"librpk.so is not built ({LIB_PATH}); run "
                           "python -m ragged_paged_kv_rope_b200.build")
        L = C.CDLL(LIB_PATH)
        _p, _i32 = C.c_void_p, C.c_int32
        L.rope_qk_paged_ragged.argtypes = [_p, _p, _p, _p, C.POINTER(PagedKV), _p, _p, _i32, _i32,
                                           _p, _i32, _i32, C.c_int, _i32, _p, _p]
        L.rope_qk_paged_ragged.restype = C.c_int
        L.rope_freqs_cis.argtypes = [_p, _i32, _i32, C.c_double, _p]
        L.rope_freqs_cis.restype = C.c_int
        L.ragged_paged_attention_workspace_size.argtypes = [_i32] * 6
        L.ragged_paged_attention_workspace_size.restype = C.c_size_t
        L.ragged_paged_attention.argtypes = [_p, _p, _p, C.POINTER(PagedKV), _i32, _i32, _i32,
                                             C.c_float, _i32, _p, _i32, _i32, _i32, _i32, C.c_int,
                                             _p, C.c_size_t, _p, _i32, _p]
        L.ragged_paged_attention.restype = C.c_int
        L.rope_freqs_cis_proportional.argtypes = [_p, _i32, _i32, _i32, C.c_double, _p]
        L.rope_freqs_cis_proportional.restype = C.c_int
        L.rpk_status_string.argtypes = [C.c_int]
        L.rpk_status_string.restype = C.c_char_p
        L.rpk_last_cuda_error.argtypes = []
        L.rpk_last_cuda_error.restype = C.c_char_p
        L.rpk_set_wait_limit_ns.argtypes = [C.c_uint64]
        L.rpk_set_wait_limit_ns.restype = None
        L.rpk_wait_limit_ns.argtypes = []
        L.rpk_wait_limit_ns.restype = C.c_uint64
        _lib = L
    return _lib


def header_symbols() -> list[str]:
    """Names of the functions include/rpk.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:rpk_status|size_t|const char\*|void|uint64_t)\s+(\w+)\s*\(", text,
                      flags=re.M)


def _check(status: int):
    if status != 0:
        L = lib()
        msg = L.rpk_status_string(status).decode()
        if status == 5:
            msg += f" ({L.rpk_last_cuda_error().decode()})"
        raise RpkError(f"{STATUS.get(status, status)}: {msg}", status)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return RPK_BF16
    if t == torch.float32:
        return RPK_F32
    raise RpkError(f"unsupported dtype {t}")


def _cache_dtype_code(t: torch.dtype) -> int:
    """Cache pools may also hold e4m3 codes (torch.float8_e4m3fn or raw uint8)."""
    if t in (torch.float8_e4m3fn, torch.uint8):
        return RPK_E4M3
    return _dtype_code(t)


def _dev(t: torch.Tensor, name: str, dtype=None, ndim=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise RpkError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise RpkError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise RpkError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise RpkError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise RpkError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


@dataclass
class PagedKVCache:
    """The paged cache: pools, block table, cached lengths, optional error word.

    The pools are [num_pages, page_size, n_kv_heads, head_dim], or, for a
    multi-layer collection, [num_layers, num_pages, page_size, n_kv_heads,
    head_dim] with layer_idx choosing the layer the calls read and write.
    Pools of torch.float8_e4m3fn (or raw uint8) hold e4m3 codes of x / scale,
    with k_scale / v_scale the fp32 [n_kv_heads] scales of K and V.
    """

    k_pages: torch.Tensor
    v_pages: torch.Tensor
    block_table: torch.Tensor      # int32 [batch, max_pages_per_seq]
    cache_lens: torch.Tensor | None = None   # int32 [batch]
    error_word: torch.Tensor | None = None   # int32 [1]
    layer_idx: int = 0
    k_scale: torch.Tensor | None = None      # fp32 [n_kv_heads], e4m3 pools only
    v_scale: torch.Tensor | None = None

    def struct(self) -> PagedKV:
        kp, vp = self.k_pages, self.v_pages
        if kp.dim() not in (4, 5):
            raise RpkError("k_pages must be [(num_layers,) num_pages, page_size, kv_heads, d]")
        _dev(kp, "k_pages", ndim=kp.dim())
        _dev(vp, "v_pages", dtype=kp.dtype, ndim=kp.dim())
        if vp.shape != kp.shape:
            raise RpkError("k_pages and v_pages differ in shape")
        _dev(self.block_table, "block_table", torch.int32, 2)
        s = PagedKV()
        s.k_pages, s.v_pages = kp.data_ptr(), vp.data_ptr()
        shape = tuple(int(x) for x in kp.shape)
        s.num_layers = shape[0] if len(shape) == 5 else 1
        s.layer_idx = int(self.layer_idx)
        s.num_pages, s.page_size, s.n_kv_heads, s.head_dim = shape[-4:]
        s.cache_dtype = _cache_dtype_code(kp.dtype)
        if s.cache_dtype == RPK_E4M3:
            if self.k_scale is None or self.v_scale is None:
                raise RpkError("an e4m3 cache needs k_scale and v_scale")
            s.k_scale = _dev(self.k_scale, "k_scale", torch.float32, 1)
            s.v_scale = _dev(self.v_scale, "v_scale", torch.float32, 1)
        s.block_table = self.block_table.data_ptr()
        s.batch, s.max_pages_per_seq = (int(x) for x in self.block_table.shape)
        s.cache_lens = (_dev(self.cache_lens, "cache_lens", torch.int32, 1)
                        if self.cache_lens is not None else None)
        s.error_word = (_dev(self.error_word, "error_word", torch.int32)
                        if self.error_word is not None else None)
        return s


def rope_qk_paged_ragged(q_proj, input_row_offsets, k_new, v_new, page_table: PagedKVCache,
                         freqs_cis, position_ids, interleaved: bool, rotary_dim: int, out_q, *,
                         mrope_section=None, stream=None) -> None:
    """Rotate q_proj into out_q and k_new into the cache; copy v_new into the cache."""
    pk = page_table.struct()
    T, H, d = (int(x) for x in q_proj.shape) if q_proj.dim() == 3 else (None,) * 3
    if T is None:
        raise RpkError("q_proj must be [tokens, n_heads, head_dim]")
    qp = _dev(q_proj, "q_proj")
    kn = _dev(k_new, "k_new", q_proj.dtype, 3)
    vn = _dev(v_new, "v_new", q_proj.dtype, 3)
    oq = _dev(out_q, "out_q", q_proj.dtype, 3)
    if tuple(out_q.shape) != tuple(q_proj.shape):
        raise RpkError("out_q must have q_proj's shape")
    if k_new.shape[0] != T or v_new.shape != k_new.shape:
        raise RpkError("k_new / v_new must be [tokens, n_kv_heads, head_dim]")
    off = _dev(input_row_offsets, "input_row_offsets", torch.int32, 1)
    fc = _dev(freqs_cis, "freqs_cis", torch.float32, 2)
    if int(freqs_cis.shape[1]) != int(rotary_dim):
        raise RpkError("freqs_cis must be [max_position, rotary_dim]")
    pid = None
    if position_ids is not None:
        pid = _dev(position_ids, "position_ids", torch.int32)
        want = (3, T) if mrope_section is not None else (T,)
        if tuple(position_ids.shape) != want:
            raise RpkError(f"position_ids must be {want}, got {tuple(position_ids.shape)}")
    ms = None
    if mrope_section is not None:
        ms_arr = (C.c_int32 * 3)(*[int(x) for x in mrope_section])
        ms = C.cast(ms_arr, C.c_void_p)
    _check(lib().rope_qk_paged_ragged(
        qp, off, kn, vn, C.byref(pk), fc, pid, int(bool(interleaved)), int(rotary_dim), oq, T, H,
        _dtype_code(q_proj.dtype), int(freqs_cis.shape[0]), ms, _stream(stream)))


def freqs_cis(max_position: int, rotary_dim: int, theta: float, device=None,
              stream=None) -> torch.Tensor:
    """fp32 [max_position, rotary_dim] table of (cos, sin) of p * theta^(-2j/R)."""
    device = device if device is not None else torch.device("cuda")
    out = torch.empty((int(max_position), int(rotary_dim)), dtype=torch.float32, device=device)
    _check(lib().rope_freqs_cis(out.data_ptr(), int(max_position), int(rotary_dim), float(theta),
                                _stream(stream)))
    return out


def freqs_cis_proportional(max_position: int, head_dim: int, factor: float, theta: float,
                           device=None, stream=None) -> torch.Tensor:
    """fp32 [max_position, head_dim] p-RoPE table (rope_half_proportional): the first
    floor(factor * head_dim / 2) rotate-half pairs turn by p * theta^(-2j/head_dim),
    the others are the identity. Use with rotary_dim = head_dim, interleaved False."""
    rotated = int(math.floor(float(factor) * int(head_dim) / 2))
    device = device if device is not None else torch.device("cuda")
    out = torch.empty((int(max_position), int(head_dim)), dtype=torch.float32, device=device)
    _check(lib().rope_freqs_cis_proportional(out.data_ptr(), int(max_position), int(head_dim),
                                             rotated, float(theta), _stream(stream)))
    return out


def ragged_paged_attention_workspace_size(total_q_tokens: int, n_heads: int, head_dim: int,
                                          batch: int, max_kv_len: int, page_size: int) -> int:
    return int(lib().ragged_paged_attention_workspace_size(
        int(total_q_tokens), int(n_heads), int(head_dim), int(batch), int(max_kv_len),
        int(page_size)))


def ragged_paged_attention(q, q_row_offsets, kv_lens, page_table: PagedKVCache, n_heads: int,
                           n_kv_heads: int, head_dim: int, scale: float | None, window: int,
                           out, *, max_q_len: int, max_kv_len: int, workspace=None,
                           log_sum_exp=None, sink_tokens: int = 0, stream=None) -> None:
    """Ragged causal (windowed) GQA attention of q over the paged cache into out.

    max_q_len / max_kv_len are host-side bounds of the device lengths (they
    size the launch). workspace: a uint8 CUDA tensor of at least
    ragged_paged_attention_workspace_size(...) bytes, or None to have one
    allocated here with torch. log_sum_exp: None, or a float32 CUDA tensor
    [tokens, n_heads] that receives each row's natural log-sum-exp of its
    scores (-inf for a row that sees no key). sink_tokens: under a window, the
    first sink_tokens keys of every sequence stay visible (attention sinks).
    """
    pk = page_table.struct()
    if q.dim() != 3:
        raise RpkError("q must be [tokens, n_heads, head_dim]")
    T = int(q.shape[0])
    qp = _dev(q, "q")
    op = _dev(out, "out", q.dtype, 3)
    if tuple(out.shape) != tuple(q.shape):
        raise RpkError("out must have q's shape")
    off = _dev(q_row_offsets, "q_row_offsets", torch.int32, 1)
    kvl = _dev(kv_lens, "kv_lens", torch.int32, 1)
    batch = int(kv_lens.shape[0])
    if scale is None:
        scale = float(head_dim) ** -0.5
    need = ragged_paged_attention_workspace_size(T, n_heads, head_dim, batch, max_kv_len,
                                                 pk.page_size)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws, ws_bytes = None, 0
    if workspace is not None:
        ws = _dev(workspace, "workspace", torch.uint8)
        ws_bytes = workspace.numel()
    lp = None
    if log_sum_exp is not None:
        lp = _dev(log_sum_exp, "log_sum_exp", torch.float32, 2)
        if tuple(log_sum_exp.shape) != (T, int(n_heads)):
            raise RpkError("log_sum_exp must be [tokens, n_heads]")
    _check(lib().ragged_paged_attention(
        qp, off, kvl, C.byref(pk), int(n_heads), int(n_kv_heads), int(head_dim), float(scale),
        int(window), op, batch, T, int(max_q_len), int(max_kv_len), _dtype_code(q.dtype), ws,
        ws_bytes, lp, int(sink_tokens), _stream(stream)))


def ragged_paged_attention_backward(q, q_row_offsets, kv_lens, page_table: PagedKVCache,
                                    n_heads: int, n_kv_heads: int, head_dim: int,
                                    scale: float | None, window: int, out, d_out, log_sum_exp,
                                    d_q, d_k_pages, d_v_pages, *, max_q_len: int, max_kv_len: int,
                                    sink_tokens: int = 0, stream=None) -> None:
    """Gradients of ragged_paged_attention: d_q [tokens, n_heads, head_dim] and the
    pool-shaped d_k_pages / d_v_pages (float32) from the forward's out and
    log_sum_exp and the output gradient d_out. Entries of d_k_pages / d_v_pages
    that hold no key of any sequence are left as they were."""
    L = lib()
    fn = L.ragged_paged_attention_backward
    if fn.argtypes is None:
        _p, _i32 = C.c_void_p, C.c_int32
        fn.argtypes = [_p, _p, _p, C.POINTER(PagedKV), _i32, _i32, _i32, C.c_float, _i32, _p, _p,
                       _p, _p, _p, _p, _i32, _i32, _i32, _i32, C.c_int, _i32, _p]
        fn.restype = C.c_int
    pk = page_table.struct()
    if q.dim() != 3:
        raise RpkError("q must be [tokens, n_heads, head_dim]")
    T = int(q.shape[0])
    qp = _dev(q, "q")
    op = _dev(out, "out", q.dtype, 3)
    gp = _dev(d_out, "d_out", q.dtype, 3)
    lp = _dev(log_sum_exp, "log_sum_exp", torch.float32, 2)
    dq = _dev(d_q, "d_q", torch.float32, 3)
    pool_shape = (pk.num_pages, pk.page_size, pk.n_kv_heads, pk.head_dim)
    for t, name in ((d_k_pages, "d_k_pages"), (d_v_pages, "d_v_pages")):
        _dev(t, name, torch.float32, 4)
        if tuple(t.shape) != pool_shape:
            raise RpkError(f"{name} must be {pool_shape}")
    for t, name in ((out, "out"), (d_out, "d_out"), (d_q, "d_q")):
        if tuple(t.shape) != tuple(q.shape):
            raise RpkError(f"{name} must have q's shape")
    if tuple(log_sum_exp.shape) != (T, int(n_heads)):
        raise RpkError("log_sum_exp must be [tokens, n_heads]")
    off = _dev(q_row_offsets, "q_row_offsets", torch.int32, 1)
    kvl = _dev(kv_lens, "kv_lens", torch.int32, 1)
    if scale is None:
        scale = float(head_dim) ** -0.5
    _check(fn(qp, off, kvl, C.byref(pk), int(n_heads), int(n_kv_heads), int(head_dim),
              float(scale), int(window), op, gp, lp, dq, d_k_pages.data_ptr(),
              d_v_pages.data_ptr(), int(kv_lens.shape[0]), T, int(max_q_len), int(max_kv_len),
              _dtype_code(q.dtype), int(sink_tokens), _stream(stream)))


def set_wait_limit_ns(limit_ns: int) -> None:
    """Bound (ns of the GPU timer) of every device-side wait of later attention
    launches (``rpk_set_wait_limit_ns``); 0 restores the 2 s default."""
    lib().rpk_set_wait_limit_ns(int(limit_ns))


def wait_limit_ns() -> int:
    return int(lib().rpk_wait_limit_ns())


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def ragged_paged_attention_noalloc(q, q_row_offsets, kv_lens, page_table: PagedKVCache,
                                   n_heads: int, n_kv_heads: int, head_dim: int,
                                   scale: float | None, window: int, out, *, max_q_len: int,
                                   max_kv_len: int, stream=None) -> None:
    """ragged_paged_attention for callers that cannot allocate device memory.

    Runs the split-KV decode path (bf16, max_q_len * group <= 16) with its
    scratch in a fixed 32 MiB array inside the library instead of a
    workspace; neither this function nor the C call allocates. Calls on one
    device share that array, so do not let two of them overlap on the GPU.
    """
    L = lib()
    fn = L.ragged_paged_attention_noalloc
    if fn.argtypes is None:
        _p, _i32 = C.c_void_p, C.c_int32
        fn.argtypes = [_p, _p, _p, C.POINTER(PagedKV), _i32, _i32, _i32, C.c_float, _i32, _p,
                       _i32, _i32, _i32, _i32, C.c_int, _p]
        fn.restype = C.c_int
    pk = page_table.struct()
    if q.dim() != 3:
        raise RpkError("q must be [tokens, n_heads, head_dim]")
    qp = _dev(q, "q")
    op = _dev(out, "out", q.dtype, 3)
    if tuple(out.shape) != tuple(q.shape):
        raise RpkError("out must have q's shape")
    off = _dev(q_row_offsets, "q_row_offsets", torch.int32, 1)
    kvl = _dev(kv_lens, "kv_lens", torch.int32, 1)
    if scale is None:
        scale = float(head_dim) ** -0.5
    _check(fn(qp, off, kvl, C.byref(pk), int(n_heads), int(n_kv_heads), int(head_dim),
              float(scale), int(window), op, int(kv_lens.shape[0]), int(q.shape[0]),
              int(max_q_len), int(max_kv_len), _dtype_code(q.dtype), _stream(stream)))
