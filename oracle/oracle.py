"""ctypes front end of the C oracle (rpk_oracle.c).

Arguments are numpy arrays or CPU torch tensors (bf16 tensors are passed as
their raw 16-bit patterns). Results are fp64 numpy arrays unless stated.
Test infrastructure only.
"""

from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

F32, BF16, E4M3 = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        # RPK_ORACLE_LIB lets the mutation test load a deliberately broken copy.
        path = os.environ.get("RPK_ORACLE_LIB") or _build.build()
        _lib = C.CDLL(path)
        _declare(_lib)
    return _lib


_p = C.c_void_p
_i32 = C.c_int32
_i64 = C.c_int64


def _declare(L):
    L.rpko_bf16_to_f64.argtypes = [C.c_uint16]
    L.rpko_bf16_to_f64.restype = C.c_double
    L.rpko_f64_to_bf16.argtypes = [C.c_double]
    L.rpko_f64_to_bf16.restype = C.c_uint16
    L.rpko_round.argtypes = [_p, C.c_size_t, C.c_int, _p]
    L.rpko_round.restype = None
    L.rpko_widen.argtypes = [_p, C.c_size_t, C.c_int, _p]
    L.rpko_widen.restype = None
    L.rpko_freqs_cis.argtypes = [_i32, _i32, C.c_double, _p]
    L.rpko_freqs_cis.restype = C.c_int
    L.rpko_rope.argtypes = [_p, C.c_int, _i32, _i32, _i32, _p, _i32, _p, _p, _p, _p, _i32,
                            C.c_int, _i32, _p]
    L.rpko_rope.restype = C.c_int
    L.rpko_cache_image.argtypes = [_p, _p, C.c_int, _i32, _i32, _i32, _p, _i32, _p, _p, _i32,
                                   _i32, _i32, _p, _p]
    L.rpko_cache_image.restype = C.c_int
    L.rpko_freqs_cis_proportional.argtypes = [_i32, _i32, _i32, C.c_double, _p]
    L.rpko_freqs_cis_proportional.restype = C.c_int
    L.rpko_visible.argtypes = [_i32] * 6
    L.rpko_visible.restype = C.c_int
    L.rpko_band.argtypes = [_i32, _i32, _i32, _i32, C.POINTER(_i32), C.POINTER(_i32)]
    L.rpko_band.restype = None
    L.rpko_attention.argtypes = [_p, C.c_int, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p,
                                 _i32, _i32, _p, _i32, C.c_double, _i32, _i32, _p, _i64, _p,
                                 _p, C.c_int]
    L.rpko_attention.restype = C.c_int
    L.rpko_e4m3_to_f64.argtypes = [C.c_uint8]
    L.rpko_e4m3_to_f64.restype = C.c_double
    L.rpko_f64_to_e4m3.argtypes = [C.c_double]
    L.rpko_f64_to_e4m3.restype = C.c_uint8
    L.rpko_cache_image_e4m3.argtypes = [_p, _p, C.c_int, _i32, _i32, _i32, _p, _i32, _p, _p,
                                        _i32, _i32, _i32, _p, _p, _p, _p]
    L.rpko_cache_image_e4m3.restype = C.c_int
    L.rpko_attention_cache.argtypes = [_p, C.c_int, _p, _p, _i32, _i32, _i32, _i32, _i32, _p,
                                       _p, C.c_int, _p, _p, _i32, _i32, _p, _i32, C.c_double,
                                       _i32, _i32, _p, _i64, _p, _p, C.c_int]
    L.rpko_attention_cache.restype = C.c_int
    L.rpko_attention_backward.argtypes = [_p, _p, C.c_int, _p, _p, _i32, _i32, _i32, _i32,
                                          _i32, _p, _p, C.c_int, _p, _p, _i32, _i32, _p, _i32,
                                          C.c_double, _i32, _i32, _p, _p, _p]
    L.rpko_attention_backward.restype = C.c_int
    L.rpko_flash_step.argtypes = [C.POINTER(C.c_double)] * 3 + [C.c_double, C.c_double]
    L.rpko_flash_step.restype = None


def _raw(x):
    """(numpy array with the raw element bits, dtype code) of a tensor/array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float32:
                return x.numpy(), F32
            if x.dtype == torch.float8_e4m3fn:
                return x.view(torch.uint8).numpy(), E4M3
            raise TypeError(f"unsupported dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.uint8:
        return x, E4M3
    raise TypeError(f"unsupported dtype {x.dtype}")


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _i32arr(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a), dtype=np.int32)


def bf16_bits_to_f64(bits: int) -> float:
    return lib().rpko_bf16_to_f64(int(bits))


def f64_to_bf16_bits(x: float) -> int:
    return int(lib().rpko_f64_to_bf16(float(x)))


def e4m3_to_f64(code: int) -> float:
    return lib().rpko_e4m3_to_f64(int(code))


def f64_to_e4m3(x: float) -> int:
    """One rounding to nearest, ties to even; beyond +-448 saturates."""
    return int(lib().rpko_f64_to_e4m3(float(x)))


def round_to(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round fp64 values once to bf16 bits (uint16) or fp32."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16 if dtype == BF16 else np.float32)
    lib().rpko_round(_ptr(x), x.size, dtype, _ptr(out))
    return out


def widen(x) -> np.ndarray:
    raw, code = _raw(x)
    out = np.empty(raw.shape, dtype=np.float64)
    lib().rpko_widen(_ptr(raw), raw.size, code, _ptr(out))
    return out


def freqs_cis(max_position: int, rotary_dim: int, base: float) -> np.ndarray:
    """fp32 [max_position, rotary_dim] table of (cos, sin) per pair."""
    out = np.empty((max_position, rotary_dim), dtype=np.float32)
    rc = lib().rpko_freqs_cis(int(max_position), int(rotary_dim), float(base), _ptr(out))
    if rc:
        raise ValueError(f"rpko_freqs_cis failed ({rc})")
    return out


def freqs_cis_proportional(max_position: int, head_dim: int, rotated_pairs: int,
                           base: float) -> np.ndarray:
    """fp32 [max_position, head_dim] p-RoPE table: (cos, sin) of p * base^(-2j/head_dim)
    for pairs j < rotated_pairs, (1, 0) for the rest (read with rotary_dim = head_dim,
    half layout)."""
    out = np.empty((max_position, head_dim), dtype=np.float32)
    rc = lib().rpko_freqs_cis_proportional(int(max_position), int(head_dim), int(rotated_pairs),
                                           float(base), _ptr(out))
    if rc:
        raise ValueError(f"rpko_freqs_cis_proportional failed ({rc})")
    return out


def rope(x, row_offsets, cache_lens, position_ids, mrope_section, table, interleaved,
         rotary_dim) -> np.ndarray:
    """fp64 rotated rows of x [T, heads, head_dim] (exact, before rounding)."""
    raw, code = _raw(x)
    T, nh, d = raw.shape
    offs = _i32arr(row_offsets)
    cl = _i32arr(cache_lens)
    pid = _i32arr(position_ids)
    ms = _i32arr(mrope_section)
    tab = np.ascontiguousarray(table, dtype=np.float32)
    out = np.empty((T, nh, d), dtype=np.float64)
    rc = lib().rpko_rope(_ptr(raw), code, T, nh, d, _ptr(offs), len(offs) - 1, _ptr(cl),
                         _ptr(pid), _ptr(ms), _ptr(tab), tab.shape[0], int(bool(interleaved)),
                         int(rotary_dim), _ptr(out))
    if rc:
        raise ValueError(f"rpko_rope failed ({rc})")
    return out


def cache_image(k_rot: np.ndarray, v_new, row_offsets, cache_lens, block_table, k_pages,
                v_pages, inplace: bool = False, k_scale=None, v_scale=None):
    """Return (k_pages', v_pages') raw arrays with the new tokens written in.

    k_rot is fp64 [T, n_kv_heads, d]; v_new, k_pages and v_pages are tensors or
    raw arrays of the cache dtype, or, for an e4m3 cache (uint8 / float8_e4m3fn
    pools), v_new of q's dtype and k_scale / v_scale the per-KV-head fp32
    scales. The inputs are copied first unless inplace is set, in which case
    k_pages / v_pages must be raw numpy arrays and are written directly.
    """
    vraw, code = _raw(v_new)
    kp, kcode = _raw(k_pages)
    vp, vcode = _raw(v_pages)
    if not inplace:
        kp, vp = kp.copy(), vp.copy()
    k_rot = np.ascontiguousarray(k_rot, dtype=np.float64)
    T, hk, d = k_rot.shape
    offs = _i32arr(row_offsets)
    bt = _i32arr(block_table)
    if kcode == E4M3:
        assert vcode == E4M3 and k_scale is not None and v_scale is not None
        ks = np.ascontiguousarray(k_scale, dtype=np.float32)
        vs = np.ascontiguousarray(v_scale, dtype=np.float32)
        rc = lib().rpko_cache_image_e4m3(_ptr(k_rot), _ptr(vraw), code, T, hk, d, _ptr(offs),
                                         len(offs) - 1, _ptr(_i32arr(cache_lens)), _ptr(bt),
                                         bt.shape[1], kp.shape[0], kp.shape[1], _ptr(ks),
                                         _ptr(vs), _ptr(kp), _ptr(vp))
        if rc:
            raise ValueError(f"rpko_cache_image_e4m3 failed ({rc})")
        return kp, vp
    assert code == kcode == vcode
    rc = lib().rpko_cache_image(_ptr(k_rot), _ptr(vraw), code, T, hk, d, _ptr(offs),
                                len(offs) - 1, _ptr(_i32arr(cache_lens)), _ptr(bt), bt.shape[1],
                                kp.shape[0], kp.shape[1], _ptr(kp), _ptr(vp))
    if rc:
        raise ValueError(f"rpko_cache_image failed ({rc})")
    return kp, vp


def visible(r: int, q_len: int, k_len: int, window: int, sinks: int, j: int) -> bool:
    """Key j is visible to row r (window and attention sinks)."""
    return bool(lib().rpko_visible(int(r), int(q_len), int(k_len), int(window), int(sinks),
                                   int(j)))


def band(r: int, q_len: int, k_len: int, window: int) -> tuple[int, int]:
    lo, hi = C.c_int32(), C.c_int32()
    lib().rpko_band(int(r), int(q_len), int(k_len), int(window), C.byref(lo), C.byref(hi))
    return lo.value, hi.value


def attention(q, q_offsets, kv_lens, k_pages, v_pages, block_table, n_kv_heads, scale,
              window, rows=None, n_threads: int | None = None, with_lse: bool = False,
              sinks: int = 0, k_scale=None, v_scale=None):
    """fp64 attention rows.

    rows=None: all rows, shape [T, n_heads, head_dim]. Otherwise rows is an
    int array [n, 2] of (token, head) pairs and the result is [n, head_dim].
    with_lse: return (out, lse), lse the natural log-sum-exp of each row's
    scores ([T, n_heads] or [n]; -inf for a row that sees no key).
    sinks: under a window, the first `sinks` keys stay visible (StreamingLLM).
    k_scale, v_scale: per-KV-head fp32 scales of an e4m3 cache (uint8 /
    float8_e4m3fn pools): key = code * k_scale[kvh], value = code * v_scale[kvh].
    """
    qraw, code = _raw(q)
    kp, kcode = _raw(k_pages)
    vp, vcode = _raw(v_pages)
    assert kcode == vcode and (kcode == code or kcode == E4M3)
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    T, H, d = qraw.shape
    offs = _i32arr(q_offsets)
    kvl = _i32arr(kv_lens)
    bt = _i32arr(block_table)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    if rows is None:
        out = np.empty((T, H, d), dtype=np.float64)
        lse = np.empty((T, H), dtype=np.float64) if with_lse else None
        rptr, n = None, T * H
    else:
        rows = _i32arr(rows).reshape(-1, 2)
        out = np.empty((rows.shape[0], d), dtype=np.float64)
        lse = np.empty(rows.shape[0], dtype=np.float64) if with_lse else None
        rptr, n = _ptr(rows), rows.shape[0]
    rc = lib().rpko_attention_cache(_ptr(qraw), code, _ptr(offs), _ptr(kvl), len(offs) - 1, T,
                                    H, int(n_kv_heads), d, _ptr(kp), _ptr(vp), kcode, _ptr(ks),
                                    _ptr(vs), kp.shape[1], kp.shape[0], _ptr(bt), bt.shape[1],
                                    float(scale), int(window), int(sinks), rptr, n, _ptr(out),
                                    None if lse is None else _ptr(lse), int(n_threads))
    if rc:
        raise ValueError(f"rpko_attention_cache failed ({rc})")
    return (out, lse) if with_lse else out


def attention_backward(q, d_out, q_offsets, kv_lens, k_pages, v_pages, block_table, n_kv_heads,
                       scale, window, sinks: int = 0, k_scale=None, v_scale=None):
    """fp64 (d_q [T, n_heads, d], d_k, d_v [num_pages, page_size, n_kv_heads, d]) of the
    attention output for the output gradient d_out (q's dtype)."""
    qraw, code = _raw(q)
    draw, dcode = _raw(d_out)
    assert dcode == code
    kp, kcode = _raw(k_pages)
    vp, vcode = _raw(v_pages)
    assert kcode == vcode and (kcode == code or kcode == E4M3)
    ks = None if k_scale is None else np.ascontiguousarray(k_scale, dtype=np.float32)
    vs = None if v_scale is None else np.ascontiguousarray(v_scale, dtype=np.float32)
    T, H, d = qraw.shape
    offs = _i32arr(q_offsets)
    kvl = _i32arr(kv_lens)
    bt = _i32arr(block_table)
    dq = np.empty((T, H, d), dtype=np.float64)
    dk = np.empty(kp.shape, dtype=np.float64)
    dv = np.empty(vp.shape, dtype=np.float64)
    rc = lib().rpko_attention_backward(_ptr(qraw), _ptr(draw), code, _ptr(offs), _ptr(kvl),
                                       len(offs) - 1, T, H, int(n_kv_heads), d, _ptr(kp),
                                       _ptr(vp), kcode, _ptr(ks), _ptr(vs), kp.shape[1],
                                       kp.shape[0], _ptr(bt), bt.shape[1], float(scale),
                                       int(window), int(sinks), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc:
        raise ValueError(f"rpko_attention_backward failed ({rc})")
    return dq, dk, dv


def flash_step(m: float, l: float, o: float, s: float, v: float) -> tuple[float, float, float]:
    cm, cl, co = C.c_double(m), C.c_double(l), C.c_double(o)
    lib().rpko_flash_step(C.byref(cm), C.byref(cl), C.byref(co), float(s), float(v))
    return cm.value, cl.value, co.value
