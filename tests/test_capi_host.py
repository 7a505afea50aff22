"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/rpk.h declares, and rejects bad arguments with the
documented status before launching anything (every call below fails
validation, so no kernel is ever queued)."""

import ctypes as C

import pytest

import ragged_paged_kv_rope_b200 as R
from ragged_paged_kv_rope_b200 import binding as B
from ragged_paged_kv_rope_b200 import build as build_mod


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return B.lib()


def test_exports_every_declared_symbol(L):
    names = B.header_symbols()
    assert {"rope_qk_paged_ragged", "ragged_paged_attention",
            "ragged_paged_attention_workspace_size", "rope_freqs_cis"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in rpk.h but not exported"


def test_status_strings(L):
    for code in range(7):
        assert L.rpk_status_string(code)
    assert L.rpk_last_cuda_error() is not None


FAKE = 0x10000  # a 16-byte aligned address that is never dereferenced

# The calls below pass fake device addresses and rely on validation rejecting
# them before any launch; they are host checks and never run where a CUDA
# device is visible, so a validation bug cannot turn into a kernel reading a
# fake address.
host_only = pytest.mark.skipif(
    __import__("torch").cuda.is_available(), reason="fake-pointer checks run on CPU hosts only")


def cache(**kw):
    s = B.PagedKV()
    s.k_pages = kw.get("k_pages", FAKE)
    s.v_pages = kw.get("v_pages", FAKE)
    s.num_pages = kw.get("num_pages", 10)
    s.page_size = kw.get("page_size", 64)
    s.n_kv_heads = kw.get("n_kv_heads", 8)
    s.head_dim = kw.get("head_dim", 128)
    s.cache_dtype = kw.get("cache_dtype", B.RPK_BF16)
    s.block_table = kw.get("block_table", FAKE)
    s.max_pages_per_seq = kw.get("max_pages_per_seq", 4)
    s.batch = kw.get("batch", 2)
    s.cache_lens = kw.get("cache_lens", FAKE)
    s.error_word = None
    s.num_layers = kw.get("num_layers", 0)
    s.layer_idx = kw.get("layer_idx", 0)
    s.k_scale = kw.get("k_scale", None)
    s.v_scale = kw.get("v_scale", None)
    return s


def rope(L, c, **kw):
    a = dict(q=FAKE, off=FAKE, k=FAKE, v=FAKE, freqs=FAKE, pid=None, il=0, R=128, out=FAKE, T=5,
             H=32, dtype=B.RPK_BF16, maxp=100, ms=None)
    a.update(kw)
    return L.rope_qk_paged_ragged(a["q"], a["off"], a["k"], a["v"], C.byref(c), a["freqs"],
                                  a["pid"], a["il"], a["R"], a["out"], a["T"], a["H"], a["dtype"],
                                  a["maxp"], a["ms"], None)


def attn(L, c, **kw):
    a = dict(q=FAKE, off=FAKE, kvl=FAKE, H=32, Hk=8, d=128, scale=0.1, w=0, out=FAKE, batch=2,
             T=5, mq=4, mk=200, dtype=B.RPK_BF16, ws=None, wsb=0, lse=None, sinks=0)
    a.update(kw)
    return L.ragged_paged_attention(a["q"], a["off"], a["kvl"], C.byref(c), a["H"], a["Hk"],
                                    a["d"], a["scale"], a["w"], a["out"], a["batch"], a["T"],
                                    a["mq"], a["mk"], a["dtype"], a["ws"], a["wsb"], a["lse"],
                                    a["sinks"], None)


@host_only
@pytest.mark.parametrize("kw,status", [
    ({"q": None}, 1), ({"off": None}, 1), ({"freqs": None}, 1), ({"out": None}, 1),
    ({"R": 0}, 2), ({"R": 3}, 2), ({"R": 130}, 2), ({"R": 8}, 4),
    ({"H": 30}, 2), ({"H": 0}, 2), ({"T": -1}, 2), ({"maxp": 0}, 2),
    ({"dtype": B.RPK_F32}, 3), ({"dtype": 7}, 3),
    ({"q": FAKE + 8}, 2), ({"ms": C.cast((C.c_int32 * 3)(16, 24, 23), C.c_void_p),
                            "pid": FAKE}, 2),
    ({"ms": C.cast((C.c_int32 * 3)(16, 24, 24), C.c_void_p)}, 1),
])
def test_rope_rejects(L, kw, status):
    assert rope(L, cache(), **kw) == status


@host_only
@pytest.mark.parametrize("ckw,status", [
    ({"k_pages": None}, 1), ({"block_table": None}, 1), ({"cache_lens": None}, 1),
    ({"page_size": 48}, 4), ({"head_dim": 96}, 4), ({"num_pages": 0}, 2),
    ({"cache_dtype": 9}, 3),
    ({"layer_idx": 1}, 2), ({"num_layers": 3, "layer_idx": 3}, 2),
    ({"num_layers": 3, "layer_idx": -1}, 2), ({"num_layers": -2}, 2),
])
def test_rope_rejects_cache(L, ckw, status):
    assert rope(L, cache(**ckw)) == status


@host_only
@pytest.mark.parametrize("kw,status", [
    ({"q": None}, 1), ({"kvl": None}, 1), ({"Hk": 6}, 2), ({"H": 30}, 2), ({"d": 64}, 2),
    ({"batch": 3}, 2), ({"scale": 0.0}, 2), ({"scale": float("inf")}, 2),
    ({"scale": float("nan")}, 2), ({"mk": 1025}, 2), ({"mq": -1}, 2),
    ({"dtype": B.RPK_F32}, 3), ({"out": FAKE + 4}, 2),
    # decode shape with several splits needs a workspace
    ({"mq": 1, "mk": 1000, "ws": None, "wsb": 0}, 6),
    ({"mq": 1, "mk": 1000, "ws": FAKE + 16, "wsb": 1 << 30}, 6),  # misaligned
    ({"mq": 1, "mk": 1000, "ws": FAKE, "wsb": 64}, 6),            # too small
    # the tcgen05 prefill path keeps its work counter in the workspace
    ({"mq": 5, "ws": None, "wsb": 0}, 6),
    ({"mq": 5, "ws": FAKE + 16, "wsb": 1 << 20}, 6),               # misaligned
    ({"mq": 5, "ws": FAKE, "wsb": 128}, 6),                        # too small
    ({"lse": FAKE + 2}, 2),                                        # misaligned log-sum-exp
    ({"sinks": -1}, 2),
])
def test_attention_rejects(L, kw, status):
    assert attn(L, cache(max_pages_per_seq=16), **kw) == status


@host_only
def test_e4m3_cache_needs_both_scales(L):
    for ks, vs in ((None, FAKE), (FAKE, None), (None, None)):
        c = cache(cache_dtype=B.RPK_E4M3, k_scale=ks, v_scale=vs, max_pages_per_seq=16)
        assert rope(L, c) == 1
        assert attn(L, c) == 1


@host_only
def test_e4m3_prefill_routes(L):
    # Prefill shapes over an e4m3 cache take the tcgen05 kernel for head_dim 64
    # and 128, which keeps its work counter in the workspace; head_dim 256 runs
    # the CUDA-core kernel, which needs none (on a host without a GPU its launch
    # then fails with a CUDA error, never a workspace error).
    for d in (64, 128):
        c = cache(cache_dtype=B.RPK_E4M3, k_scale=FAKE, v_scale=FAKE, head_dim=d,
                  max_pages_per_seq=16)
        assert attn(L, c, d=d, mq=5, ws=None, wsb=0) == 6
        assert attn(L, c, d=d, mq=5, ws=FAKE, wsb=128) == 6
    c = cache(cache_dtype=B.RPK_E4M3, k_scale=FAKE, v_scale=FAKE, head_dim=256,
              max_pages_per_seq=16)
    assert attn(L, c, d=256, mq=5, ws=None, wsb=0) == 5


@host_only
def test_e4m3_cache_takes_bf16_and_f32_tensors_only(L):
    c = cache(cache_dtype=B.RPK_E4M3, k_scale=FAKE, v_scale=FAKE, max_pages_per_seq=16)
    assert rope(L, c, dtype=B.RPK_E4M3) == 3       # e4m3 is a cache dtype only
    assert attn(L, c, dtype=B.RPK_E4M3) == 3
    assert rope(L, c, R=6, dtype=B.RPK_F32) == 4    # validation continues past the dtype
    # the no-allocation decode entry point does not take e4m3 caches
    assert L.ragged_paged_attention_noalloc(
        C.c_void_p(FAKE), C.c_void_p(FAKE), C.c_void_p(FAKE), C.byref(c), 32, 8, 128,
        C.c_float(0.1), 0, C.c_void_p(FAKE), 2, 2, 1, 200, B.RPK_BF16, None) == 3


@host_only
def test_backward_rejects(L):
    fn = L.ragged_paged_attention_backward
    fn.restype = C.c_int
    P = C.c_void_p
    base = dict(q=FAKE, off=FAKE, kvl=FAKE, H=32, Hk=8, d=128, scale=0.1, w=0, out=FAKE,
                dout=FAKE, lse=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, batch=2, T=5, mq=4, mk=200,
                dtype=B.RPK_BF16, sinks=0)

    def call(c, **kw):
        a = dict(base, **kw)
        return fn(P(a["q"]), P(a["off"]), P(a["kvl"]), C.byref(c), a["H"], a["Hk"], a["d"],
                  C.c_float(a["scale"]), a["w"], P(a["out"]), P(a["dout"]), P(a["lse"]),
                  P(a["dq"]), P(a["dk"]), P(a["dv"]), a["batch"], a["T"], a["mq"], a["mk"],
                  a["dtype"], a["sinks"], None)

    c = cache(max_pages_per_seq=16)
    for kw, status in [({"dout": None}, 1), ({"lse": None}, 1), ({"dk": None}, 1),
                       ({"Hk": 6}, 2), ({"scale": 0.0}, 2), ({"sinks": -1}, 2),
                       ({"dq": FAKE + 4}, 2), ({"dtype": B.RPK_F32}, 3), ({"mk": 1025}, 2)]:
        assert call(c, **kw) == status, kw
    assert call(cache(cache_dtype=B.RPK_E4M3, max_pages_per_seq=16)) == 1   # scales missing


@host_only
def test_attention_rejects_layer_out_of_range(L):
    assert attn(L, cache(max_pages_per_seq=16, num_layers=2, layer_idx=2)) == 2
    assert L.ragged_paged_attention_noalloc(
        C.c_void_p(FAKE), C.c_void_p(FAKE), C.c_void_p(FAKE),
        C.byref(cache(max_pages_per_seq=16, layer_idx=1)), 32, 8, 128, C.c_float(0.1), 0,
        C.c_void_p(FAKE), 2, 2, 1, 200, B.RPK_BF16, None) == 2


def test_workspace_size(L):
    f = R.ragged_paged_attention_workspace_size
    assert f(0, 32, 128, 64, 8193, 64) == 0
    # never below the prefill work counter's 256 bytes
    assert f(1, 1, 64, 1, 1, 16) >= 256
    a = f(64, 32, 128, 64, 8193, 64)
    b = f(64, 32, 128, 64, 16000, 64)
    assert 0 < a <= b
    assert a % 256 == 0
    # bounded number of splits: very long contexts do not grow it without limit
    assert f(64, 32, 128, 64, 1 << 24, 64) <= 64 * 64 * 32 * (128 * 4 + 8) + 512


@host_only
def test_freqs_rejects(L):
    assert L.rope_freqs_cis(None, 10, 8, 1e4, None) == 1
    assert L.rope_freqs_cis(FAKE, 10, 7, 1e4, None) == 2
    assert L.rope_freqs_cis(FAKE, 10, 8, -1.0, None) == 2
    assert L.rope_freqs_cis_proportional(None, 10, 128, 16, 1e4, None) == 1
    assert L.rope_freqs_cis_proportional(FAKE, 10, 127, 16, 1e4, None) == 2
    assert L.rope_freqs_cis_proportional(FAKE, 10, 128, 65, 1e4, None) == 2
    assert L.rope_freqs_cis_proportional(FAKE, 10, 128, -1, 1e4, None) == 2
    assert L.rope_freqs_cis_proportional(FAKE, 10, 128, 16, 0.0, None) == 2


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(2, 4, 64)
    c = R.PagedKVCache(torch.zeros(4, 16, 2, 64), torch.zeros(4, 16, 2, 64),
                       torch.zeros(1, 4, dtype=torch.int32), torch.zeros(1, dtype=torch.int32))
    with pytest.raises(R.RpkError):
        R.rope_qk_paged_ragged(x, torch.zeros(2, dtype=torch.int32), x, x, c, torch.zeros(8, 64),
                               None, False, 64, x)


def test_wait_limit_setting():
    # process-wide bound of the kernels' device-side waits; 0 restores 2 s
    from ragged_paged_kv_rope_b200 import binding as B
    try:
        B.set_wait_limit_ns(12345)
        assert B.wait_limit_ns() == 12345
    finally:
        B.set_wait_limit_ns(0)
    assert B.wait_limit_ns() == 2_000_000_000
