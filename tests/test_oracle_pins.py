"""The fp64 oracle against what the pages and the mathematics fix.

Each test pins one part of the oracle to a value the pages print, a closed
form, an invariant or a special case, so that a dropped term, a wrong sign or
index, or a transposed operand fails one of them. No GPU is used.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O

# ----------------------------------------------------------------- helpers


def paged(k_dense, v_dense, page_size, seed=0, spare=3, dtype=np.float32):
    """Scatter per-sequence dense K/V ([k_len, Hk, d] each) into a shuffled pool.

    Written here, independently of the oracle, so that tests can compare the
    oracle's paged reads with dense formulations.
    """
    rng = np.random.default_rng(seed)
    n_pages = [(k.shape[0] + page_size - 1) // page_size for k in k_dense]
    total = sum(n_pages) + spare
    perm = rng.permutation(total)
    Hk, d = k_dense[0].shape[1:]
    # unused slots hold NaN (for e4m3 codes, 0x7F: the format's NaN)
    fill = 0x7F if dtype == np.uint8 else np.nan
    kp = np.full((total, page_size, Hk, d), fill, dtype=dtype)
    vp = np.full((total, page_size, Hk, d), fill, dtype=dtype)
    bt = np.full((len(k_dense), max(1, max(n_pages))), -1, dtype=np.int32)
    cur = 0
    for b, (k, v) in enumerate(zip(k_dense, v_dense)):
        for pg in range(n_pages[b]):
            bt[b, pg] = perm[cur]
            rows = k[pg * page_size:(pg + 1) * page_size]
            kp[perm[cur], :rows.shape[0]] = rows
            vp[perm[cur], :rows.shape[0]] = v[pg * page_size:(pg + 1) * page_size]
            cur += 1
    return kp, vp, bt


def one_row_attention(q_vec, keys, values, scale, window=0):
    """Attention of one query row (q_len = 1) over k_len keys, via the oracle."""
    q = np.asarray(q_vec, dtype=np.float32)[None, None, :]
    k = np.asarray(keys, dtype=np.float32)[:, None, :]
    v = np.asarray(values, dtype=np.float32)[:, None, :]
    kp, vp, bt = paged([k], [v], page_size=2)
    out = O.attention(q, [0, 1], [k.shape[0]], kp, vp, bt, 1, scale, window)
    return out[0, 0]


def e(i, d, scale=1.0):
    x = np.zeros(d, dtype=np.float32)
    x[i] = scale
    return x


# --------------------------------------------------------- bf16 narrowing


def test_bf16_matches_library_rounding_of_fp32_values():
    # For values exactly representable in fp32, one rounding fp64 -> bf16 is the
    # same as torch's fp32 -> bf16 (round to nearest, ties to even).
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    # add exact ties: bf16 values plus half an ulp
    base = (rng.integers(0, 2**16, size=20_000, dtype=np.uint32) << 16).astype(np.uint32)
    ties = (base | 0x8000).view(np.float32)
    f = np.concatenate([f, ties[np.isfinite(ties)]])
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.round_to(f.astype(np.float64), O.BF16)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("x,bits", [
    (1.0 + 2**-8, 0x3F80),                 # tie -> even mantissa (1.0)
    (1.0 + 3 * 2**-8, 0x3F82),             # tie -> even mantissa (1 + 2^-6)
    (1.0 + 2**-8 + 2**-40, 0x3F81),        # just above the tie: one rounding goes up
    (-(1.0 + 2**-8 + 2**-40), 0xBF81),
    (2.0**-133, 0x0001),                   # smallest subnormal
    (2.0**-134, 0x0000),                   # tie with zero -> even (zero)
    (3 * 2.0**-134, 0x0002),               # tie between 1 and 2 units -> 2
    (2.0**127 * (2 - 2**-7), 0x7F7F),      # largest finite
    (2.0**127 * (2 - 2**-8), 0x7F80),      # tie above the largest finite -> inf
    (2.0**127 * (2 - 2**-8) * (1 - 2**-40), 0x7F7F),
    (-0.0, 0x8000),
    (float("inf"), 0x7F80),
    (float("-inf"), 0xFF80),
])
def test_bf16_rounding_cases(x, bits):
    assert O.f64_to_bf16_bits(x) == bits


def test_bf16_nan_and_widening():
    assert O.f64_to_bf16_bits(float("nan")) & 0x7F80 == 0x7F80
    assert O.f64_to_bf16_bits(float("nan")) & 0x007F != 0
    assert O.bf16_bits_to_f64(0x3F80) == 1.0
    assert O.bf16_bits_to_f64(0xC0A0) == -5.0
    assert O.bf16_bits_to_f64(0x0001) == 2.0**-133


# ------------------------------------------------- scores and softmax pins


def test_scaled_score_worked_example(golden):
    # q.k = 8 with d = 64 scores 1.0: against a key scoring 0 the weights are
    # e/(1+e) and 1/(1+e).
    g = golden["scaled_score"]
    d = g["d_k"]
    keys = [e(0, d), np.zeros(d, np.float32)]
    out = one_row_attention(e(0, d, g["dot"]), keys, [e(0, d), e(1, d)], 1 / math.sqrt(d))
    s = g["score"]
    assert out[0] == pytest.approx(math.exp(s) / (math.exp(s) + 1.0), rel=1e-15)
    assert out[1] == pytest.approx(1.0 / (math.exp(s) + 1.0), rel=1e-15)


def test_cross_attention_score_worked_example(golden):
    g = golden["cross_attention_score"]
    d = g["d_k"]
    out = one_row_attention(e(0, d, g["q"]), [e(0, d, g["k"]), np.zeros(d, np.float32)],
                            [e(0, d), e(1, d)], 1 / math.sqrt(d))
    s = g["score"]
    assert out[0] == pytest.approx(math.exp(s) / (math.exp(s) + 1.0), rel=1e-15)


def test_stable_softmax_worked_example(golden):
    g = golden["stable_softmax"]
    d = 4
    keys = [e(0, d, s) for s in g["scores"]]
    w = one_row_attention(e(0, d), keys, [e(i, d) for i in range(3)], 1.0)
    assert w[0] == pytest.approx(g["weight0"], rel=1e-15)
    # sum_exp = 1 / (weight of the max-score key)
    assert 1.0 / w[2] == pytest.approx(g["sum_exp"], rel=1e-15)
    assert w.sum() == pytest.approx(1.0, abs=1e-15)


def test_two_pass_reproduces_online_worked_example(golden):
    g = golden["online_softmax"]
    d = 4
    out = one_row_attention(e(0, d), [e(0, d, s) for s in g["scores"]],
                            [e(0, d, v) for v in g["values"]], 1.0)
    assert out[0] == pytest.approx(g["final"], rel=1e-15)
    assert np.all(out[1:] == 0.0)


def test_online_state_worked_example(golden):
    # Every printed value is matched exactly: the page prints o after key 1
    # with 17 significant digits (17.357588823428847), which parses to the same
    # fp64 value as the shortest form 17.35758882342885 of 10 + e^-1 * 20.
    g = golden["online_softmax"]
    m, l, o = g["m0"], 0.0, 0.0
    for s, v, want in zip(g["scores"], g["values"], g["steps"]):
        m, l, o = O.flash_step(m, l, o, s, v)
        assert m == want["m"]
        assert l == want["l"]
        assert o == want["o"]
    assert o / l == g["final"]


def test_online_state_agrees_with_two_pass_random():
    rng = np.random.default_rng(3)
    for _ in range(20):
        n = int(rng.integers(1, 40))
        d = n
        scores = rng.normal(0, 3, size=n).astype(np.float32)
        vals = rng.normal(size=n).astype(np.float32)
        m, l, o = -math.inf, 0.0, 0.0
        for s, v in zip(scores, vals):
            m, l, o = O.flash_step(m, l, o, float(s), float(v))
        two = one_row_attention(e(0, d), [e(0, d, s) for s in scores],
                                [e(0, d, v) for v in vals], 1.0)
        assert o / l == pytest.approx(two[0], rel=1e-13, abs=1e-15)


def test_weights_sum_to_one():
    rng = np.random.default_rng(4)
    d, n = 32, 20
    q = rng.normal(size=d).astype(np.float32)
    keys = rng.normal(size=(n, d)).astype(np.float32)
    w = one_row_attention(q, keys, [e(i, d) for i in range(n)], 0.3)
    assert w[:n].sum() == pytest.approx(1.0, abs=1e-14)
    assert np.all(w[:n] > 0)


# ------------------------------------------------------------- the band


def test_causal_mask_worked_example(golden):
    # q_len = k_len = 6 prefill: row r sits at position r.
    for qpos, kpos in golden["causal_mask"]["attend"]:
        lo, hi = O.band(qpos, 6, 6, 0)
        assert lo <= kpos <= hi
    for qpos, kpos in golden["causal_mask"]["masked"]:
        lo, hi = O.band(qpos, 6, 6, 0)
        assert not (lo <= kpos <= hi)


def test_causal_mask_functional():
    # Changing value 5 leaves row 3 bit-identical; changing value 3 moves row 5.
    rng = np.random.default_rng(5)
    d, L = 16, 6
    q = rng.normal(size=(L, 1, d)).astype(np.float32)
    k = rng.normal(size=(L, 1, d)).astype(np.float32)
    v = rng.normal(size=(L, 1, d)).astype(np.float32)

    def run(vv):
        kp, vp, bt = paged([k], [vv], page_size=4)
        return O.attention(q, [0, L], [L], kp, vp, bt, 1, 0.25, 0)

    base = run(v)
    v5 = v.copy(); v5[5] += 1.0
    v3 = v.copy(); v3[3] += 1.0
    assert np.array_equal(run(v5)[3], base[3])
    assert not np.array_equal(run(v3)[5], base[5])


def test_band_alignment_and_window():
    # decode: one row over k keys sits at position k - 1
    assert O.band(0, 1, 10, 0) == (0, 9)
    # window w: w keys including the row's own
    assert O.band(0, 1, 10, 4) == (6, 9)
    # chunked prefill: 3 new rows appended to 7 cached keys
    assert O.band(0, 3, 10, 0) == (0, 7)
    assert O.band(2, 3, 10, 0) == (0, 9)
    # more rows than keys: early rows see nothing
    lo, hi = O.band(0, 4, 2, 0)
    assert hi < lo


def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(6)
    d, L = 8, 9
    q = rng.normal(size=(L, 2, d)).astype(np.float32)
    k = rng.normal(size=(L, 1, d)).astype(np.float32)
    v = rng.normal(size=(L, 1, d)).astype(np.float32)
    kp, vp, bt = paged([k], [v], page_size=4)
    out = O.attention(q, [0, L], [L], kp, vp, bt, 1, 0.5, window=1)
    for r in range(L):
        for h in range(2):
            assert np.array_equal(out[r, h], v[r, 0].astype(np.float64))


def test_rows_without_keys_are_zero():
    rng = np.random.default_rng(7)
    d = 8
    q = rng.normal(size=(4, 1, d)).astype(np.float32)
    k = rng.normal(size=(2, 1, d)).astype(np.float32)
    v = rng.normal(size=(2, 1, d)).astype(np.float32)
    kp, vp, bt = paged([k], [v], page_size=4)
    out = O.attention(q, [0, 4], [2], kp, vp, bt, 1, 0.5, 0)
    assert np.all(out[0] == 0.0) and np.all(out[1] == 0.0)
    assert np.array_equal(out[2, 0], v[0, 0].astype(np.float64))   # sees key 0 only
    assert not np.all(out[3] == 0.0)


# ------------------------------------------------------ log-sum-exp output
# NumKong attention_packed fills a (tokens, heads) log-sum-exp for training:
# the natural log of the row's sum of e^score over its visible keys.


def one_row_lse(q_vec, keys, scale, window=0):
    q = np.asarray(q_vec, dtype=np.float32)[None, None, :]
    k = np.asarray(keys, dtype=np.float32)[:, None, :]
    kp, vp, bt = paged([k], [k], page_size=2)
    _, lse = O.attention(q, [0, 1], [k.shape[0]], kp, vp, bt, 1, scale, window, with_lse=True)
    return lse[0, 0]


def test_lse_worked_example_score(golden):
    # q.k = 8 with d = 64 scores exactly 1.0: alone, its log-sum-exp is 1.0;
    # beside a key scoring 0 it is ln(e + 1).
    g = golden["scaled_score"]
    d = g["d_k"]
    s = g["score"]
    assert one_row_lse(e(0, d, g["dot"]), [e(0, d)], 1 / math.sqrt(d)) == s
    lse2 = one_row_lse(e(0, d, g["dot"]), [e(0, d), np.zeros(d, np.float32)], 1 / math.sqrt(d))
    assert lse2 == pytest.approx(math.log(math.exp(s) + 1.0), rel=1e-15)


@pytest.mark.parametrize("n,score", [(2, 0.0), (3, 1.5), (8, -2.0), (5, 40.0)])
def test_lse_of_equal_scores(n, score):
    # n keys of one score s: ln(n e^s) = s + ln n.
    d = 4
    lse = one_row_lse(e(0, d, score), [e(0, d)] * n, 1.0)
    assert lse == pytest.approx(score + math.log(n), rel=1e-14, abs=1e-14)


def test_lse_of_rows_without_keys_is_minus_infinity():
    rng = np.random.default_rng(7)
    d = 8
    q = rng.normal(size=(4, 1, d)).astype(np.float32)
    k = rng.normal(size=(2, 1, d)).astype(np.float32)
    kp, vp, bt = paged([k], [k], page_size=4)
    _, lse = O.attention(q, [0, 4], [2], kp, vp, bt, 1, 0.5, 0, with_lse=True)
    assert lse[0, 0] == -math.inf and lse[1, 0] == -math.inf
    assert np.isfinite(lse[2, 0]) and np.isfinite(lse[3, 0])


def test_lse_normalises_the_output():
    # e^(s_j - lse) are the softmax weights: they sum to one and weight V into
    # the output. Scores are recomputed here from the dense inputs.
    rng = np.random.default_rng(11)
    d, L, scale = 16, 13, 0.3
    q = rng.normal(size=(L, 2, d)).astype(np.float32)
    k = rng.normal(size=(L, 1, d)).astype(np.float32)
    v = rng.normal(size=(L, 1, d)).astype(np.float32)
    kp, vp, bt = paged([k], [v], page_size=4)
    out, lse = O.attention(q, [0, L], [L], kp, vp, bt, 1, scale, 0, with_lse=True)
    for r in range(L):
        for h in range(2):
            sc = scale * (k[:r + 1, 0].astype(np.float64) @ q[r, h].astype(np.float64))
            w = np.exp(sc - lse[r, h])
            assert w.sum() == pytest.approx(1.0, abs=1e-13)
            np.testing.assert_allclose(out[r, h], w @ v[:r + 1, 0].astype(np.float64),
                                       rtol=1e-12, atol=1e-13)


# ------------------------------------------------ attention sinks + window


def test_sinks_worked_example(golden):
    # The last of seq_len keys is the query (q_len 1); it sees the 4 sink
    # tokens and the 20-key recent window, nothing in between.
    g = golden["streaming_llm_sinks"]
    n = g["seq_len"]
    got = [int(O.visible(0, 1, n, g["window_size"], g["n_sink_tokens"], p))
           for p in g["positions"]]
    assert got == g["attended"]
    assert sum(O.visible(0, 1, n, g["window_size"], g["n_sink_tokens"], j) for j in range(n)) \
        == g["n_sink_tokens"] + g["window_size"]


def test_sinks_are_causal_and_need_a_window():
    # a row at position 2 (8 rows over 10 keys, row 0) with window 1 and 4 sinks
    # sees keys 0, 1, 2: sink 3 lies after it
    assert [O.visible(0, 8, 10, 1, 4, j) for j in range(5)] == [True, True, True, False, False]
    # without a window every earlier key is visible whatever the sinks
    assert all(O.visible(3, 4, 50, 0, 2, j) for j in range(50))
    assert not O.visible(3, 4, 50, 0, 2, 50)


def test_sinks_attention_equals_explicit_key_subset():
    # 1 query row over 40 keys, window 6, 3 sinks: the same as plain attention
    # over the 9 visible keys placed in a sequence of their own.
    rng = np.random.default_rng(23)
    d = 8
    k = rng.normal(size=(40, 1, d)).astype(np.float32)
    v = rng.normal(size=(40, 1, d)).astype(np.float32)
    q = rng.normal(size=(1, 1, d)).astype(np.float32)
    kp, vp, bt = paged([k], [v], page_size=4)
    got, lse = O.attention(q, [0, 1], [40], kp, vp, bt, 1, 0.4, 6, sinks=3, with_lse=True)
    keep = [0, 1, 2] + list(range(34, 40))
    kp2, vp2, bt2 = paged([k[keep]], [v[keep]], page_size=4)
    want, lse2 = O.attention(q, [0, 1], [len(keep)], kp2, vp2, bt2, 1, 0.4, 0, with_lse=True)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-15)
    assert lse[0, 0] == pytest.approx(lse2[0, 0], rel=1e-14)
    full = O.attention(q, [0, 1], [40], kp, vp, bt, 1, 0.4, 0, sinks=3)
    assert np.array_equal(full, O.attention(q, [0, 1], [40], kp, vp, bt, 1, 0.4, 0))


def test_decode_equals_last_prefill_row():
    rng = np.random.default_rng(8)
    d, L, H, Hk = 16, 13, 4, 2
    q = rng.normal(size=(L, H, d)).astype(np.float32)
    k = rng.normal(size=(L, Hk, d)).astype(np.float32)
    v = rng.normal(size=(L, Hk, d)).astype(np.float32)
    kp, vp, bt = paged([k], [v], page_size=4)
    for w in (0, 5):
        full = O.attention(q, [0, L], [L], kp, vp, bt, Hk, 0.3, w)
        dec = O.attention(q[L - 1:], [0, 1], [L], kp, vp, bt, Hk, 0.3, w)
        assert np.array_equal(full[L - 1], dec[0])


def test_gqa_head_mapping(golden):
    g = golden["gqa_group"]
    H, Hk = g["n_heads"], g["n_kv_heads"]
    assert H // Hk == g["group"]
    rng = np.random.default_rng(9)
    d, L = 8, 5
    q = rng.normal(size=(L, H, d)).astype(np.float32)
    k = rng.normal(size=(L, Hk, d)).astype(np.float32)
    v = rng.normal(size=(L, Hk, d)).astype(np.float32)
    kp, vp, bt = paged([k], [v], page_size=4)
    gqa = O.attention(q, [0, L], [L], kp, vp, bt, Hk, 0.4, 0)
    # multi-head attention with each KV head repeated group times
    kr = np.repeat(k, g["group"], axis=1)
    vr = np.repeat(v, g["group"], axis=1)
    kp2, vp2, bt2 = paged([kr], [vr], page_size=4)
    mha = O.attention(q, [0, L], [L], kp2, vp2, bt2, H, 0.4, 0)
    assert np.array_equal(gqa, mha)
    # query head 5 reads KV head 1 (5 // 4)
    assert np.array_equal(gqa[:, 5], O.attention(
        q[:, 5:6], [0, L], [L], *paged([k[:, 1:2]], [v[:, 1:2]], page_size=4), 1, 0.4, 0)[:, 0])


def test_attention_selected_rows_match_all_rows():
    rng = np.random.default_rng(10)
    d, H, Hk = 8, 4, 2
    lens = [3, 7]
    k = [rng.normal(size=(n, Hk, d)).astype(np.float32) for n in lens]
    v = [rng.normal(size=(n, Hk, d)).astype(np.float32) for n in lens]
    kp, vp, bt = paged(k, v, page_size=4)
    q = rng.normal(size=(sum(lens), H, d)).astype(np.float32)
    full = O.attention(q, [0, 3, 10], lens, kp, vp, bt, Hk, 0.3, 0)
    rows = np.array([[9, 3], [0, 0], [4, 2]])
    part = O.attention(q, [0, 3, 10], lens, kp, vp, bt, Hk, 0.3, 0, rows=rows)
    for i, (t, h) in enumerate(rows):
        assert np.array_equal(part[i], full[t, h])


def test_kv_bytes_formula(golden):
    from ragged_paged_kv_rope_b200 import metrics
    g = golden["kv_cache_bytes"]
    assert metrics.kv_cache_bytes(g["layers"], g["heads"], g["head_dim"], g["seq_len"],
                                  g["batch"], g["bytes_per_elt"]) == g["bytes"]


# ------------------------------------------------------------ RoPE table


def test_table_pair0_is_position_in_radians(golden):
    g = golden["sin_position_1"]
    t = O.freqs_cis(50, 128, 500000.0)
    assert t[g["position"], 1] == np.float32(g["value"])
    for p in range(50):
        assert t[p, 0] == np.float32(math.cos(p)) and t[p, 1] == np.float32(math.sin(p))


def test_table_position0_and_known_frequency():
    R, base = 128, 10000.0
    t = O.freqs_cis(201, R, base)
    assert np.all(t[0, 0::2] == 1.0) and np.all(t[0, 1::2] == 0.0)
    # pair j = R/4 has frequency base^(-1/2) = 0.01: at position 100 the angle is 1
    j = R // 4
    assert abs(float(t[100, 2 * j]) - math.cos(1.0)) <= 2 * 2**-24
    assert abs(float(t[100, 2 * j + 1]) - math.sin(1.0)) <= 2 * 2**-24
    # the last pair of R = 2 has frequency 1 as well
    t2 = O.freqs_cis(5, 2, base)
    assert t2[3, 1] == np.float32(math.sin(3.0))
    # cos^2 + sin^2 = 1 up to fp32 rounding of both entries
    c, s = t[:, 0::2].astype(np.float64), t[:, 1::2].astype(np.float64)
    assert np.max(np.abs(c * c + s * s - 1.0)) < 4 * 2**-24


def test_table_frequencies_decrease_geometrically():
    # ratio of the angles of consecutive pairs is base^(-2/R) everywhere
    R, base, p = 64, 10000.0, 3
    t = O.freqs_cis(p + 1, R, base)
    ang = np.arctan2(t[p, 1::2].astype(np.float64), t[p, 0::2].astype(np.float64))
    ratio = base ** (-2.0 / R)
    for j in range(1, R // 2):
        assert ang[j] / ang[j - 1] == pytest.approx(ratio, rel=1e-5)


# ------------------------------------------------------------------ RoPE


def _rope(x, offs, cache_lens, table, interleaved, R, pos=None, mrope=None):
    return O.rope(x, offs, cache_lens, pos, mrope, table, interleaved, R)


# ------------------------------------------------- p-RoPE (proportional)
# algenta rope_half_proportional: the first factor * head_dim / 2 pairs of
# the rotate-half layout turn with frequencies over the full head_dim, the
# remaining pairs stay as they are.


def test_p_rope_table_uses_full_head_dim_denominator():
    # head_dim 128, 32 rotated pairs: pair 16 has frequency 10000^(-32/128) = 0.1,
    # so position 10 turns it by exactly 1 radian (a rotated-subset denominator,
    # 64, would give 0.01).
    t = O.freqs_cis_proportional(11, 128, 32, 10000.0)
    assert abs(float(t[10, 32]) - math.cos(1.0)) <= 2 * 2**-24
    assert abs(float(t[10, 33]) - math.sin(1.0)) <= 2 * 2**-24
    assert np.all(t[0, 0:64:2] == 1.0) and np.all(t[0, 1:64:2] == 0.0)


def test_p_rope_table_tail_pairs_are_identity():
    t = O.freqs_cis_proportional(50, 256, 32, 10000.0)
    assert np.all(t[:, 64::2] == 1.0) and np.all(t[:, 65::2] == 0.0)
    assert np.any(t[1:, 62] != 1.0)  # the last rotated pair does turn


def test_p_rope_table_factor_one_is_the_full_table():
    for d in (64, 128):
        assert np.array_equal(O.freqs_cis_proportional(300, d, d // 2, 500000.0),
                              O.freqs_cis(300, d, 500000.0))


def test_p_rope_rotation_pairs_and_identity_tail():
    # Pair j = (x[j], x[j + d/2]) turns by pos * 10000^(-2j/d) for j < 16; the
    # others (and so channels 16..63 and 80..127) come back bit for bit.
    rng = np.random.default_rng(21)
    d, rot = 128, 16
    x = rng.normal(size=(6, 2, d)).astype(np.float32)
    pos = np.array([0, 1, 7, 100, 2047, 5], np.int32)
    tab = O.freqs_cis_proportional(2048, d, rot, 10000.0)
    out = _rope(x, [0, 6], [0], tab, False, d, pos=pos)
    keep = np.r_[rot:d // 2, d // 2 + rot:d]
    assert np.array_equal(out[..., keep], x[..., keep].astype(np.float64))
    for t, p in enumerate(pos):
        for j in range(rot):
            ang = float(p) * 10000.0 ** (-2.0 * j / d)
            a, b = x[t, :, j].astype(np.float64), x[t, :, j + d // 2].astype(np.float64)
            np.testing.assert_allclose(out[t, :, j], a * math.cos(ang) - b * math.sin(ang),
                                       atol=4e-7 * (1 + np.abs(a) + np.abs(b)).max())
            np.testing.assert_allclose(out[t, :, j + d // 2], b * math.cos(ang) + a * math.sin(ang),
                                       atol=4e-7 * (1 + np.abs(a) + np.abs(b)).max())


def test_rope_position0_is_identity():
    rng = np.random.default_rng(11)
    x = torch.from_numpy(rng.normal(size=(5, 3, 64)).astype(np.float32)).to(torch.bfloat16)
    tab = O.freqs_cis(4, 64, 10000.0)
    for il in (False, True):
        out = _rope(x, [0, 5], [0], tab, il, 64, pos=np.zeros(5, np.int32))
        assert np.array_equal(out, O.widen(x))


def test_rope_rotation_sign_on_unit_pair():
    # (1, 0) at position p becomes (cos theta, sin theta): multiplication by e^{i theta}
    d = R = 8
    tab = O.freqs_cis(10, R, 100.0)
    x = np.zeros((1, 1, d), np.float32)
    x[0, 0, 0] = 1.0
    out = _rope(x, [0, 1], [7], tab, False, R)
    assert out[0, 0, 0] == tab[7, 0] and out[0, 0, R // 2] == tab[7, 1]
    out = _rope(x, [0, 1], [7], tab, True, R)
    assert out[0, 0, 0] == tab[7, 0] and out[0, 0, 1] == tab[7, 1]
    # pair j of the half layout is (x[j], x[j + R/2])
    x = np.zeros((1, 1, d), np.float32)
    x[0, 0, 3 + R // 2] = 1.0       # second member of pair 3
    out = _rope(x, [0, 1], [7], tab, False, R)
    assert out[0, 0, 3] == -tab[7, 7] and out[0, 0, 3 + R // 2] == tab[7, 6]


def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(12)
    d, R = 128, 128
    x = rng.normal(size=(20, 4, d)).astype(np.float32)
    tab = O.freqs_cis(400, R, 500000.0)
    pos = rng.integers(0, 400, size=20).astype(np.int32)
    for il in (False, True):
        out = _rope(x, [0, 20], [0], tab, il, R, pos=pos)
        xd = x.astype(np.float64)
        if il:
            n_in = xd[..., 0::2] ** 2 + xd[..., 1::2] ** 2
            n_out = out[..., 0::2] ** 2 + out[..., 1::2] ** 2
        else:
            n_in = xd[..., :R // 2] ** 2 + xd[..., R // 2:] ** 2
            n_out = out[..., :R // 2] ** 2 + out[..., R // 2:] ** 2
        # |(a,b)|^2 (c^2 + s^2): the fp32 table entries give c^2 + s^2 = 1 +- 2^-22
        assert np.max(np.abs(n_out / n_in - 1.0)) < 4 * 2**-24


def test_rope_half_and_interleaved_agree_under_pair_permutation():
    rng = np.random.default_rng(13)
    d, R = 64, 48
    x = rng.normal(size=(6, 2, d)).astype(np.float32)
    tab = O.freqs_cis(30, R, 10000.0)
    pos = rng.integers(0, 30, size=6).astype(np.int32)
    half = R // 2
    # interleaved channel 2j <- half channel j, 2j+1 <- j + R/2; the rest as is
    perm = np.arange(d)
    perm[0:R:2] = np.arange(half)
    perm[1:R:2] = np.arange(half, R)
    x_il = x[..., perm]
    out_half = _rope(x, [0, 6], [0], tab, False, R, pos=pos)
    out_il = _rope(x_il, [0, 6], [0], tab, True, R, pos=pos)
    assert np.array_equal(out_il, out_half[..., perm])


def test_partial_rope_passes_tail_channels():
    rng = np.random.default_rng(14)
    d, R = 256, 128
    x = torch.from_numpy(rng.normal(size=(4, 3, d)).astype(np.float32)).to(torch.bfloat16)
    tab = O.freqs_cis(100, R, 10000.0)
    for il in (False, True):
        out = _rope(x, [0, 4], [50], tab, il, R)
        assert np.array_equal(out[..., R:], O.widen(x)[..., R:])
        assert not np.array_equal(out[..., :R], O.widen(x)[..., :R])


def test_rope_composes_by_position():
    # rotating by a then by b equals rotating by a + b (angle linear in position)
    rng = np.random.default_rng(15)
    d = R = 32
    x = rng.normal(size=(3, 2, d)).astype(np.float32)
    tab = O.freqs_cis(64, R, 10000.0)
    a = np.array([3, 10, 0], np.int32)
    b = np.array([5, 20, 7], np.int32)
    once = _rope(x, [0, 3], [0], tab, False, R, pos=a)
    twice = _rope(once.astype(np.float32), [0, 3], [0], tab, False, R, pos=b)
    direct = _rope(x, [0, 3], [0], tab, False, R, pos=a + b)
    assert np.max(np.abs(twice - direct)) < 1e-5


def test_rope_implicit_positions_from_cache_lens():
    rng = np.random.default_rng(16)
    d = R = 16
    x = rng.normal(size=(7, 2, d)).astype(np.float32)
    tab = O.freqs_cis(64, R, 10000.0)
    offs, cl = [0, 3, 7], [10, 20]
    implicit = _rope(x, offs, cl, tab, False, R)
    explicit = _rope(x, offs, None, tab, False, R,
                     pos=np.array([10, 11, 12, 20, 21, 22, 23], np.int32))
    assert np.array_equal(implicit, explicit)


def test_mrope_sections():
    rng = np.random.default_rng(17)
    d = R = 128
    sec = (16, 24, 24)
    x = rng.normal(size=(5, 2, d)).astype(np.float32)
    tab = O.freqs_cis(100, R, 10000.0)
    p = rng.integers(0, 100, size=5).astype(np.int32)
    same = np.stack([p, p, p])
    plain = _rope(x, [0, 5], None, tab, False, R, pos=p)
    m = _rope(x, [0, 5], None, tab, False, R, pos=same, mrope=sec)
    assert np.array_equal(m, plain)
    # only section 1 (pairs 16..39) moves when only its positions change
    moved = same.copy()
    moved[1] = (p + 9) % 100
    m2 = _rope(x, [0, 5], None, tab, False, R, pos=moved, mrope=sec)
    changed = np.any(m2 != m, axis=(0, 1))
    pairs = np.zeros(d, bool)
    pairs[16:40] = True
    pairs[64 + 16:64 + 40] = True
    assert np.array_equal(changed, pairs)
    # the section's rotation is the plain rotation at the section's positions
    plain_moved = _rope(x, [0, 5], None, tab, False, R, pos=moved[1])
    assert np.array_equal(m2[..., pairs], plain_moved[..., pairs])


def test_rope_rejects_out_of_range_position():
    tab = O.freqs_cis(4, 8, 10000.0)
    x = np.zeros((1, 1, 8), np.float32)
    with pytest.raises(ValueError):
        _rope(x, [0, 1], [4], tab, False, 8)


# ----------------------------------------------------------- cache image


def test_cache_image_hand_example():
    # one sequence, page size 2, pages [3, 1, 0], one cached token, two new:
    # slot 1 -> page 3 row 1, slot 2 -> page 1 row 0
    Hk, d = 1, 2
    kp = np.full((4, 2, Hk, d), -7.0, np.float32)
    vp = np.full((4, 2, Hk, d), -9.0, np.float32)
    k_rot = np.array([[[1.25, 2.5]], [[3.0, 4.0]]], np.float64)
    v_new = np.array([[[5.0, 6.0]], [[7.0, 8.0]]], np.float32)
    k2, v2 = O.cache_image(k_rot, v_new, [0, 2], [1], np.array([[3, 1, 0]]), kp, vp)
    want_k = kp.copy(); want_v = vp.copy()
    want_k[3, 1, 0] = [1.25, 2.5]; want_v[3, 1, 0] = [5.0, 6.0]
    want_k[1, 0, 0] = [3.0, 4.0]; want_v[1, 0, 0] = [7.0, 8.0]
    assert np.array_equal(k2, want_k) and np.array_equal(v2, want_v)


def test_cache_image_logical_order_invariant():
    from ragged_paged_kv_rope_b200 import workloads as W
    wl = W.make("mixed_chunked_mrope", seed=2, batch=4, n_heads=4, n_kv_heads=2,
                head_dim=16, rotary_dim=16, new_tokens=("uniform", 1, 9),
                cache_tokens=("uniform", 0, 20), page_size=4, mrope_section=(2, 3, 3))
    k_rot = O.widen(wl.k_new)
    kp, vp = O.cache_image(k_rot, wl.v_new, wl.q_offsets, wl.cache_lens, wl.block_table,
                           wl.k_pages, wl.v_pages)
    kp0 = wl.k_pages.view(torch.int16).numpy()
    kp_new = kp.view(np.int16)
    P = 4
    touched = np.zeros(kp0.shape[:2], bool)
    for b in range(4):
        for i in range(int(wl.q_lens[b])):
            slot = int(wl.cache_lens[b]) + i
            page = wl.block_table[b, slot // P]
            touched[page, slot % P] = True
            t = int(wl.q_offsets[b]) + i
            assert np.array_equal(vp[page, slot % P], wl.v_new[t].view(torch.int16).numpy().view(np.uint16))
            assert np.array_equal(kp[page, slot % P], O.round_to(k_rot[t], O.BF16))
    assert touched.sum() == wl.total_tokens
    assert np.array_equal(kp_new[~touched], kp0[~touched])


# ------------------------------------------------------------- e4m3 cache
# NumKong's scalar-type table fixes e4m3 as 1 sign, 4 exponent and 3 mantissa
# bits, range +-448, no infinity, with NaN, and its conversion policy rounds
# narrowing conversions to nearest with ties to even. torch's float8_e4m3fn is
# the same format, so it serves as an independent reference for every code
# and for rounding inside the finite range.


def _torch_e4m3_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_every_code():
    ref = _torch_e4m3_values()
    got = np.array([O.e4m3_to_f64(c) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.nanmax(got) == 448.0 and np.nanmin(got) == -448.0
    assert O.e4m3_to_f64(0x01) == 2.0 ** -9          # smallest subnormal
    assert O.e4m3_to_f64(0x08) == 2.0 ** -6          # smallest normal


def test_e4m3_encode_round_trips_every_finite_code():
    for c in range(256):
        v = O.e4m3_to_f64(c)
        if not math.isnan(v):
            assert O.f64_to_e4m3(v) == c, hex(c)


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.uniform(-464.0, 464.0, 20000),
        rng.uniform(-0.03, 0.03, 20000),                 # subnormals and small normals
        np.ldexp(rng.uniform(1.0, 2.0, 20000), rng.integers(-12, 9, 20000)) *
        rng.choice([-1.0, 1.0], 20000),
    ]).astype(np.float32)
    x = x[np.abs(x) <= 464.0]   # beyond, torch gives NaN where the cache saturates
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.f64_to_e4m3(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("x,code", [
    (17.0, 0x58), (19.0, 0x5A),          # ties between 16 / 18 and 18 / 20 go to the even mantissa
    (1.0625, 0x38), (1.1875, 0x3A),      # 1 + 1/16 -> 1, 1 + 3/16 -> 1.25
    (2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02), (1.5 * 2.0 ** -10, 0x01),
    (464.0, 0x7E),                       # tie between 448 and the missing 480: the even 448
    (-0.0, 0x80),
])
def test_e4m3_ties_to_even(x, code):
    assert O.f64_to_e4m3(x) == code


@pytest.mark.parametrize("x", [448.5, 470.0, 480.0, 1e6, math.inf])
def test_e4m3_saturates_beyond_largest_finite(x):
    assert O.f64_to_e4m3(x) == 0x7E
    assert O.f64_to_e4m3(-x) == 0xFE


def test_e4m3_nan_stays_nan():
    assert math.isnan(O.e4m3_to_f64(O.f64_to_e4m3(math.nan)))


def _e4m3_case(seed=0, Hk=2, d=8, P=4, lens=(5, 3), cache=(2, 0)):
    rng = np.random.default_rng(seed)
    B = len(lens)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(offs[-1])
    n_pages = sum((c + l + P - 1) // P for c, l in zip(cache, lens)) + 2
    perm = rng.permutation(n_pages)
    bt = np.full((B, 4), -1, dtype=np.int32)
    cur = 0
    for b in range(B):
        for i in range((cache[b] + lens[b] + P - 1) // P):
            bt[b, i] = perm[cur]
            cur += 1
    k_rot = rng.standard_normal((T, Hk, d)) * 3.0
    v = rng.standard_normal((T, Hk, d)).astype(np.float32)
    ks = np.array([0.02, 0.037], dtype=np.float32)[:Hk]
    vs = np.array([0.011, 0.05], dtype=np.float32)[:Hk]
    kp = np.full((n_pages, P, Hk, d), 0x7F, dtype=np.uint8)   # NaN code sentinel
    vp = np.full((n_pages, P, Hk, d), 0x7F, dtype=np.uint8)
    return offs, np.array(cache, dtype=np.int32), bt, k_rot, v, ks, vs, kp, vp


def test_e4m3_cache_image_codes_and_slots():
    offs, cl, bt, k_rot, v, ks, vs, kp, vp = _e4m3_case()
    k2, v2 = O.cache_image(k_rot, v, offs, cl, bt, kp, vp, k_scale=ks, v_scale=vs)
    P = kp.shape[1]
    written = np.zeros(kp.shape[:3], dtype=bool)
    for b in range(len(offs) - 1):
        for i in range(offs[b + 1] - offs[b]):
            t = offs[b] + i
            slot = cl[b] + i
            page, row = bt[b, slot // P], slot % P
            written[page, row] = True
            for h in range(kp.shape[2]):
                for c in range(kp.shape[3]):
                    assert k2[page, row, h, c] == O.f64_to_e4m3(k_rot[t, h, c] / float(ks[h]))
                    assert v2[page, row, h, c] == O.f64_to_e4m3(float(v[t, h, c]) / float(vs[h]))
    assert np.all(k2[~written] == 0x7F) and np.all(v2[~written] == 0x7F)
    # the stored value is code * scale within half an e4m3 step of the exact one
    t, h = 0, 1
    page, row = bt[0, cl[0] // P], cl[0] % P
    back = np.array([O.e4m3_to_f64(c) for c in k2[page, row, h]]) * float(ks[h])
    assert np.all(np.abs(back - k_rot[t, h]) <= 2.0 ** -4 * np.abs(k_rot[t, h]) + 2.0 ** -10 * ks[h])


def test_e4m3_attention_reads_code_times_scale():
    # Power-of-two scales make code * scale exact in fp32, so the e4m3 read must
    # equal the plain attention over those fp32 values to the last bit.
    rng = np.random.default_rng(3)
    Hk, d, P, H = 2, 8, 4, 4
    lens = [6, 9]
    kd = [rng.integers(0, 256, (n, Hk, d)).astype(np.uint8) for n in lens]
    vd = [rng.integers(0, 256, (n, Hk, d)).astype(np.uint8) for n in lens]
    for arr in kd + vd:
        arr[(arr & 0x7F) == 0x7F] = 0x3C   # no NaN codes in used slots
    ks = np.array([0.25, 2.0 ** -5], dtype=np.float32)
    vs = np.array([2.0 ** -3, 4.0], dtype=np.float32)
    kp8, vp8, bt = paged(kd, vd, P, dtype=np.uint8)
    dec = np.vectorize(O.e4m3_to_f64)
    kf = [(dec(k) * ks[None, :, None]).astype(np.float32) for k in kd]
    vf = [(dec(v) * vs[None, :, None]).astype(np.float32) for v in vd]
    kpf, vpf, bt2 = paged(kf, vf, P)
    assert np.array_equal(bt, bt2)
    q = rng.standard_normal((sum(lens), H, d)).astype(np.float32)
    offs = np.array([0, lens[0], sum(lens)], dtype=np.int32)
    for w in (0, 3):
        got = O.attention(q, offs, lens, kp8, vp8, bt, Hk, 0.3, w, k_scale=ks, v_scale=vs)
        ref = O.attention(q, offs, lens, kpf, vpf, bt, Hk, 0.3, w)
        assert np.array_equal(got, ref)


# ----------------------------------------------------------------- gradients
# attention_packed_gradients (NumKong "Attention with a Pre-Packed KV-Cache")
# gives the query, key and value gradients of the output under the same band.
# The oracle writes out the definition; here it is pinned to central finite
# differences of the (separately pinned) forward oracle, to the single-key
# case and to a conservation law.


def _grad_case(seed=0, window=0, sinks=0):
    rng = np.random.default_rng(seed)
    Hk, H, d, P = 2, 4, 8, 4
    q_lens, kv_lens = [4, 2], [6, 3]
    # values on a 2^-6 grid in [-2, 2]: +- 2^-10 perturbations stay exact in fp32
    grid = lambda shape: (rng.integers(-128, 129, shape) / 64.0).astype(np.float32)
    kd = [grid((n, Hk, d)) for n in kv_lens]
    vd = [grid((n, Hk, d)) for n in kv_lens]
    kp, vp, bt = paged(kd, vd, P, seed=seed)
    kp = np.nan_to_num(kp, nan=0.0)   # unused slots: any finite value
    vp = np.nan_to_num(vp, nan=0.0)
    T = sum(q_lens)
    q = grid((T, H, d))
    dout = grid((T, H, d))
    offs = np.array([0, q_lens[0], T], dtype=np.int32)
    return q, dout, offs, np.array(kv_lens, np.int32), kp, vp, bt, Hk


@pytest.mark.parametrize("window,sinks", [(0, 0), (3, 0), (2, 1)])
def test_gradients_match_finite_differences(window, sinks):
    q, dout, offs, kvl, kp, vp, bt, Hk = _grad_case(window=window, sinks=sinks)
    scale = 0.37
    dq, dk, dv = O.attention_backward(q, dout, offs, kvl, kp, vp, bt, Hk, scale, window, sinks)
    h = 2.0 ** -10

    def loss(qq, kk, vv):
        out = O.attention(qq, offs, kvl, kk, vv, bt, Hk, scale, window, sinks=sinks, n_threads=1)
        return float(np.sum(out * dout.astype(np.float64)))

    def fd(arr, idx, other):
        plus, minus = arr.copy(), arr.copy()
        plus[idx] += np.float32(h)
        minus[idx] -= np.float32(h)
        return (loss(*other(plus)) - loss(*other(minus))) / (2 * h)

    for idx in np.ndindex(q.shape):
        want = fd(q, idx, lambda a: (a, kp, vp))
        assert abs(dq[idx] - want) <= 1e-6 + 1e-5 * abs(want), ("dq", idx, dq[idx], want)
    used = np.unique(bt[bt >= 0])
    for page in used:
        for idx in np.ndindex(kp.shape[1:]):
            full = (page,) + idx
            want_k = fd(kp, full, lambda a: (q, a, vp))
            want_v = fd(vp, full, lambda a: (q, kp, a))
            assert abs(dk[full] - want_k) <= 1e-6 + 1e-5 * abs(want_k), ("dk", full, dk[full], want_k)
            assert abs(dv[full] - want_v) <= 1e-6 + 1e-5 * abs(want_v), ("dv", full, dv[full], want_v)


def test_gradients_of_a_single_visible_key():
    # one key: the output is its value whatever q and k are, so dQ = dK = 0 and dV = dO
    rng = np.random.default_rng(1)
    d = 8
    q = rng.standard_normal((1, 2, d)).astype(np.float32)
    dout = rng.standard_normal((1, 2, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, d)).astype(np.float32)
    v = rng.standard_normal((1, 1, d)).astype(np.float32)
    kp, vp, bt = paged([k], [v], page_size=2)
    dq, dk, dv = O.attention_backward(q, dout, [0, 1], [1], kp, vp, bt, 1, 0.5, 0)
    assert np.all(dq == 0.0) and np.all(dk[bt[0, 0], 0] == 0.0)
    assert np.allclose(dv[bt[0, 0], 0, 0], dout[0].astype(np.float64).sum(axis=0), rtol=0,
                       atol=1e-15)


def test_key_gradients_sum_to_zero():
    # each row's dS sums to zero (its weights sum to one), so sum_j dK_j = 0 for
    # every KV head
    q, dout, offs, kvl, kp, vp, bt, Hk = _grad_case(seed=4, window=3, sinks=1)
    dq, dk, dv = O.attention_backward(q, dout, offs, kvl, kp, vp, bt, Hk, 0.8, 3, 1)
    assert np.max(np.abs(dk.sum(axis=(0, 1)))) <= 1e-12
    assert np.any(dk != 0.0)
