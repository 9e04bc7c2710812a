"""Pins for the oracle's decode attention, score and dequantization.

* The one-pass decode (rotated query, centroid lookup, QJL term, softmax)
  equals the brute-force softmax over explicitly dequantized K/V to 1e-12
  relative (linearity: <Pi q, c> = <q, Pi^T c>, <S q, sigma> = <q, S^T sigma>).
* Special cases: one cached token gives out = v_hat_0 exactly; identical keys
  give the mean of v_hat; the GQA head mapping is hq -> hq // G.
* A two-token case with Pi = S = I is checked against softmax written out by
  hand with the 1/sqrt(d) scale.
"""

import math

import numpy as np

from kv_cache_quantization_turboquantprod_b200 import workloads
from oracle import attention, codebook, quant


def _random_cache(n, hkv, d, kb, vb, g, seed):
    pi, s = workloads.rotation_and_sketch(d, seed)
    cent, bnd, _ = codebook.lloyd_max_gaussian(kb - 1, d)
    rng = np.random.default_rng(seed)
    recs = []
    for h in range(hkv):
        k = rng.standard_normal((n, d)) * np.exp(0.5 * rng.standard_normal(d))
        v = (rng.standard_normal((n, d)) * 2).astype(np.float32)
        ke = quant.encode_keys(k, pi, s, cent, bnd)
        ve = quant.encode_values(v, vb, g)
        recs.append({"idx": ke["idx"], "sign": ke["sign"], "nk16": ke["nk16"],
                     "rn16": ke["rn16"], "codes": ve["codes"],
                     "scale16": ve["scale16"], "zero16": ve["zero16"]})
    return attention.stack_heads(recs), pi, s, cent


def test_one_pass_equals_brute_force():
    for (n, hkv, hq, kb, vb) in [(50, 2, 4, 3, 2), (37, 1, 6, 4, 3), (64, 2, 2, 2, 4)]:
        rec, pi, s, cent = _random_cache(n, hkv, 128, kb, vb, 32, seed=n)
        q = np.random.default_rng(n + 1).standard_normal((hq, 128))
        a = attention.decode_one_sequence(q, rec, pi, s, cent, 32)
        b = attention.brute_force_one_sequence(q, rec, pi, s, cent, 32)
        rel = np.max(np.abs(a - b)) / np.max(np.abs(b))
        assert rel < 1e-12, rel


def test_score_equals_dot_with_dequantized_key():
    rec, pi, s, cent = _random_cache(20, 1, 128, 3, 2, 32, seed=3)
    q = np.random.default_rng(4).standard_normal(128)
    sc = attention.score_keys(q, rec["idx"][:, 0], rec["sign"][:, 0], rec["nk16"][:, 0],
                              rec["rn16"][:, 0], pi, s, cent)
    kh = quant.dequantize_keys(rec["idx"][:, 0], rec["sign"][:, 0], rec["nk16"][:, 0],
                               rec["rn16"][:, 0], pi, s, cent)
    assert np.allclose(sc, kh @ q, rtol=1e-12, atol=1e-12)


def test_single_token_returns_its_value():
    rec, pi, s, cent = _random_cache(1, 2, 128, 3, 2, 32, seed=5)
    q = np.random.default_rng(6).standard_normal((4, 128)) * 10
    out = attention.decode_one_sequence(q, rec, pi, s, cent, 32)
    for hq in range(4):
        h = hq // 2
        vh = quant.dequantize_values(rec["codes"][:, h], rec["scale16"][:, h],
                                     rec["zero16"][:, h], 32)[0]
        assert np.array_equal(out[hq], vh)


def test_identical_keys_average_values():
    rec, pi, s, cent = _random_cache(9, 1, 128, 3, 2, 32, seed=7)
    for f in ("idx", "sign", "nk16", "rn16"):
        rec[f][:] = rec[f][:1]
    q = np.random.default_rng(8).standard_normal((3, 128))
    out = attention.decode_one_sequence(q, rec, pi, s, cent, 32)
    vh = quant.dequantize_values(rec["codes"][:, 0], rec["scale16"][:, 0],
                                 rec["zero16"][:, 0], 32)
    for hq in range(3):
        assert np.allclose(out[hq], vh.mean(axis=0), rtol=1e-13, atol=1e-13)


def test_gqa_mapping_is_consecutive():
    rec, pi, s, cent = _random_cache(5, 2, 128, 3, 2, 32, seed=9)
    # make head 0's values all -3 and head 1's all +5 (zero-point only)
    rec["codes"][:] = 0
    rec["scale16"][:] = 1.0
    rec["zero16"][:, 0] = -3.0
    rec["zero16"][:, 1] = 5.0
    q = np.random.default_rng(10).standard_normal((6, 128))
    out = attention.decode_one_sequence(q, rec, pi, s, cent, 32)
    assert np.allclose(out[:3], -3.0) and np.allclose(out[3:], 5.0)


def test_two_tokens_by_hand():
    d = 8
    cent, bnd, _ = codebook.lloyd_max_gaussian(1, d)
    a = cent[1]
    pi = np.eye(d)
    s = np.eye(d)
    idx = np.array([[1, 0, 1, 0, 1, 0, 1, 0], [0, 0, 0, 0, 1, 1, 1, 1]])
    sign = np.array([[1, 1, 0, 0, 1, 1, 0, 0], [1, 0, 1, 0, 1, 0, 1, 0]], np.uint8)
    nk = np.array([2.0, 3.0])
    rn = np.array([0.5, 0.25])
    q = np.array([1.0, -2.0, 0.5, 0.0, 1.5, -1.0, 2.0, 0.25])
    kap = math.sqrt(math.pi / 2) / d
    scores = []
    for n in range(2):
        mse = sum(q[j] * (a if idx[n, j] else -a) for j in range(d))
        qjl = sum(q[j] * (1.0 if sign[n, j] else -1.0) for j in range(d))
        scores.append(nk[n] * (mse + kap * rn[n] * qjl))
    w = [math.exp(sc / math.sqrt(d)) for sc in scores]
    p = [x / sum(w) for x in w]
    v0 = np.arange(8, dtype=float)
    v1 = -np.arange(8, dtype=float) * 2
    expect = p[0] * v0 + p[1] * v1
    rec = {"idx": idx[:, None], "sign": sign[:, None], "nk16": nk[:, None],
           "rn16": rn[:, None], "codes": np.stack([np.arange(8), np.zeros(8, int)])[:, None],
           "scale16": np.array([[[1.0]], [[1.0]]]),
           "zero16": np.array([[[0.0]], [[0.0]]])}
    # token 1's value: zero -14 with codes 0..7 scaled by 2 -> build via scale/zero
    rec["codes"][1, 0] = 7 - np.arange(8)
    rec["scale16"][1, 0, 0] = 2.0
    rec["zero16"][1, 0, 0] = -14.0
    out = attention.decode_one_sequence(q[None], rec, pi, s, cent, group=8)
    assert np.allclose(out[0], expect, rtol=1e-14, atol=1e-14)


def test_large_logits_stay_finite():
    """Scores of order 1e4 (fp16-range norms) must not overflow the softmax."""
    rec, pi, s, cent = _random_cache(16, 1, 128, 3, 2, 32, seed=11)
    rec["nk16"][:] = 60000.0
    q = np.random.default_rng(12).standard_normal((2, 128)) * 30
    out = attention.decode_one_sequence(q, rec, pi, s, cent, 32)
    assert np.all(np.isfinite(out))
    b = attention.brute_force_one_sequence(q, rec, pi, s, cent, 32)
    assert np.allclose(out, b, rtol=1e-9, atol=1e-9)


# ---------------------------------------------------------------------------
# recent-token window (exact) merged into the same softmax
# ---------------------------------------------------------------------------

def test_window_empty_equals_compressed_decode():
    rec, pi, s, cent = _random_cache(40, 2, 128, 3, 2, 32, seed=11)
    q = np.random.default_rng(12).standard_normal((4, 128))
    empty = np.zeros((0, 2, 128))
    a = attention.decode_with_window(q, rec, empty, empty, pi, s, cent, 32)
    b = attention.decode_one_sequence(q, rec, pi, s, cent, 32)
    assert np.array_equal(a, b)


def test_window_alone_is_textbook_attention():
    """No compressed tokens: exactly softmax(K q / sqrt d) V over the window,
    written out here with explicit sums."""
    rng = np.random.default_rng(13)
    wk = rng.standard_normal((7, 1, 128))
    wv = rng.standard_normal((7, 1, 128))
    q = rng.standard_normal((3, 128))
    out = attention.decode_with_window(q, None, wk, wv, None, None, None, 32)
    for j in range(3):
        logits = [float(np.dot(wk[t, 0], q[j])) / math.sqrt(128) for t in range(7)]
        top = max(logits)
        w = [math.exp(x - top) for x in logits]
        ref = sum(w[t] * wv[t, 0] for t in range(7)) / sum(w)
        assert np.allclose(out[j], ref, rtol=1e-12, atol=1e-12)


def test_window_merge_matches_log_sum_exp_of_the_parts():
    """The one softmax over compressed + window tokens equals the log-sum-exp
    merge of the two parts computed separately (a different route: split-K
    combine of two partial states)."""
    rec, pi, s, cent = _random_cache(33, 2, 128, 4, 2, 32, seed=14)
    rng = np.random.default_rng(15)
    wk = rng.standard_normal((5, 2, 128)) * 3
    wv = rng.standard_normal((5, 2, 128))
    q = rng.standard_normal((4, 128))
    out = attention.decode_with_window(q, rec, wk, wv, pi, s, cent, 32)
    for qh in range(4):
        h = qh // 2
        sc = attention.score_keys(q[qh], rec["idx"][:, h], rec["sign"][:, h], rec["nk16"][:, h],
                                  rec["rn16"][:, h], pi, s, cent) / math.sqrt(128)
        vh = quant.dequantize_values(rec["codes"][:, h], rec["scale16"][:, h],
                                     rec["zero16"][:, h], 32)
        lw = (wk[:, h] @ q[qh]) / math.sqrt(128)
        parts = []
        for logits, vals in ((sc, vh), (lw, wv[:, h])):
            m = logits.max()
            e = np.exp(logits - m)
            parts.append((m, e.sum(), e @ vals / e.sum()))
        M = max(p[0] for p in parts)
        num = sum(np.exp(m - M) * l * o for m, l, o in parts)
        den = sum(np.exp(m - M) * l for m, l, o in parts)
        assert np.allclose(out[qh], num / den, rtol=1e-11, atol=1e-12)


def test_window_nothing_cached_gives_zeros():
    empty = np.zeros((0, 2, 128))
    out = attention.decode_with_window(np.ones((2, 128)), None, empty, empty, None, None, None, 32)
    assert not out.any()


# ---- chunked prefill over the compressed cache (causal) ----------------------

def test_prefill_single_token_is_decode():
    rec, pi, s, cent = _random_cache(40, 2, 128, 3, 2, 32, seed=7)
    q = np.random.default_rng(8).standard_normal((1, 8, 128))
    a = attention.prefill_one_sequence(q, rec, pi, s, cent, 32)
    b = attention.decode_one_sequence(q[0], rec, pi, s, cent, 32)
    assert np.array_equal(a[0], b)


def test_prefill_equals_causal_brute_force():
    # causal softmax over explicitly dequantized K/V, query t sees the first
    # N - (T - 1 - t) tokens
    n, hkv, hq, t_chunk = 30, 2, 4, 5
    rec, pi, s, cent = _random_cache(n, hkv, 128, 3, 2, 32, seed=11)
    q = np.random.default_rng(12).standard_normal((t_chunk, hq, 128))
    got = attention.prefill_one_sequence(q, rec, pi, s, cent, 32)
    g = hq // hkv
    for t in range(t_chunk):
        m = n - (t_chunk - 1 - t)
        for h in range(hkv):
            khat = attention.dequantize_keys(rec["idx"][:m, h], rec["sign"][:m, h], rec["nk16"][:m, h],
                                             rec["rn16"][:m, h], pi, s, cent)
            vhat = attention.dequantize_values(rec["codes"][:m, h], rec["scale16"][:m, h],
                                               rec["zero16"][:m, h], 32)
            for j in range(g):
                logits = khat @ q[t, h * g + j] / math.sqrt(128)
                w = np.exp(logits - logits.max())
                ref = (w / w.sum()) @ vhat
                assert np.max(np.abs(got[t, h * g + j] - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_prefill_is_causal():
    n, t_chunk = 24, 4
    rec, pi, s, cent = _random_cache(n, 1, 128, 3, 2, 32, seed=13)
    q = np.random.default_rng(14).standard_normal((t_chunk, 2, 128))
    a = attention.prefill_one_sequence(q, rec, pi, s, cent, 32)
    # change the last cached token (the chunk's last one): only the last query sees it
    rec2 = {k: v.copy() for k, v in rec.items()}
    rec2["nk16"][-1] = rec2["nk16"][-1] * 2
    rec2["codes"][-1] = (rec2["codes"][-1] + 1) % 4
    b = attention.prefill_one_sequence(q, rec2, pi, s, cent, 32)
    assert np.array_equal(a[:-1], b[:-1])
    assert not np.array_equal(a[-1], b[-1])


def test_prefill_token_seeing_nothing_is_zero():
    rec, pi, s, cent = _random_cache(2, 1, 128, 3, 2, 32, seed=15)
    q = np.random.default_rng(16).standard_normal((4, 1, 128))
    out = attention.prefill_one_sequence(q, rec, pi, s, cent, 32)
    assert np.all(out[:2] == 0.0)
    assert np.all(np.isfinite(out)) and np.any(out[3] != 0.0)
