"""Pins for the oracle at head dims d = 64 and d = 256 (the oracle takes any
d; the pages sweep bit widths, "turboquant/audit_claims.py" AUDIT 5 and
AUDIT 6, and the method is stated for any d).

* Lloyd-Max codebooks scale as 1/sqrt(d) (the coordinate law N(0, 1/d)).
* MSE distortion of the rotated Lloyd-Max stage matches the exact Beta-law
  prediction for that d within 4 SE, and sits between 4^-b and 2.72 4^-b.
* The QJL estimator with a d x d sketch is unbiased over seeds of S and has
  the closed-form variance (pi/2 |q|^2 |r|^2 - <q,r>^2) / d.
* Decode equals softmax attention over explicitly dequantized K/V (1e-12).
* Record sizes follow the byte accounting: (kb + vb) d/8 + 4 + 4 d/32.
"""

import math

import numpy as np
import pytest

from kv_cache_quantization_turboquantprod_b200 import workloads
from oracle import attention, codebook, layout, quant
from test_oracle_statistics import exact_mse_distortion


@pytest.mark.parametrize("d", [64, 256])
def test_codebook_scales_with_inverse_sqrt_d(d):
    c128, b128, _ = codebook.lloyd_max_gaussian(2, 128)
    c, b, _ = codebook.lloyd_max_gaussian(2, d)
    assert np.allclose(c * math.sqrt(d), c128 * math.sqrt(128), rtol=0, atol=1e-12)
    assert np.allclose(b * math.sqrt(d), b128 * math.sqrt(128), rtol=0, atol=1e-12)


@pytest.mark.parametrize("d,mb", [(64, 2), (256, 2), (64, 3), (256, 1)])
def test_mse_distortion_matches_beta_prediction(d, mb):
    pi, s = workloads.rotation_and_sketch(d, 900 + d + mb)
    cent, bnd, _ = codebook.lloyd_max_gaussian(mb, d)
    rng = np.random.default_rng(d * 10 + mb)
    x = rng.standard_normal((8000, d))
    u = x / np.linalg.norm(x, axis=1, keepdims=True)
    enc = quant.encode_keys(u, pi, s, cent, bnd)
    e2 = np.sum((u - cent[enc["idx"]] @ pi) ** 2, axis=1)
    pred = exact_mse_distortion(mb, d)
    se = e2.std(ddof=1) / math.sqrt(len(e2))
    assert abs(e2.mean() - pred) < 4 * se, (e2.mean(), pred, se)
    assert 4.0 ** -mb <= pred <= 2.72 * 4.0 ** -mb


@pytest.mark.parametrize("d", [64, 256])
def test_qjl_unbiased_with_closed_form_variance(d):
    rng = np.random.default_rng(d)
    q = rng.standard_normal(d)
    r = rng.standard_normal(d) * 0.05
    truth = float(q @ r)
    n = 4000
    est = np.empty(n)
    for i in range(n):
        s = np.random.default_rng(70_000 + d * 10_000 + i).standard_normal((d, d))
        sign = (s @ r >= 0).astype(np.uint8)
        est[i] = attention.qjl_term(s @ q, sign, float(np.linalg.norm(r)), d)
    se = est.std(ddof=1) / math.sqrt(n)
    assert abs(est.mean() - truth) < 4 * se, (est.mean(), truth, se)
    var_pred = (math.pi / 2 * (q @ q) * (r @ r) - truth ** 2) / d
    assert abs(est.var(ddof=1) / var_pred - 1.0) < 0.1


@pytest.mark.parametrize("d", [64, 256])
def test_decode_equals_brute_force(d):
    pi, s = workloads.rotation_and_sketch(d, 5 + d)
    cent, bnd, _ = codebook.lloyd_max_gaussian(2, d)
    rng = np.random.default_rng(3 + d)
    n, hkv, hq = 200, 2, 8
    keys = rng.standard_normal((n, hkv, d)) * 1.5
    vals = rng.standard_normal((n, hkv, d))
    recs = []
    for h in range(hkv):
        ke = quant.encode_keys(keys[:, h], pi, s, cent, bnd)
        ve = quant.encode_values(vals[:, h], 2, 32)
        recs.append({"idx": ke["idx"], "sign": ke["sign"], "nk16": ke["nk16"], "rn16": ke["rn16"],
                     "codes": ve["codes"], "scale16": ve["scale16"], "zero16": ve["zero16"]})
    rec = attention.stack_heads(recs)
    q = rng.standard_normal((hq, d))
    got = attention.decode_one_sequence(q, rec, pi, s, cent, 32)
    ref = attention.brute_force_one_sequence(q, rec, pi, s, cent, 32)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_record_sizes_at_other_head_dims():
    assert layout.record_bytes(64, 3, 2, 32) == 5 * 8 + 4 + 8 == 52
    assert layout.record_bytes(256, 3, 2, 32) == 5 * 32 + 4 + 32 == 196
    assert layout.record_bytes(256, 4, 2, 32) == 6 * 32 + 4 + 32
    assert layout.record_bytes(64, 3, 3, 32, "mse") == 6 * 8 + 4 + 2
