"""Pins for the random matrices the method draws: the rotation Pi and the QJL
sketch S, which both sides consume as data.

* Pi is orthogonal: max |Pi Pi^T - I| <= 1e-12 and max |Pi^T Pi - I| <= 1e-12
  in float64, at d = 64, 128 and 256 over several seeds.
* The float32 copy of Pi that the library and the parity oracle both read is
  orthogonal to 1e-6 (rounding each entry to float32 moves Pi Pi^T by a few
  1e-9; 1e-6 leaves a wide margin).
* Pi is Haar-distributed (a uniformly random rotation, "TurboQuant"
  explainer, troisinh.com, "Ý tưởng cốt lõi"): its first column is uniform on
  the sphere, so Pi[0, 0] is symmetric about zero with E[d Pi[0,0]^2] = 1.  A
  QR factorisation without the sign fix of diag(R) gives a first column whose
  leading entry always has one sign, which this catches.
* S has i.i.d. N(0, 1) entries stored exactly in float32 ("turboquant/
  audit_claims.py", AUDIT 1 counts S as D*D fp32).
"""

import math

import numpy as np
import pytest

from kv_cache_quantization_turboquantprod_b200 import workloads


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("seed", [0, 1, 1003, 1004, 77])
def test_pi_is_orthogonal_to_1e12(d, seed):
    pi, _ = workloads.rotation_and_sketch(d, seed)
    eye = np.eye(d)
    assert np.max(np.abs(pi @ pi.T - eye)) <= 1e-12
    assert np.max(np.abs(pi.T @ pi - eye)) <= 1e-12


@pytest.mark.parametrize("name", ["tiny", "llama8b", "qwen15b", "batched", "longctx"])
def test_float32_pi_of_every_workload_is_orthogonal_to_1e6(name):
    wl = workloads.by_name(name)
    pi64, pi32, s32 = workloads.layer_matrices(wl)
    p = pi32.astype(np.float64)
    err = np.max(np.abs(p @ p.T - np.eye(wl.d)))
    assert err <= 1e-6, err
    # the float32 copy is the float64 Pi rounded entry by entry
    assert np.max(np.abs(p - pi64)) <= 2.0 ** -24 * np.max(np.abs(pi64))
    assert np.max(np.abs(pi64 @ pi64.T - np.eye(wl.d))) <= 1e-12


def test_pi_first_column_is_sign_symmetric():
    d, n = 16, 800
    x = np.array([workloads.rotation_and_sketch(d, 5000 + i)[0][0, 0] for i in range(n)])
    frac = float(np.mean(x > 0))
    assert abs(frac - 0.5) < 4 * math.sqrt(0.25 / n), frac
    m2 = float(np.mean(d * x * x))
    # d * Pi[0,0]^2 ~ d * Beta(1/2, (d-1)/2): mean 1, variance 2 (d - 1) / (d + 2)
    se = math.sqrt(2 * (d - 1) / (d + 2) / n)
    assert abs(m2 - 1.0) < 4 * se, m2


def test_sketch_is_standard_gaussian_in_float32():
    _, s = workloads.rotation_and_sketch(128, 1003)
    assert np.array_equal(s, s.astype(np.float32).astype(np.float64))
    n = s.size
    assert abs(float(s.mean())) < 4 / math.sqrt(n)
    assert abs(float(s.var()) - 1.0) < 4 * math.sqrt(2.0 / n)
