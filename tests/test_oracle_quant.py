"""Pins for the oracle's key and value encoders on hand-checkable cases.

The rotation and sketch are replaced by non-symmetric permutation matrices,
so that a transposed Pi or S, a wrong index or a dropped term changes the
expected bits; every expectation is derived inline from the definitions
(bucketize the rotated unit vector; residual in the original space; sign of
S r), not from oracle helpers.
"""

import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import codebook, quant

D8 = 8


def _cyclic(d):
    """Pi with (Pi u)_i = u_{(i+1) mod d}."""
    p = np.zeros((d, d))
    for i in range(d):
        p[i, (i + 1) % d] = 1.0
    return p


def _signed_perm(d):
    """S with (S r)_i = eps_i * r_{perm_i}, perm and eps fixed, S != S^T."""
    perm = [3, 0, 6, 1, 7, 2, 5, 4]
    eps = [1, -1, 1, 1, -1, 1, -1, 1]
    s = np.zeros((d, d))
    for i in range(d):
        s[i, perm[i]] = eps[i]
    return s, perm, eps


def test_identity_like_special_case_one_bit():
    x = np.array([3.0, -1.0, 0.5, 0.25, 2.0, -2.0, 1.0, -0.25])
    pi = _cyclic(D8)
    s, perm, eps = _signed_perm(D8)
    cent, bnd, _ = codebook.lloyd_max_gaussian(1, D8)
    a = math.sqrt(2 / math.pi) / math.sqrt(D8)
    assert np.allclose(cent, [-a, a])
    enc = quant.encode_keys(x[None], pi, s, cent, bnd)

    nk = math.sqrt(sum(v * v for v in x))
    u = [v / nk for v in x]
    y = [u[(i + 1) % D8] for i in range(D8)]
    idx = [1 if yi > 0 else 0 for yi in y]
    c = [a if b else -a for b in idx]
    # (Pi^T c)_j = c_i for the i with (i+1) mod d == j
    pit_c = [c[(j - 1) % D8] for j in range(D8)]
    r = [u[j] - pit_c[j] for j in range(D8)]
    rn = math.sqrt(sum(v * v for v in r))
    z = [eps[i] * r[perm[i]] for i in range(D8)]
    sign = [1 if zi >= 0 else 0 for zi in z]

    assert list(enc["idx"][0]) == idx
    assert list(enc["sign"][0]) == sign
    assert enc["nk16"][0] == float(np.float16(nk))
    assert enc["rn16"][0] == float(np.float16(rn))
    assert abs(enc["rn"][0] - rn) < 1e-15


def test_two_bit_bucketize_and_ties():
    d = 128
    cent, bnd, _ = codebook.lloyd_max_gaussian(2, d)
    y = np.array([bnd[2], bnd[0], 0.0, cent[3] * 1.01, np.nextafter(bnd[2], 1.0),
                  np.nextafter(bnd[0], -1.0), cent[0], cent[1]])
    # a value on a boundary goes to the lower cell
    assert list(quant.bucketize(y, bnd)) == [2, 0, 1, 3, 3, 0, 0, 1]


def test_two_bit_encode_matches_cellwise_definition():
    """encode_keys with Pi = S = I: idx_j is the cell of u_j, signs are
    sign(u_j - c_j)."""
    d = 128
    cent, bnd, _ = codebook.lloyd_max_gaussian(2, d)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((20, d))
    enc = quant.encode_keys(x, np.eye(d), np.eye(d), cent, bnd)
    for i in range(20):
        u = x[i] / math.sqrt(float(np.sum(x[i] ** 2)))
        for j in range(d):
            cell = sum(1 for t in bnd if t < u[j])
            assert enc["idx"][i, j] == cell
            assert enc["sign"][i, j] == (1 if u[j] - cent[cell] >= 0 else 0)


def test_exact_zero_residual_component_counts_positive():
    d = 8
    cent, bnd, _ = codebook.lloyd_max_gaussian(1, d)
    a = cent[1]
    # u_0 = a exactly, so r_0 = u_0 - c_0 = 0 with Pi = S = I
    rest = math.sqrt((1.0 - a * a) / 7.0)
    u = np.array([a] + [rest] * 7)
    u = u / np.linalg.norm(u)
    enc = quant.encode_keys(u[None], np.eye(d), np.eye(d), cent, bnd)
    assert enc["z"][0][0] == pytest.approx(u[0] - a, abs=1e-16)
    expect = 1 if enc["z"][0][0] >= 0 else 0
    assert enc["sign"][0][0] == expect


def test_zero_key_stores_zeros():
    d = 128
    cent, bnd, _ = codebook.lloyd_max_gaussian(2, d)
    enc = quant.encode_keys(np.zeros((1, d)), np.eye(d), np.eye(d), cent, bnd)
    assert enc["nk16"][0] == 0 and enc["rn16"][0] == 0
    assert not enc["idx"].any() and not enc["sign"].any()


def test_norm_rounding_is_nearest_even():
    d = 8
    cent, bnd, _ = codebook.lloyd_max_gaussian(1, d)
    x = np.zeros(d)
    x[0] = 1.0 + 2.0 ** -11        # halfway between fp16 1.0 and 1.0 + 2^-10
    enc = quant.encode_keys(x[None], np.eye(d), np.eye(d), cent, bnd)
    assert enc["nk16"][0] == 1.0
    x[0] = 1.0 + 3 * 2.0 ** -11    # halfway between 1+2^-10 and 1+2^-9 -> even
    enc = quant.encode_keys(x[None], np.eye(d), np.eye(d), cent, bnd)
    assert enc["nk16"][0] == 1.0 + 2.0 ** -9


def test_values_on_grid_reconstruct_exactly():
    g = 32
    v = np.tile(np.array([-1.0, -0.5, 0.0, 0.5], np.float32), 8)[None]   # one group
    enc = quant.encode_values(v, 2, g)
    assert enc["zero16"][0, 0] == -1.0 and enc["scale16"][0, 0] == 0.5
    assert list(enc["codes"][0, :4]) == [0, 1, 2, 3]
    vh = quant.dequantize_values(enc["codes"], enc["scale16"], enc["zero16"], g)
    assert np.array_equal(vh, v.astype(np.float64))


def test_value_rounding_half_even_and_clamp():
    g = 32
    # zero = 0, max = 3 -> scale = 1; 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    base = np.zeros(32, np.float32)
    base[1], base[2], base[3], base[4] = 0.5, 1.5, 2.5, 3.0
    enc = quant.encode_values(base[None], 2, g)
    assert enc["scale16"][0, 0] == 1.0 and enc["zero16"][0, 0] == 0.0
    assert list(enc["codes"][0, :5]) == [0, 0, 2, 2, 3]


def test_constant_group_has_zero_scale():
    v = np.full((1, 64), 0.3, np.float32)
    enc = quant.encode_values(v, 3, 32)
    assert np.all(enc["scale16"] == 0) and not enc["codes"].any()
    vh = quant.dequantize_values(enc["codes"], enc["scale16"], enc["zero16"], 32)
    assert np.all(vh == float(np.float16(np.float32(0.3))))


def _fp16_exact(x: Fraction) -> Fraction:
    """Round a rational to the nearest fp16 value, ties to an even
    significand, by exact arithmetic (normal range and subnormals)."""
    if x == 0:
        return Fraction(0)
    sgn = -1 if x < 0 else 1
    a = abs(x)
    e = -14
    while e < 15 and a >= Fraction(2) ** (e + 1):
        e += 1
    ulp = Fraction(2) ** (e - 10)
    k = a / ulp
    lo = k.numerator // k.denominator
    rem = k - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sgn * lo * ulp


def test_fp16_exact_helper_against_known_values():
    assert _fp16_exact(Fraction(1, 3)) == Fraction(1365, 4096)          # 0x3555
    assert _fp16_exact(Fraction(1) + Fraction(1, 2048)) == 1             # tie -> even
    assert _fp16_exact(Fraction(1) + Fraction(3, 2048)) == Fraction(1) + Fraction(1, 512)
    assert _fp16_exact(Fraction(-2, 3)) == -Fraction(1365, 2048)
    assert _fp16_exact(Fraction(1, 2 ** 25)) == 0                       # half the least subnormal -> 0
    assert _fp16_exact(Fraction(3, 2 ** 25)) == Fraction(1, 2 ** 23)    # 1.5 subnormal ulps -> 2
    assert _fp16_exact(Fraction(65504)) == 65504                        # largest finite


@pytest.mark.parametrize("vb", [2, 3, 4])
def test_value_scale_and_zero_are_nearest_fp16_of_exact_values(vb):
    """scale16 is the fp16 nearest to the exact rational (mx - mn)/(2^vb - 1)
    and zero16 the fp16 nearest to mn, by exact arithmetic on the inputs."""
    rng = np.random.default_rng(50 + vb)
    v = (rng.standard_normal((60, 64)) * 7).astype(np.float32)
    v[0, :32] = np.float32(0.1)                      # a constant group
    enc = quant.encode_values(v, vb, 32)
    for i in range(v.shape[0]):
        for gi in range(2):
            grp = [Fraction(float(x)) for x in v[i, 32 * gi:32 * gi + 32]]
            mn, mx = min(grp), max(grp)
            assert Fraction(enc["zero16"][i, gi]) == _fp16_exact(mn)
            assert Fraction(enc["scale16"][i, gi]) == _fp16_exact((mx - mn) / (2 ** vb - 1))


@pytest.mark.parametrize("vb", [2, 3])
def test_value_codes_are_nearest_levels_by_brute_force(vb):
    """Each code is the index of the nearest level zero16 + k scale16
    (k = 0 .. 2^vb - 1), ties to the even k, searched over every level with
    exact arithmetic; includes values exactly halfway between two levels."""
    rng = np.random.default_rng(70 + vb)
    v = (rng.standard_normal((40, 32)) * 3).astype(np.float32)
    # a group with exact half-level values: zero 0, scale 1 after rounding
    lv = 2 ** vb - 1
    v[0] = 0.0
    v[0, 1] = lv
    v[0, 2:2 + lv] = np.arange(lv, dtype=np.float32) + 0.5
    enc = quant.encode_values(v, vb, 32)
    assert enc["scale16"][0, 0] == 1.0 and enc["zero16"][0, 0] == 0.0
    for i in range(v.shape[0]):
        z = Fraction(enc["zero16"][i, 0])
        s = Fraction(enc["scale16"][i, 0])
        for j in range(32):
            x = Fraction(float(v[i, j]))
            if s == 0:
                assert enc["codes"][i, j] == 0
                continue
            dist = [abs(x - (z + k * s)) for k in range(lv + 1)]
            best = min(dist)
            cands = [k for k in range(lv + 1) if dist[k] == best]
            want = cands[0] if len(cands) == 1 else [k for k in cands if k % 2 == 0][0]
            assert enc["codes"][i, j] == want, (i, j)


@pytest.mark.parametrize("vb", [2, 3, 4])
def test_value_error_bound(vb):
    rng = np.random.default_rng(vb)
    v = (rng.standard_normal((500, 128)) * np.exp(rng.standard_normal(128))).astype(np.float32)
    enc = quant.encode_values(v, vb, 32)
    assert enc["codes"].min() >= 0 and enc["codes"].max() <= 2 ** vb - 1
    vh = quant.dequantize_values(enc["codes"], enc["scale16"], enc["zero16"], 32)
    sc = np.repeat(enc["scale16"], 32, axis=1)
    ze = np.repeat(enc["zero16"], 32, axis=1)
    mn = np.repeat(v.reshape(500, 4, 32).min(2), 32, axis=1)
    # |v - v_hat| <= scale/2 + |zero16 - mn| + fp16 scale error * codes
    bound = 0.5 * sc + np.abs(ze - mn) + (2 ** vb) * sc * 2 ** -10 + 1e-6
    assert np.all(np.abs(vh - v) <= bound)
