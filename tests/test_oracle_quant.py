"""Pins for the oracle's key and value encoders on hand-checkable cases.

The rotation and sketch are replaced by non-symmetric permutation matrices,
so that a transposed Pi or S, a wrong index or a dropped term changes the
expected bits; every expectation is derived inline from the definitions
(bucketize the rotated unit vector; residual in the original space; sign of
S r), not from oracle helpers.
"""

import math

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


def test_value_scale_is_computed_in_float32_then_rounded():
    """scale16 = fp16(f32(f32(mx - mn) / 3)) -- the float32 steps, not fp64."""
    rng = np.random.default_rng(5)
    v = rng.standard_normal((200, 32)).astype(np.float32) * 7
    enc = quant.encode_values(v, 2, 32)
    for i in range(200):
        mn, mx = np.float32(v[i].min()), np.float32(v[i].max())
        s32 = np.float32(np.float32(mx - mn) / np.float32(3.0))
        assert enc["scale16"][i, 0] == float(np.float16(s32))
        assert enc["zero16"][i, 0] == float(np.float16(mn))


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
