"""Pins for the oracle's TurboQuant-MSE value path (3-bit Lloyd-Max cells of
the rotated unit value plus an fp16 norm; "03. Results & Benchmarks",
turboquant_cutile, "At a Glance -> Compression" and "Live Generation").

* Record accounting: 102 bytes per (token, head) at 3-bit keys and values,
  so an fp16 K+V cache shrinks 512/102 = 5.02x, the page's printed ratio
  (1,288 KB -> 257 KB; tests/golden/results_compression.json).
* A hand-built d = 8 case with a cyclic Pi: cells are the bucketized
  permuted unit vector, the norm is the fp16 norm.
* Reconstruction distortion E||v - v_hat||^2 / ||v||^2 equals the exact
  Beta-law prediction of the vb-bit Lloyd-Max stage within 4 SE.
* Decode accumulated in the rotated space and rotated back once per head
  equals softmax attention over explicitly dequantized values (1e-12), with
  Pi^T applied on the correct side (a transposed Pi fails).
* Zero vectors, layout placement by hand and the layout round trip.
"""

import json
import math

import numpy as np
import pytest

from kv_cache_quantization_turboquantprod_b200 import workloads
from oracle import accounting, attention, codebook, layout, quant
from test_oracle_statistics import exact_mse_distortion

D = 128


def test_record_is_102_bytes_and_ratio_matches_the_page(golden_dir):
    g = json.load(open(f"{golden_dir}/results_compression.json"))
    assert layout.record_bytes(D, 3, 3, 32, "mse") == 102
    r = accounting.ratios(4096, 8, D, 3, 3, 32, "mse")["data_only"]
    assert round(r, 2) == g["ratio"]
    assert round(g["kb_before"] / r) == g["kb_after"]
    # the group-quantized 3-bit value layout is larger (116 bytes, 4.41x)
    assert layout.record_bytes(D, 3, 3, 32) == 116


def test_hand_built_cyclic_rotation():
    d = 8
    pi = np.zeros((d, d))
    for i in range(d):
        pi[i, (i + 1) % d] = 1.0
    cent, bnd, _ = codebook.lloyd_max_gaussian(3, d)
    v = np.array([[0.5, -2.0, 1.0, 0.25, -0.75, 3.0, -1.5, 0.1]])
    enc = quant.encode_values_mse(v, pi, cent, bnd)
    nv = math.sqrt(float(np.sum(v * v)))
    w = v[0] / nv
    y = [w[(i + 1) % d] for i in range(d)]
    want = [sum(1 for t in bnd if t < yi) for yi in y]
    assert list(enc["vidx"][0]) == want
    assert enc["nv16"][0] == float(np.float16(nv))
    vhat = quant.dequantize_values_mse(enc["vidx"], enc["nv16"], pi, cent)
    # (Pi^T c)_j = c_i for the i with (i + 1) mod d == j
    c = [cent[k] for k in want]
    assert np.allclose(vhat[0], [enc["nv16"][0] * c[(j - 1) % d] for j in range(d)], atol=1e-15)


@pytest.mark.parametrize("vb", [2, 3])
def test_reconstruction_distortion_matches_beta_prediction(vb):
    pi, _ = workloads.rotation_and_sketch(D, 321 + vb)
    cent, bnd, _ = codebook.lloyd_max_gaussian(vb, D)
    rng = np.random.default_rng(77 + vb)
    v = rng.standard_normal((20_000, D)) * np.exp(rng.standard_normal())
    enc = quant.encode_values_mse(v, pi, cent, bnd)
    # distortion of the unit vector (the fp16 norm is a separate, tiny factor)
    w = v / np.linalg.norm(v, axis=1, keepdims=True)
    e2 = np.sum((w - cent[enc["vidx"]] @ pi) ** 2, axis=1)
    pred = exact_mse_distortion(vb)
    se = e2.std(ddof=1) / math.sqrt(len(e2))
    assert abs(e2.mean() - pred) < 4 * se, (e2.mean(), pred, se)
    vhat = quant.dequantize_values_mse(enc["vidx"], enc["nv16"], pi, cent)
    rel = np.sum((v - vhat) ** 2, axis=1) / np.sum(v * v, axis=1)
    assert abs(rel.mean() - pred) < 4 * se + 1e-6


def _mse_rec(n, hkv, rng, pi, s, kcent, kbnd, vcent, vbnd):
    keys = rng.standard_normal((n, hkv, D)) * 2.0
    vals = rng.standard_normal((n, hkv, D)) * np.exp(rng.standard_normal((1, hkv, D)))
    recs = []
    for h in range(hkv):
        ke = quant.encode_keys(keys[:, h], pi, s, kcent, kbnd)
        ve = quant.encode_values_mse(vals[:, h], pi, vcent, vbnd)
        recs.append({"idx": ke["idx"], "sign": ke["sign"], "nk16": ke["nk16"],
                     "rn16": ke["rn16"], "vidx": ve["vidx"], "nv16": ve["nv16"]})
    return attention.stack_heads(recs)


def test_rotated_space_decode_equals_brute_force():
    pi, s = workloads.rotation_and_sketch(D, 11)
    kcent, kbnd, _ = codebook.lloyd_max_gaussian(2, D)
    vcent, vbnd, _ = codebook.lloyd_max_gaussian(3, D)
    rng = np.random.default_rng(5)
    rec = _mse_rec(300, 2, rng, pi, s, kcent, kbnd, vcent, vbnd)
    q = rng.standard_normal((8, D))
    got = attention.decode_one_sequence(q, rec, pi, s, kcent, 32, value_centroids=vcent)
    ref = attention.brute_force_one_sequence(q, rec, pi, s, kcent, 32, value_centroids=vcent)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))
    # rotating back with Pi instead of Pi^T gives a different answer
    wrong = attention.decode_one_sequence(q, rec, pi.T, s, kcent, 32, value_centroids=vcent)
    assert np.max(np.abs(wrong - ref)) > 1e-3 * np.max(np.abs(ref))
    # one token: the output is that token's reconstructed value
    one = {k: v[:1] for k, v in rec.items()}
    out1 = attention.decode_one_sequence(q, one, pi, s, kcent, 32, value_centroids=vcent)
    v0 = quant.dequantize_values_mse(rec["vidx"][:1, 0], rec["nv16"][:1, 0], pi, vcent)[0]
    assert np.allclose(out1[:4], v0[None], rtol=0, atol=1e-12)


def test_zero_value_vector():
    pi, _ = workloads.rotation_and_sketch(D, 3)
    vcent, vbnd, _ = codebook.lloyd_max_gaussian(3, D)
    enc = quant.encode_values_mse(np.zeros((2, D)), pi, vcent, vbnd)
    assert not enc["vidx"].any() and not enc["nv16"].any()
    assert not quant.dequantize_values_mse(enc["vidx"], enc["nv16"], pi, vcent).any()


def test_mse_layout_by_hand_and_round_trip():
    spec = layout.CacheSpec(2, 3, 256, D, 3, 3, 32, value_mode="mse")
    assert spec.tile_bytes == 128 * 102
    off = layout.section_offsets(D, 3, 3, 32, "mse")
    assert (off["vplanes"], off["norms"], off["vsz"], off["end"]) == (6144, 12288, 12800, 13056)
    buf = spec.empty()
    n = 5
    kr = {"idx": np.zeros((n, D), np.int64), "sign": np.zeros((n, D), np.uint8),
          "nk16": np.zeros(n), "rn16": np.zeros(n)}
    vr = {"vidx": np.zeros((n, D), np.int64), "nv16": np.zeros(n)}
    vr["vidx"][0, 13] = 5          # bits 0 and 2 of coordinate 13: planes 0 and 2, byte 1, bit 5
    vr["nv16"][0] = 2.0            # fp16 0x4000
    b, h, pos = 1, 2, 130          # tile 1, slot 2
    spec.write(buf, b, h, pos, kr, vr, 0)
    base = ((b * 3 + h) * 2 + 1) * 128 * 102
    assert buf[base + 6144 + 0 * 2048 + 2 * 16 + 1] == 1 << 5
    assert buf[base + 6144 + 1 * 2048 + 2 * 16 + 1] == 0
    assert buf[base + 6144 + 2 * 2048 + 2 * 16 + 1] == 1 << 5
    assert buf[base + 12800 + 2 * 2] == 0x00 and buf[base + 12800 + 2 * 2 + 1] == 0x40
    rng = np.random.default_rng(2)
    kr = {"idx": rng.integers(0, 4, (n, D)), "sign": rng.integers(0, 2, (n, D)).astype(np.uint8),
          "nk16": quant.fp16(rng.random(n)), "rn16": quant.fp16(rng.random(n))}
    vr = {"vidx": rng.integers(0, 8, (n, D)), "nv16": quant.fp16(rng.random(n) * 9)}
    spec.write_sequence(buf, 0, 1, 126, kr, vr)
    a = spec.read(buf, 0, 1, 126, n)
    o = spec.read_one(buf, 0, 1, 126, n)
    for k in ("idx", "sign", "vidx", "nk16", "rn16", "nv16"):
        assert np.array_equal(a[k], o[k]), k
        want = vr[k] if k in vr else kr[k]
        assert np.array_equal(a[k], want), k
