"""TurboQuant-prod key encoding and group quantization of values.

Test infrastructure only (see oracle/__init__.py).

Keys ("TurboQuant" explainer, troisinh.com, "Ý tưởng cốt lõi" and "Tại sao nó
hoạt động"; "turboquant/audit_claims.py", AUDIT 1, AUDIT 5, AUDIT 6):
  1. keep the norm nk = ||k||; work on the unit vector u = k / nk (the
     distortion bound is stated for unit-norm vectors, AUDIT 5);
  2. rotate: y = Pi u;
  3. bucketize every coordinate against the Lloyd-Max decision boundaries:
     idx_j = #{ i : t_i < y_j }   (a value on a boundary goes to the lower
     cell; reading);
  4. residual in the original space: r = u - Pi^T c, c_j = centroids[idx_j];
  5. 1-bit QJL sketch of the residual: s_j = [ (S r)_j >= 0 ] (an exact zero
     counts as +1; reading) and rn = ||r||;
  6. store nk and rn as fp16, round-to-nearest-even (reading: fp16 norms make
     the audit's 5.1x record accounting come out exactly; see accounting.py).
  A zero key stores nk = rn = 0 and all-zero codes and signs.

Values ("turboquant/audit_claims.py", AUDIT 1: ``value_bits``,
``value_group_size``): asymmetric min/max quantization per group of
``group`` contiguous channels of one token's head vector, no rotation.
Reading: fp16 scale and zero per group (the audit's record accounting), and
each code is the nearest of the 2^vb levels zero16 + k scale16, found by
rounding the exact quotient half-to-even and clamping.  In float64:
  mn, mx      = min, max of the group (exact)
  zero16      = fp16(mn)
  scale16     = fp16((mx - mn) / (2^vb - 1))
  code        = clamp(rint((v - zero16) / scale16), 0, 2^vb - 1),
                0 when scale16 == 0
  dequantized = code * scale16 + zero16
For inputs of at most float32 precision, mx - mn and v - zero16 are exact in
float64 and each quotient is within one float64 rounding of the exact one,
so a float64 tie is an exact tie.

TurboQuant-MSE values ("03. Results & Benchmarks", turboquant_cutile, "At a
Glance -> Compression": 3 bits per coordinate for keys and values, a 5.02x
smaller cache; "Live Generation": the value cache replaced by the 3-bit
TurboQuant version): the MSE stage of the key encoder applied to values,
with no QJL bit.  nv = ||v||; w = v / nv; y = Pi w; idx_j = #{t_i < y_j}
against the vb-bit Lloyd-Max boundaries; nv stored as fp16.  The value is
reconstructed as nv16 * Pi^T c[idx].  A zero vector stores nv = 0 and all-zero
codes.
"""

from __future__ import annotations

import math

import numpy as np


def kappa(d: int) -> float:
    """QJL estimator constant sqrt(pi/2) / m with m = d sketch rows."""
    return math.sqrt(math.pi / 2.0) / d


def fp16(x) -> np.ndarray:
    """Round to fp16, nearest-even, returned as float64 values."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def bucketize(y: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """idx = number of boundaries strictly below y (ties go to the lower cell)."""
    return np.searchsorted(np.asarray(boundaries, np.float64), y, side="left")


def encode_keys(keys: np.ndarray, pi: np.ndarray, s: np.ndarray,
                centroids: np.ndarray, boundaries: np.ndarray) -> dict:
    """Encode a batch of key vectors [n, d] (any float dtype).

    Returns a dict of logical fields:
      idx   [n, d] int   Lloyd-Max cell indices
      sign  [n, d] uint8 QJL sign bits (1 means +1)
      nk16  [n]   fp16-rounded key norms (float64)
      rn16  [n]   fp16-rounded residual norms (float64)
      y     [n, d] rotated unit coordinates (float64, for boundary bands)
      z     [n, d] S r (float64, for sign bands)
      nk, rn [n]   unrounded norms
    """
    x = np.asarray(keys, dtype=np.float64)
    pi = np.asarray(pi, dtype=np.float64)
    n, d = x.shape
    nk = np.sqrt(np.sum(x * x, axis=1))
    zero = nk == 0.0
    u = np.where(zero[:, None], 0.0, x / np.where(zero, 1.0, nk)[:, None])
    y = u @ pi.T                         # y = Pi u, row by row
    idx = bucketize(y, boundaries)
    res = residual_sketch(u, idx, pi, s, centroids)
    idx[zero] = 0
    sign, rn = res["sign"], res["rn"]
    sign[zero] = 0
    rn = np.where(zero, 0.0, rn)
    return {"idx": idx, "sign": sign, "nk16": fp16(nk), "rn16": fp16(rn),
            "y": y, "z": res["z"], "nk": nk, "rn": rn}


def unit_keys(keys: np.ndarray) -> np.ndarray:
    """Step 1 alone: u = k / ||k|| (0 for a zero key), float64."""
    x = np.asarray(keys, dtype=np.float64)
    nk = np.sqrt(np.sum(x * x, axis=1))
    return np.where((nk == 0.0)[:, None], 0.0, x / np.where(nk == 0.0, 1.0, nk)[:, None])


def residual_sketch(u: np.ndarray, idx: np.ndarray, pi: np.ndarray, s: np.ndarray,
                    centroids: np.ndarray) -> dict:
    """Steps 4 and 5 for given cells: r = u - Pi^T c[idx], rn = ||r||,
    z = S r, sign = [z >= 0].  The residual and its sketch are functions of
    the chosen cells, so a coordinate that lies on a decision boundary (where
    either cell is a correct bucketization) determines them through the cell
    actually chosen."""
    pi = np.asarray(pi, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)[idx]
    r = np.asarray(u, dtype=np.float64) - c @ pi     # r = u - Pi^T c, row by row
    z = r @ s.T                                      # z = S r, row by row
    return {"r": r, "rn": np.sqrt(np.sum(r * r, axis=1)), "z": z,
            "sign": (z >= 0.0).astype(np.uint8)}


def encode_values(values: np.ndarray, value_bits: int, group: int) -> dict:
    """Group-quantize value vectors [n, d] in float64.  Returns codes [n, d]
    int, scale16 / zero16 [n, d/group] (float64 holding fp16 values), the
    code coordinate t = (v - zero16) / scale16 [n, d] (0 where scale16 == 0)
    and the unrounded scale quotient (mx - mn) / (2^vb - 1) [n, d/group], the
    last two for the parity bands."""
    v = np.asarray(values, dtype=np.float64)
    n, d = v.shape
    if d % group:
        raise ValueError("d must be a multiple of the group size")
    ng = d // group
    vg = v.reshape(n, ng, group)
    mn = vg.min(axis=2)
    mx = vg.max(axis=2)
    levels = float(2 ** value_bits - 1)
    zero16 = fp16(mn)
    scale_q = (mx - mn) / levels
    scale16 = fp16(scale_q)
    sc = scale16[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(sc == 0.0, 0.0, (vg - zero16[:, :, None]) / np.where(sc == 0.0, 1.0, sc))
    codes = np.clip(np.rint(t), 0, levels).astype(np.int64)
    return {"codes": codes.reshape(n, d), "scale16": scale16, "zero16": zero16,
            "t": t.reshape(n, d), "scale_q": scale_q}


def dequantize_values(codes: np.ndarray, scale16: np.ndarray,
                      zero16: np.ndarray, group: int) -> np.ndarray:
    """v_hat = code * scale16 + zero16, per group, float64 [n, d]."""
    codes = np.asarray(codes, np.float64)
    n, d = codes.shape
    sc = np.repeat(np.asarray(scale16, np.float64), group, axis=1)
    ze = np.repeat(np.asarray(zero16, np.float64), group, axis=1)
    return codes * sc + ze


def dequantize_keys(idx: np.ndarray, sign: np.ndarray, nk16: np.ndarray,
                    rn16: np.ndarray, pi: np.ndarray, s: np.ndarray,
                    centroids: np.ndarray) -> np.ndarray:
    """Explicit reconstruction k_hat = nk * (Pi^T c + kappa * rn * S^T (2s - 1))
    [n, d] float64 (the audit's ``quantizer.dequantize(prod_q)``, AUDIT 2)."""
    pi = np.asarray(pi, np.float64)
    s = np.asarray(s, np.float64)
    d = pi.shape[0]
    c = np.asarray(centroids, np.float64)[idx]
    sigma = 2.0 * np.asarray(sign, np.float64) - 1.0
    mse = c @ pi                          # Pi^T c, row by row
    qjl = sigma @ s                       # S^T sigma, row by row
    return nk16[:, None] * (mse + kappa(d) * rn16[:, None] * qjl)


def encode_values_mse(values: np.ndarray, pi: np.ndarray, centroids: np.ndarray,
                      boundaries: np.ndarray) -> dict:
    """TurboQuant-MSE encoding of value vectors [n, d]: Lloyd-Max cells of the
    rotated unit vector and the fp16 norm.  Returns vidx [n, d] int, nv16 [n]
    (float64 holding fp16 values), vy [n, d] = Pi v / ||v|| (for boundary
    bands) and the unrounded norm nv [n]."""
    x = np.asarray(values, dtype=np.float64)
    nv = np.sqrt(np.sum(x * x, axis=1))
    zero = nv == 0.0
    w = np.where(zero[:, None], 0.0, x / np.where(zero, 1.0, nv)[:, None])
    y = w @ np.asarray(pi, np.float64).T          # y = Pi w, row by row
    idx = bucketize(y, boundaries)
    idx[zero] = 0
    return {"vidx": idx, "nv16": fp16(nv), "vy": y, "nv": nv}


def dequantize_values_mse(vidx: np.ndarray, nv16: np.ndarray, pi: np.ndarray,
                          centroids: np.ndarray) -> np.ndarray:
    """v_hat = nv16 * Pi^T c[vidx], float64 [n, d]."""
    c = np.asarray(centroids, np.float64)[vidx]
    return np.asarray(nv16, np.float64)[:, None] * (c @ np.asarray(pi, np.float64))
