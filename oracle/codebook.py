"""Lloyd-Max scalar codebook for the post-rotation coordinate law.

Test infrastructure only (see oracle/__init__.py).

After a Haar rotation, each coordinate of a unit vector in R^d follows a
concentrated law that is close to N(0, 1/d) ("TurboQuant" explainer,
troisinh.com, "Ý tưởng cốt lõi": rotated coordinates become i.i.d. and
concentrated; "Tại sao nó hoạt động": the same scalar quantizer then serves
every coordinate).  The quantizer is the MSE-optimal (Lloyd-Max) one: the
audit script's ``mse_quantizer`` keeps centroids, boundaries and decision
boundaries ("turboquant/audit_claims.py", AUDIT 1).

Reading: the codebook is fitted to the Gaussian N(0, sigma^2 = 1/d), not to
the exact Beta law, so that the Gaussian Lloyd-Max constants
(+-0.7979 sigma at 1 bit; +-0.4528 sigma, +-1.510 sigma at 2 bits) hold.
The law is symmetric, so its Lloyd-Max quantizer is: the iteration's
floating-point result is made exactly antisymmetric (c_i = -c_{n-1-i}, the
mean of the two magnitudes) and the boundaries are the midpoints of that,
the middle one exactly 0.

Algorithm (Lloyd's two optimality conditions, iterated to a fixed point):
  t_i = (c_i + c_{i+1}) / 2                       (nearest-neighbour boundary)
  c_i = E[X | t_{i-1} < X <= t_i]
      = sigma * (phi(a_i) - phi(b_i)) / (Phi(b_i) - Phi(a_i)),
        a_i = t_{i-1} / sigma, b_i = t_i / sigma  (centroid condition)
The density is log-concave, so the fixed point is unique and the starting
point does not matter.
"""

from __future__ import annotations

import math

import numpy as np


def _phi(x: float) -> float:
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _Phi_interval(a: float, b: float) -> float:
    """P(a < Z <= b) for a standard normal Z, via erfc for accuracy."""
    # Phi(x) = 0.5 * erfc(-x / sqrt 2)
    fa = 0.0 if a == -math.inf else 0.5 * math.erfc(-a / math.sqrt(2.0))
    fb = 1.0 if b == math.inf else 0.5 * math.erfc(-b / math.sqrt(2.0))
    return fb - fa


def conditional_mean(a: float, b: float, sigma: float) -> float:
    """E[X | a < X <= b] for X ~ N(0, sigma^2), a and b in X units."""
    za, zb = a / sigma, b / sigma
    return sigma * (_phi(za) - _phi(zb)) / _Phi_interval(za, zb)


def lloyd_max_gaussian(mse_bits: int, d: int, tol: float = 1e-14,
                       max_iter: int = 100000):
    """Centroids (ascending, 2^b) and decision boundaries (2^b - 1) of the
    Lloyd-Max quantizer for N(0, 1/d).  Returns (centroids, boundaries,
    iterations)."""
    if mse_bits < 1:
        raise ValueError("mse_bits must be >= 1")
    sigma = 1.0 / math.sqrt(d)
    levels = 2 ** mse_bits
    c = np.linspace(-2.0, 2.0, levels) * sigma
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate(([-math.inf], t, [math.inf]))
        c_new = np.array([conditional_mean(edges[i], edges[i + 1], sigma)
                          for i in range(levels)])
        delta = float(np.max(np.abs(c_new - c)))
        c = c_new
        if delta < tol * sigma:
            break
    # exact antisymmetry (the iteration leaves last-bit differences)
    mag = 0.5 * (c[::-1] - c)
    c = -mag
    t = 0.5 * (c[:-1] + c[1:])
    return c, t, it


def fixed_point_residual(centroids: np.ndarray, boundaries: np.ndarray,
                         d: int) -> float:
    """max |c_i - E[X | cell i]| / sigma plus max |t_i - midpoint| / sigma."""
    sigma = 1.0 / math.sqrt(d)
    edges = np.concatenate(([-math.inf], boundaries, [math.inf]))
    r1 = max(abs(centroids[i] - conditional_mean(edges[i], edges[i + 1], sigma))
             for i in range(len(centroids)))
    r2 = float(np.max(np.abs(boundaries - 0.5 * (centroids[:-1] + centroids[1:]))))
    return max(r1, r2) / sigma
