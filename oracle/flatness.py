"""The linear-time flatness check of composed randomized Hadamard transforms
(oracle side, fp64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

[RHT] "Quantizing With Randomized Hadamard Transforms: Efficient Heuristic Now
Proven", Methodology ("adaptive verification") and Key contribution 4
("adaptive linear-time check"): before rotating, an O(d) pass over the input
evaluates its l3 norm (the measure for scalar quantization) and its l_inf
norm (the measure for vector quantization), to decide whether the input is
already "flat" enough that fewer than the worst-case number of transforms
(two for scalar, three for vector quantization) will do.  The 2-RHT analysis
(same page, Methodology, "scalar marginal") bounds a coordinate's distance to
the Gaussian through the Berry-Esseen theorem, whose ratio for the unit
vector x^ = x / ||x||_2 is exactly sum_i |x^_i|^3.

Readings of what the page leaves open:

* The norms are taken of the unit vector (the page's analysis normalises the
  input, x^), so both measures are scale-free:
      rho3   = ||x||_3^3 / ||x||_2^3 = sum_i |x_i|^3 / (sum_i x_i^2)^(3/2)
      rhoinf = ||x||_inf / ||x||_2
  Both lie in [d^(-1/2), 1]: d^(-1/2) for a row of equal magnitudes, 1 for a
  one-hot row.  A zero row has no direction; both are reported as 0.
* Granularity: one rotation serves a whole layer (the weights are rotated
  once, offline, by the same matrix), so the decision is taken per batch of
  rows; the check reports every row's value and the batch maximum.
* The page prints no thresholds; the mapping from these measures to a round
  count is left to the caller.
"""

import numpy as np


def flatness(X):
    """(rho3, rhoinf), fp64 arrays of one value per row of X (any float array)."""
    X = np.atleast_2d(np.asarray(X, dtype=np.float64))
    a = np.abs(X)
    s2 = np.sum(a * a, axis=1)
    s3 = np.sum(a * a * a, axis=1)
    mx = np.max(a, axis=1) if X.shape[1] else np.zeros(X.shape[0])
    nz = s2 > 0
    rho3 = np.zeros(X.shape[0])
    rhoinf = np.zeros(X.shape[0])
    rho3[nz] = s3[nz] / s2[nz] ** 1.5
    rhoinf[nz] = mx[nz] / np.sqrt(s2[nz])
    return rho3, rhoinf


def batch_max(X):
    """The batch's worst row for each measure: (max rho3, max rhoinf)."""
    rho3, rhoinf = flatness(X)
    if rho3.size == 0:
        return 0.0, 0.0
    return float(rho3.max()), float(rhoinf.max())
