"""Pins for the oracle's flatness check (CPU only).

[RHT] "Quantizing With Randomized Hadamard Transforms", Key contribution 4:
the O(d) check measures the l3 norm (scalar quantization) and the l_inf norm
(vector quantization) of the unit input.  Pinned by closed forms (one-hot,
k-sparse and constant rows, a 3-4 row), invariances, the power-mean bounds,
the Gaussian law of large numbers, and the Berry-Esseen bound that motivates
the l3 measure, checked exactly by enumerating every sign pattern.
"""

import itertools
import math

import numpy as np
import pytest

from oracle import flatness as ofl
from oracle import rpbh


def test_closed_forms():
    d = 64
    one_hot = np.zeros(d); one_hot[17] = -3.5
    rho3, rhoinf = ofl.flatness(one_hot)
    assert rho3[0] == 1.0 and rhoinf[0] == 1.0
    for k in (2, 4, 9, 16, 64):
        x = np.zeros(d)
        x[np.arange(k) * (d // k)] = 0.7 * np.where(np.arange(k) % 3 == 0, -1.0, 1.0)
        r3, ri = ofl.flatness(x)
        assert abs(r3[0] - k ** -0.5) < 1e-15 and abs(ri[0] - k ** -0.5) < 1e-15
    # a 3-4 row: (27 + 64) / 125 and 4 / 5
    x = np.zeros(d); x[0], x[5] = 3.0, -4.0
    r3, ri = ofl.flatness(x)
    assert abs(r3[0] - 91.0 / 125.0) < 1e-15 and abs(ri[0] - 0.8) < 1e-15


def test_zero_row_and_shapes():
    r3, ri = ofl.flatness(np.zeros((3, 32)))
    assert np.all(r3 == 0) and np.all(ri == 0)
    assert ofl.batch_max(np.zeros((0, 32))) == (0.0, 0.0)
    X = np.random.default_rng(0).standard_normal((5, 96))
    X[2] = 0.0
    X[4] = 0.0; X[4, 3] = 1.0
    assert ofl.batch_max(X) == (1.0, 1.0)


def test_invariances_and_bounds():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((50, 300)) * np.exp(rng.standard_normal(300))
    X[::7] *= rng.random((8, 300)) < 0.05          # some sparse rows
    r3, ri = ofl.flatness(X)
    s3, si = ofl.flatness(-4096.0 * X[:, rng.permutation(300)])   # scale, sign, order
    assert np.allclose(r3, s3, rtol=1e-13) and np.allclose(ri, si, rtol=1e-13)
    d = X.shape[1]
    nz = np.any(X != 0, axis=1)
    # power means: d^-1/2 <= rho3, rhoinf <= 1, and rhoinf^3 <= rho3 <= rhoinf
    assert np.all(r3[nz] >= d ** -0.5 - 1e-15) and np.all(ri[nz] >= d ** -0.5 - 1e-15)
    assert np.all(r3 <= 1 + 1e-15) and np.all(ri <= 1 + 1e-15)
    assert np.all(ri ** 3 <= r3 + 1e-15) and np.all(r3 <= ri + 1e-15)


def test_gaussian_rows_follow_the_law_of_large_numbers():
    # E|g|^3 = 2 sqrt(2/pi) and E g^2 = 1, so rho3 -> 2 sqrt(2/pi) / sqrt(d)
    d = 16384
    X = np.random.default_rng(2).standard_normal((16, d))
    r3, ri = ofl.flatness(X)
    want = 2.0 * math.sqrt(2.0 / math.pi) / math.sqrt(d)
    assert np.all(np.abs(r3 / want - 1.0) < 0.04)
    # the largest of d standard Gaussians is about sqrt(2 ln d)
    assert np.all((ri * math.sqrt(d) > 0.6 * math.sqrt(2 * math.log(d))) &
                  (ri * math.sqrt(d) < 1.4 * math.sqrt(2 * math.log(d))))


@pytest.mark.parametrize("support", [[1.0], [1.0, 1.0], [3.0, -1.0, 2.0], [1.0] * 6, [5.0, 1.0, 1.0, 1.0, 1.0],
                                     list(np.linspace(0.1, 1.0, 11))])
def test_one_rht_coordinate_obeys_berry_esseen_in_rho3(support):
    # One coordinate of H D x (full Hadamard, Rademacher D) times sqrt(d) is the
    # Rademacher sum sum_j s_j x^_j with x^ = x / ||x||.  Its Kolmogorov distance
    # to N(0, 1), computed exactly over all 2^k sign patterns, is at most
    # 0.5600 * rho3 (Berry-Esseen, non-identical summands, Shevtsova's constant).
    d = 64
    x = np.zeros(d)
    pos = np.arange(len(support)) * 5
    x[pos] = support
    rho3 = ofl.flatness(x)[0][0]
    H = rpbh.hadamard(d)                     # normalised rows: entries +-1/sqrt(d)
    xh = x / np.linalg.norm(x)
    i = 5
    vals = []
    for s in itertools.product((-1.0, 1.0), repeat=len(support)):
        D = np.ones(d); D[pos] = s
        vals.append(math.sqrt(d) * float(H[i] @ (D * xh)))
    vals = np.sort(np.array(vals))
    n = len(vals)
    # Kolmogorov distance of the discrete law to the standard normal CDF
    Phi = np.array([0.5 * (1 + math.erf(v / math.sqrt(2))) for v in vals])
    upper = np.arange(1, n + 1) / n
    lower = np.arange(0, n) / n
    dk = max(np.max(np.abs(upper - Phi)), np.max(np.abs(Phi - lower)))
    assert dk <= 0.5600 * rho3 + 1e-12
