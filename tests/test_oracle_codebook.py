"""Pins for the oracle's f_d and Lloyd-Max codebook (CPU only).

Independent references used here (none of them calls the oracle's integrator):
* the law of one coordinate of a uniform point on S^{d-1}: t^2 ~ Beta(1/2, (d-1)/2)
  (scipy.special.betainc), and the closed-form first moment of f_d;
* direct quadrature of the density formula printed on the OrbitQuant page
  ("Theoretical Basis") with scipy.integrate.quad;
* the closed-form 1-bit optimum and the d = 3 uniform case;
* the Gaussian Lloyd-Max quantizer (scipy.stats.norm closed forms), the d >= 64
  limit stated on the OrbitQuant page and derived on TurboQuant slide 15;
* the centroids printed on TurboQuant slide 16 and the distortion bounds of slide 17;
* Monte-Carlo points on the sphere and brute-force minimisation for d <= 16.
"""

import math
import os

import numpy as np
import pytest
from scipy import integrate, optimize, special, stats

from oracle import codebook as cbm
from oracle.quantize import nearest_centroid

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _beta_cdf(t, d):
    """P(T <= t) for one coordinate of a uniform point on S^{d-1}."""
    t = np.asarray(t, dtype=np.float64)
    half = 0.5 * special.betainc(0.5, 0.5 * (d - 1), np.minimum(t * t, 1.0))
    return 0.5 + np.sign(t) * half


def _first_moment(a, b, d):
    """int_a^b t f_d(t) dt in closed form: C/(d-1) [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)]."""
    C = math.exp(cbm.log_fd_constant(d))
    return C / (d - 1) * ((1 - a * a) ** ((d - 1) / 2) - (1 - b * b) ** ((d - 1) / 2))


def _printed_density(t, d):
    # the formula as printed on the OrbitQuant page, evaluated with scipy's gamma
    return special.gamma(d / 2) / (math.sqrt(math.pi) * special.gamma((d - 1) / 2)) * (1 - t * t) ** ((d - 3) / 2)


@pytest.mark.parametrize("d", [3, 4, 16, 64, 100])
def test_fd_matches_printed_formula_and_normalises(d):
    ts = np.linspace(-0.99, 0.99, 41)
    assert np.allclose(cbm.f_d(ts, d), _printed_density(ts, d), rtol=1e-12)
    total, _ = integrate.quad(lambda t: _printed_density(t, d), -1, 1)
    second, _ = integrate.quad(lambda t: t * t * _printed_density(t, d), -1, 1)
    assert abs(total - 1) < 1e-10
    assert abs(second - 1.0 / d) < 1e-10


def test_fd_d3_is_uniform():
    assert np.allclose(cbm.f_d(np.linspace(-0.9, 0.9, 7), 3), 0.5, rtol=1e-14)


@pytest.mark.parametrize("d", [3, 5, 16, 64, 256, 3072, 12288])
def test_integrator_cell_masses_match_beta_law(d):
    integ = cbm._ThetaIntegrator(d)
    sd = math.sqrt(d)
    edges = np.concatenate([[-1.0], np.linspace(-3.5, 3.5, 15) / sd, [1.0]])
    edges = np.clip(edges, -1, 1)
    m0 = integ.cell_integrals(edges, 0)
    ref0 = np.diff(_beta_cdf(edges, d))
    assert np.allclose(m0, ref0, rtol=1e-10, atol=1e-15)
    m1 = integ.cell_integrals(edges, 1)
    ref1 = np.array([_first_moment(a, b, d) for a, b in zip(edges[:-1], edges[1:])])
    assert np.allclose(m1, ref1, rtol=1e-10, atol=1e-16)


@pytest.mark.parametrize("d", [3, 8, 64, 256, 1536, 3072, 12288])
def test_one_bit_closed_form(d, codebooks):
    # optimum for 1 bit: +-E|t| = +-Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    c = codebooks(d, 1)["centroids"]
    e_abs = math.exp(math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2))
    assert np.allclose(c, [-e_abs, e_abs], rtol=1e-12)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_d3_uniform_closed_form(bits, codebooks):
    # f_3 = 1/2 on [-1, 1]: Lloyd-Max is the uniform quantizer
    L = 1 << bits
    cb = codebooks(3, bits)
    expect = (2 * np.arange(L) + 1) / L - 1
    assert np.allclose(cb["centroids"], expect, atol=1e-12)
    assert abs(cb["distortion"] - (2.0 / L) ** 2 / 12) < 1e-13


@pytest.mark.parametrize("d,bits", [(64, 2), (64, 4), (256, 4), (3072, 4), (3072, 6), (8960, 4), (12288, 2)])
def test_lloyd_max_fixed_point_conditions(d, bits, codebooks):
    cb = codebooks(d, bits)
    c, beta = cb["centroids"], cb["boundaries"]
    L = 1 << bits
    assert np.all(np.diff(c) > 0)
    assert np.array_equal(beta, 0.5 * (c[1:] + c[:-1]))             # midpoint condition
    assert np.array_equal(c, -c[::-1])                               # exact symmetry
    assert beta[L // 2 - 1] == 0.0
    edges = np.concatenate([[-1.0], beta, [1.0]])
    mass = np.diff(_beta_cdf(edges, d))
    mom = np.array([_first_moment(a, b, d) for a, b in zip(edges[:-1], edges[1:])])
    cond_mean = mom / mass                                           # centroid condition
    sd = math.sqrt(d)
    assert np.max(np.abs(cond_mean - c)) * sd < 1e-9


def _gauss_lloyd_max(L, iters=20000):
    """Lloyd-Max for N(0, 1) with closed-form cell means (scipy.stats.norm)."""
    c = np.linspace(-2.0, 2.0, L)
    for _ in range(iters):
        b = 0.5 * (c[1:] + c[:-1])
        e = np.concatenate([[-np.inf], b, [np.inf]])
        m = stats.norm.cdf(e[1:]) - stats.norm.cdf(e[:-1])
        new = (stats.norm.pdf(e[:-1]) - stats.norm.pdf(e[1:])) / m
        if np.max(np.abs(new - c)) < 1e-13:
            c = new
            break
        c = new
    return c


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_gaussian_limit(bits, codebooks):
    # f_d ~ N(0, 1/d) for d >= 64: sqrt(d) C^(d,b) approaches the Gaussian Lloyd-Max
    # quantizer, with an O(1/d) gap.
    g = _gauss_lloyd_max(1 << bits)
    gaps = []
    for d in (256, 3072, 12288):
        c = codebooks(d, bits)["centroids"] * math.sqrt(d)
        gaps.append(np.max(np.abs(c - g)))
    assert gaps[0] > gaps[1] > gaps[2]
    assert gaps[2] < 1e-3
    # O(1/d): a 4x larger d shrinks the gap about 4x (12x for 256 -> 3072)
    assert 3.0 < gaps[1] / gaps[2] < 5.0
    assert 9.0 < gaps[0] / gaps[1] < 15.0


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def test_printed_centroids_slide16(codebooks):
    for row in _read_table("turboquant_slide16_centroids.txt"):
        bits, decimals = int(row[0]), int(row[1])
        printed = np.array([float(v) for v in row[2:]])
        for d in (3072, 12288):
            c = codebooks(d, bits)["centroids"] * math.sqrt(d)
            pos = c[len(c) // 2:]
            tol = 0.5 * 10.0 ** (-min(decimals, 3)) + 2.0 / d
            assert np.all(np.abs(pos - printed) <= tol), (bits, d, pos, printed)


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 5, 6])
def test_distortion_sandwich_slide17(bits, codebooks):
    consts = {r[0]: float(r[1]) for r in _read_table("turboquant_slide17_bounds.txt")}
    for d in (64, 3072):
        if bits >= 5 and d == 64:
            continue
        total = d * codebooks(d, bits)["distortion"]
        assert consts["lower_factor"] * 4.0 ** -bits <= total <= consts["upper_factor"] * 4.0 ** -bits


@pytest.mark.parametrize("d,bits", [(16, 2), (64, 4), (256, 4)])
def test_monte_carlo_on_sphere(d, bits, codebooks):
    # Uniform points on S^{d-1} (normalised Gaussians): the coordinate law is f_d
    # (KS test against the Beta law) and the per-coordinate MSE of nearest-centroid
    # quantization equals the codebook's distortion.
    rng = np.random.default_rng(123)
    n = 20000
    g = rng.standard_normal((n, d))
    pts = g / np.linalg.norm(g, axis=1, keepdims=True)
    ks = stats.kstest(pts[:, 0], lambda t: _beta_cdf(t, d))
    assert ks.pvalue > 1e-3
    cb = codebooks(d, bits)
    q = cb["centroids"][nearest_centroid(pts, cb["centroids"])]
    per_coord = np.mean((pts - q) ** 2, axis=0)
    mse = per_coord.mean()
    se = per_coord.std() / math.sqrt(d) + np.std((pts - q) ** 2) / math.sqrt(n * d) * 3
    assert abs(mse - cb["distortion"]) < 6 * se + 1e-3 * cb["distortion"]


@pytest.mark.parametrize("d", [4, 8, 16])
def test_brute_force_small_d(d, codebooks):
    # direct minimisation of the distortion over symmetric centroid positions,
    # with the distortion evaluated by scipy quadrature of the printed density
    def dist(cpos):
        c = np.sort(np.concatenate([-cpos, cpos]))
        b = 0.5 * (c[1:] + c[:-1])
        e = np.concatenate([[-1.0], b, [1.0]])
        tot = 0.0
        for k in range(len(c)):
            v, _ = integrate.quad(lambda t: (t - c[k]) ** 2 * _printed_density(t, d), e[k], e[k + 1],
                                  epsabs=1e-14, epsrel=1e-12)
            tot += v
        return tot
    # 1 bit: one parameter
    r1 = optimize.minimize_scalar(lambda x: dist(np.array([x])), bounds=(0.01, 0.99), method="bounded",
                                  options={"xatol": 1e-12})
    assert abs(r1.x - codebooks(d, 1)["centroids"][1]) < 1e-6
    # 2 bits: two parameters
    c2 = codebooks(d, 2)["centroids"][2:]
    r2 = optimize.minimize(lambda x: dist(np.sort(np.abs(x))), x0=c2 * 0.8 + 0.05, method="Nelder-Mead",
                           options={"xatol": 1e-10, "fatol": 1e-16, "maxiter": 4000})
    assert np.allclose(np.sort(np.abs(r2.x)), c2, atol=1e-5)
    assert dist(c2) <= r2.fun + 1e-14


def test_fp16_lut_declared_rounding(codebooks):
    cb = codebooks(3072, 4)
    lut = cbm.fp16_lut(cb["centroids"], 3072)
    exact = math.sqrt(3072) * cb["centroids"]
    # round to nearest: within half an fp16 ulp of the exact scaled centroid
    ulp = np.spacing(lut.astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(lut.astype(np.float64) - exact) <= 0.5 * ulp)
    assert lut.dtype == np.float16
