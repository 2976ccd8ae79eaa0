"""Sphere marginal f_d and the Lloyd-Max codebook C^(d,b) (oracle side, fp64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

[OQ] "Introduction and Theoretical Foundation / Theoretical Basis":
one coordinate t of a uniform point on S^{d-1} has density

    f_d(t) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - t^2)^((d-3)/2),  t in [-1, 1]

(also derived on [TQ] slides 14-15), and the codebook C^(d,b) is the 2^b-level
MSE-optimal (Lloyd-Max) scalar quantizer for it, built offline with no data
([OQ] eq. for q_hat, "Data-Agnostic Codebook"; [TQ] slide 16: "continuous
k-means").

Algorithm (Lloyd-Max, in its own order): start from centroids c, then repeat
  (1) boundaries beta_k = (c_k + c_{k+1}) / 2     (nearest-neighbour condition)
  (2) c_k = int_cell t f_d(t) dt / int_cell f_d(t) dt   (centroid condition)
until max_k |delta c_k| * sqrt(d) < TOL or MAX_ITERS iterations.

Numerical integration: substitute t = sin(theta); then
f_d(t) dt = C cos(theta)^(d-2) dtheta, smooth at the ends of the support for
every d >= 3.  The theta range is cut at min(pi/2, 40/sqrt(d-2)) (beyond that
cos^(d-2) < e^-800), split into equal panels of width <= 0.25/sqrt(d-2), and
each panel or part of a panel is integrated with 16-point Gauss-Legendre.
Whole panels are summed in extended precision so that small tail cells keep
their relative accuracy.

Readings of what the pages leave open:

* Initial centroids: linspace(-a, a, 2^b) with a = min(3/sqrt(d), 0.9).
  f_d is log-concave for d >= 3, so Lloyd-Max has one fixed point and the
  start only changes the iteration count.
* The optimum is symmetric; after convergence the centroids are made exactly
  antisymmetric (c_k = -c_{2^b-1-k}) so that the middle boundary is exactly 0.
* TOL = 1e-13 (in units of 1/sqrt(d)), MAX_ITERS = 200000.
"""

import math

import numpy as np

TOL = 1e-13
MAX_ITERS = 200000
GL_ORDER = 16


def log_fd_constant(d: int) -> float:
    """log of Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    return math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2.0)


def f_d(t, d: int):
    """The marginal density itself, for direct use in tests."""
    t = np.asarray(t, dtype=np.float64)
    out = np.zeros_like(t)
    inside = np.abs(t) < 1.0
    out[inside] = np.exp(log_fd_constant(d) + 0.5 * (d - 3) * np.log1p(-t[inside] ** 2))
    return out


class _ThetaIntegrator:
    """Composite Gauss-Legendre in theta for  int g(sin theta) C cos^(d-2)(theta) dtheta."""

    def __init__(self, d: int):
        if d < 3:
            raise ValueError("d >= 3 required")
        self.d = d
        self.logC = log_fd_constant(d)
        self.theta_max = min(math.pi / 2.0, 40.0 / math.sqrt(d - 2.0))
        width = 0.25 / math.sqrt(d - 2.0)
        per_side = max(1, math.ceil(self.theta_max / width))
        self.n_panels = 2 * per_side
        self.edges = np.linspace(-self.theta_max, self.theta_max, self.n_panels + 1)
        self.x, self.w = np.polynomial.legendre.leggauss(GL_ORDER)
        # Whole-panel integrals of the three moments (t^0, t^1, t^2).
        lo, hi = self.edges[:-1], self.edges[1:]
        self.panel = [self._gl(lo, hi, p) for p in range(3)]
        self.cum = [np.concatenate([[0.0], np.cumsum(v.astype(np.longdouble))]) for v in self.panel]

    def _weight(self, theta):
        c = np.cos(theta)
        with np.errstate(divide="ignore"):
            return np.exp(self.logC + (self.d - 2) * np.log(np.maximum(c, 0.0)))

    def _gl(self, a, b, power):
        """Gauss-Legendre on [a, b] (vectorised over a, b) of sin^power * C cos^(d-2)."""
        a = np.asarray(a, dtype=np.float64)
        b = np.asarray(b, dtype=np.float64)
        half = 0.5 * (b - a)
        mid = 0.5 * (b + a)
        th = mid[..., None] + half[..., None] * self.x
        vals = self._weight(th) * np.sin(th) ** power
        return half * (vals @ self.w)

    def cell_integrals(self, t_edges, power):
        """int over [t_edges[k], t_edges[k+1]] of t^power f_d(t) dt, for every k."""
        th = np.arcsin(np.clip(np.asarray(t_edges, dtype=np.float64), -1.0, 1.0))
        th = np.clip(th, -self.theta_max, self.theta_max)
        p = np.floor((th + self.theta_max) / (self.edges[1] - self.edges[0])).astype(np.int64)
        p = np.clip(p, 0, self.n_panels - 1)
        a, b = th[:-1], th[1:]
        pa, pb = p[:-1], p[1:]
        same = pa == pb
        out = np.zeros(len(a), dtype=np.float64)
        # cells inside one panel
        out[same] = self._gl(a[same], b[same], power)
        # cells spanning panels: tail of panel pa + whole panels in between + head of panel pb
        sp = ~same
        if np.any(sp):
            right = self._gl(a[sp], self.edges[pa[sp] + 1], power)
            left = self._gl(self.edges[pb[sp]], b[sp], power)
            mid = (self.cum[power][pb[sp]] - self.cum[power][pa[sp] + 1]).astype(np.float64)
            out[sp] = right + mid + left
        return out


def lloyd_max(d: int, bits: int, tol: float = TOL, max_iters: int = MAX_ITERS):
    """Lloyd-Max codebook for f_d with 2^bits levels.

    Returns dict(centroids, boundaries, iterations, distortion) with
    centroids float64[2^b] ascending, boundaries float64[2^b - 1] (midpoints),
    distortion = int (t - q(t))^2 f_d(t) dt per coordinate.
    """
    if not (1 <= bits <= 8):
        raise ValueError("bits in 1..8")
    L = 1 << bits
    integ = _ThetaIntegrator(d)
    sd = math.sqrt(d)
    a = min(3.0 / sd, 0.9)
    c = np.linspace(-a, a, L)
    it = 0
    for it in range(1, max_iters + 1):
        beta = 0.5 * (c[1:] + c[:-1])                       # step (1)
        edges = np.concatenate([[-1.0], beta, [1.0]])
        m0 = integ.cell_integrals(edges, 0)
        m1 = integ.cell_integrals(edges, 1)
        c_new = m1 / m0                                      # step (2)
        delta = np.max(np.abs(c_new - c)) * sd
        c = c_new
        if delta < tol:
            break
    c = 0.5 * (c - c[::-1])                                  # exact antisymmetry
    beta = 0.5 * (c[1:] + c[:-1])
    edges = np.concatenate([[-1.0], beta, [1.0]])
    m0 = integ.cell_integrals(edges, 0)
    m1 = integ.cell_integrals(edges, 1)
    m2 = integ.cell_integrals(edges, 2)
    distortion = float(np.sum(m2 - 2.0 * c * m1 + c * c * m0))
    return {"centroids": c, "boundaries": beta, "iterations": it, "distortion": distortion}


def fp16_lut(centroids: np.ndarray, d: int) -> np.ndarray:
    """Declared dequantisation table: fp16 (round to nearest even) of sqrt(d) * c_k.

    The pages fix no dequant precision; this reading keeps the GEMM operands on
    the 16-bit tensor-core path.  Returned as float16.
    """
    return (np.sqrt(d) * np.asarray(centroids, dtype=np.float64)).astype(np.float16)
