"""Data-independent Lloyd-Max codebook for a rotated unit-vector coordinate.

TEST INFRASTRUCTURE (see ``oracle/__init__``).

[tqai] section "TurboQuant的核心创新：极坐标量化与随机旋转": after the random
rotation each coordinate follows a concentrated Beta law, nearly
independent of the others, so an optimal scalar (Lloyd-Max) quantiser can
be precomputed from the known density alone, with no calibration data.

The density of one coordinate of a uniform point on the unit sphere in
R^d is

    f_d(x) = C_d (1 - x^2)^((d-3)/2),  |x| <= 1,
    C_d    = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)).

Lloyd-Max (Lloyd 1957/1982, Max 1960) alternates the two optimality
conditions of a scalar quantiser with 2^b cells:

    t_j = (c_j + c_{j+1}) / 2                       (nearest neighbour)
    c_j = int_{t_{j-1}}^{t_j} x f / int_{t_{j-1}}^{t_j} f   (centroid)

with t_{-1} = -1 and t_{2^b-1} = +1.  Readings for what the pages leave
open: start from 2^b points evenly spaced inside +-min(1, 3/sqrt(d)); stop
when no centroid moves by more than 1e-15 times the largest centroid (or
after 200000 sweeps); then
make the table exactly odd-symmetric, c_j = -c_{2^b-1-j}, which the
density's symmetry implies.  f_d is log-concave for d >= 3, so the fixed
point is unique (Fleischer 1964) and the start does not matter.

Integrals: the numerator has the closed form
    int_a^b x f_d = C_d [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1);
the cell mass is integrated by composite Gauss-Legendre quadrature after
the substitution x = sin(theta), which turns (1-x^2)^((d-3)/2) dx into the
smooth cos(theta)^(d-2) dtheta.
"""

import math

import numpy as np

_GL_NODES, _GL_WEIGHTS = np.polynomial.legendre.leggauss(32)


def density_constant(d):
    """C_d, the normalising constant of f_d."""
    return math.exp(math.lgamma(d / 2.0) - math.lgamma((d - 1) / 2.0)) / math.sqrt(math.pi)


def density(x, d):
    """f_d(x) for |x| <= 1 (zero outside)."""
    x = np.asarray(x, dtype=np.float64)
    inside = np.abs(x) <= 1.0
    val = np.zeros_like(x)
    xi = x[inside]
    val[inside] = density_constant(d) * np.exp((d - 3) / 2.0 * np.log1p(-xi * xi))
    return val


def cell_mass(a, b, d):
    """P(a < X < b) for X ~ f_d, by composite Gauss-Legendre in theta."""
    if b <= a:
        return 0.0
    ta, tb = math.asin(max(-1.0, a)), math.asin(min(1.0, b))
    if d > 3:
        lim = min(math.pi / 2, 14.0 / math.sqrt(d - 2))
        ta, tb = max(ta, -lim), min(tb, lim)
        if tb <= ta:
            return 0.0
    h = min(0.25, 1.0 / math.sqrt(d))
    pieces = max(1, int(math.ceil((tb - ta) / h)))
    edges = np.linspace(ta, tb, pieces + 1)
    lo, hi = edges[:-1, None], edges[1:, None]
    theta = 0.5 * (hi - lo) * _GL_NODES[None, :] + 0.5 * (hi + lo)
    # cos(theta)^(d-2) with log(cos theta) = log1p(-2 sin^2(theta/2)), accurate near 0
    vals = np.exp((d - 2) * np.log1p(-2.0 * np.sin(0.5 * theta) ** 2))
    total = np.sum(0.5 * (hi - lo) * (vals * _GL_WEIGHTS[None, :]))
    return density_constant(d) * float(total)


def cell_moment(a, b, d):
    """int_a^b x f_d(x) dx, closed form."""
    a, b = max(-1.0, a), min(1.0, b)
    if b <= a:
        return 0.0
    p = (d - 1) / 2.0
    pa = math.exp(p * math.log1p(-a * a)) if abs(a) < 1.0 else 0.0
    pb = math.exp(p * math.log1p(-b * b)) if abs(b) < 1.0 else 0.0
    return density_constant(d) * (pa - pb) / (d - 1)


def _lloyd_max(mass_fn, moment_fn, lo, hi, n_cells, start_span, tol, max_iter):
    c = np.array([-start_span + (2 * j + 1) * start_span / n_cells for j in range(n_cells)])
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[lo], t, [hi]])
        new = np.array([moment_fn(edges[j], edges[j + 1]) / mass_fn(edges[j], edges[j + 1])
                        for j in range(n_cells)])
        moved = np.max(np.abs(new - c))
        c = new
        if moved <= tol * np.max(np.abs(c)):
            break
    c = 0.5 * (c - c[::-1])
    return c


def lloyd_max(d, bits, tol=1e-15, max_iter=200000):
    """Centroids (2^bits,) and boundaries (2^bits - 1,) for f_d, fp64."""
    if d < 3:
        raise ValueError("the density is defined for d >= 3")
    n = 1 << bits
    c = _lloyd_max(lambda a, b: cell_mass(a, b, d), lambda a, b: cell_moment(a, b, d),
                   -1.0, 1.0, n, min(1.0, 3.0 / math.sqrt(d)), tol, max_iter)
    t = 0.5 * (c[:-1] + c[1:])
    return c, t


def cell_masses(boundaries, d):
    """P_j for every cell of the given boundaries."""
    edges = np.concatenate([[-1.0], np.asarray(boundaries, dtype=np.float64), [1.0]])
    return np.array([cell_mass(edges[j], edges[j + 1], d) for j in range(len(edges) - 1)])


def distortion(centroids, boundaries, d):
    """Per-coordinate MSE D = E[X^2] - sum_j P_j c_j^2 (valid at the centroid condition)."""
    p = cell_masses(boundaries, d)
    return 1.0 / d - float(np.sum(p * np.asarray(centroids) ** 2))


def gaussian_lloyd_max(bits, tol=1e-15, max_iter=200000):
    """Lloyd-Max quantiser of N(0,1), the d -> infinity limit of sqrt(d) X."""
    def mass(a, b):
        return 0.5 * (math.erfc(-b / math.sqrt(2.0)) - math.erfc(-a / math.sqrt(2.0)))

    def moment(a, b):
        phi = lambda x: 0.0 if math.isinf(x) else math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
        return phi(a) - phi(b)

    n = 1 << bits
    c = _lloyd_max(mass, moment, -math.inf, math.inf, n, 3.0, tol, max_iter)
    return c, 0.5 * (c[:-1] + c[1:])
