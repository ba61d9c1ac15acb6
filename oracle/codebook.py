"""Lloyd-Max scalar codebooks for the coordinate law of a randomly rotated unit vector.

Sources:
* "Google presenta TurboQuant..." (7minutos.es), section "La mecanica geometrica
  de TurboQuant": a random rotation makes every coordinate follow a Beta law on
  [-1, 1]; the b-bit quantizer minimises the MSE cost C(f_X, b), a 1-D
  k-means / Lloyd-Max problem solved once offline and stored.
* "FibQuant ..." (gist.science 2605.11478), section 2.1 "La Sorgente Canonica":
  after normalisation and a Haar rotation the unit vector is uniform on
  S^{d-1}; one coordinate of it is the k=1 case of the spherical-Beta law.

Reading (where the pages are silent): the density is the marginal of one
coordinate of a uniform point on S^{d-1},
    f_d(x) = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) * (1 - x^2)^((d-3)/2),
equivalently (1+X)/2 ~ Beta((d-1)/2, (d-1)/2).  The cost integral's outer
cells extend to the support ends -1 and +1; thresholds are midpoints of
adjacent centroids.  Centroids and thresholds are solved in fp64 and stored
as fp32.

Method: cell masses by composite Gauss-Legendre quadrature (equal pieces per
cell), first moments in closed form, plain Lloyd iteration from evenly spaced
centroids until the largest centroid move is below 1e-14.  Because f_d is even
the fixed point is odd-symmetric; each step is symmetrised so rounding cannot
break that (the middle threshold of an even number of levels stays exactly 0).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

_GL_X, _GL_W = np.polynomial.legendre.leggauss(24)
_PIECES = 64


def log_norm_const(d: int) -> float:
    """log of Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2))."""
    return math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2.0)


def coord_pdf(x, d: int) -> np.ndarray:
    """f_d(x) on [-1, 1] (zero outside)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    inside = np.abs(x) < 1.0
    out[inside] = np.exp(log_norm_const(d) + 0.5 * (d - 3) * np.log1p(-x[inside] ** 2))
    return out


def _quad_cells(edges: np.ndarray, d: int, fn) -> np.ndarray:
    """Integral of fn(x) * f_d(x) over each cell [edges[m], edges[m+1]]."""
    a, b = edges[:-1], edges[1:]
    frac = np.linspace(0.0, 1.0, _PIECES + 1)
    pe = a[:, None] + (b - a)[:, None] * frac[None, :]          # [cells, pieces+1]
    lo, hi = pe[:, :-1], pe[:, 1:]
    half = 0.5 * (hi - lo)
    mid = 0.5 * (hi + lo)
    xs = mid[..., None] + half[..., None] * _GL_X                 # [cells, pieces, nodes]
    vals = fn(xs) * coord_pdf(xs, d)
    return np.sum(half[..., None] * _GL_W * vals, axis=(1, 2))


def cell_masses(edges: np.ndarray, d: int) -> np.ndarray:
    return _quad_cells(edges, d, lambda x: np.ones_like(x))


def cell_first_moments(edges: np.ndarray, d: int) -> np.ndarray:
    """Closed form: int_a^b x f_d(x) dx = C_d/(d-1) [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)]."""
    c = math.exp(log_norm_const(d)) / (d - 1)

    def g(x):
        x = np.asarray(x, dtype=np.float64)
        out = np.zeros_like(x)
        inside = np.abs(x) < 1.0
        out[inside] = np.exp(0.5 * (d - 1) * np.log1p(-x[inside] ** 2))
        return out

    return c * (g(edges[:-1]) - g(edges[1:]))


@dataclass(frozen=True)
class Codebook:
    d: int
    bits: int
    centroids: np.ndarray      # fp64, ascending, 2^bits
    thresholds: np.ndarray     # fp64, 2^bits - 1 midpoints
    mse_per_coord: float       # E[(X - Q(X))^2] at the fixed point
    iterations: int

    @property
    def centroids32(self) -> np.ndarray:
        return self.centroids.astype(np.float32)

    @property
    def thresholds32(self) -> np.ndarray:
        return self.thresholds.astype(np.float32)


def lloyd_max(d: int, bits: int, tol: float = 1e-14, max_iter: int = 500000) -> Codebook:
    """Solve the Lloyd-Max conditions c_m = E[X | t_m <= X < t_{m+1}],
    t_k = (c_{k-1} + c_k)/2 for f_d, following the MSE cost C(f_X, b) of the
    TurboQuant page ("La mecanica geometrica de TurboQuant")."""
    if d < 4 or bits < 1:
        raise ValueError("need d >= 4 and bits >= 1")
    n = 1 << bits
    sigma = 1.0 / math.sqrt(d)
    c = sigma * np.linspace(-2.0, 2.0, n) if n > 2 else np.array([-sigma, sigma])
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[:-1] + c[1:])
        edges = np.concatenate([[-1.0], t, [1.0]])
        c_new = cell_first_moments(edges, d) / cell_masses(edges, d)
        c_new = 0.5 * (c_new - c_new[::-1])   # f_d is even: keep c exactly odd
        moved = float(np.max(np.abs(c_new - c)))
        c = c_new
        if moved < tol:
            break
    t = 0.5 * (c[:-1] + c[1:])
    edges = np.concatenate([[-1.0], t, [1.0]])
    mse = float(np.sum([
        _quad_cells(edges[m:m + 2], d, lambda x, cm=c[m]: (x - cm) ** 2)[0] for m in range(n)
    ]))
    return Codebook(d, bits, c, t, mse, it)


_CACHE: dict[tuple[int, int], Codebook] = {}


def codebook(d: int, bits: int) -> Codebook:
    key = (d, bits)
    if key not in _CACHE:
        _CACHE[key] = lloyd_max(d, bits)
    return _CACHE[key]
