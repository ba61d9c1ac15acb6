"""Pins for oracle.codebook (Lloyd-Max on the Beta coordinate law).

Each check is independent of the solver's own formulas: closed forms, an
independent incomplete-Beta routine (scipy), textbook Gaussian levels and the
TurboQuant page's distortion constants."""
import json
import math
import os

import numpy as np
import pytest
from scipy import integrate, special

from oracle import codebook as cb

CASES = [(64, 2), (64, 3), (128, 1), (128, 2), (128, 3), (128, 4), (1536, 3), (1536, 4)]


def closed_form_abs_mean(d):
    # E|X| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))
    return math.exp(math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d + 1) / 2))


@pytest.mark.parametrize("d,expected", [(64, 0.10012591), (128, 0.07066157), (1536, 0.02036175)])
def test_b1_centroid_closed_form(d, expected):
    c = cb.codebook(d, 1).centroids
    assert abs(c[1] - closed_form_abs_mean(d)) < 1e-13
    assert abs(c[1] - expected) < 5e-9
    assert c[0] == -c[1]


def _cdf(x, d):
    # (1+X)/2 ~ Beta((d-1)/2, (d-1)/2): independent incomplete-Beta routine
    a = (d - 1) / 2
    return special.betainc(a, a, (1 + np.asarray(x)) / 2)


@pytest.mark.parametrize("d,bits", CASES)
def test_fixed_point_against_incomplete_beta(d, bits):
    book = cb.codebook(d, bits)
    edges = np.concatenate([[-1.0], book.thresholds, [1.0]])
    mass = np.diff(_cdf(edges, d))
    lc = math.lgamma(d / 2) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2)
    # first moment by adaptive quadrature of x f_d(x) (scipy), not the closed form
    mom = []
    for a, b in zip(edges[:-1], edges[1:]):
        f = lambda x: x * math.exp(lc + 0.5 * (d - 3) * math.log1p(-x * x))
        lo, hi = max(a, -1 + 1e-15), min(b, 1 - 1e-15)
        brk = [p for p in np.linspace(-12, 12, 49) / math.sqrt(d) if lo < p < hi]
        val, _ = integrate.quad(f, lo, hi, points=brk or None, limit=400, epsabs=0, epsrel=1e-13)
        mom.append(val)
    cond_mean = np.array(mom) / mass
    assert np.max(np.abs(cond_mean - book.centroids)) < 1e-11
    assert abs(mass.sum() - 1.0) < 1e-12


@pytest.mark.parametrize("d,bits", CASES)
def test_symmetry_and_order(d, bits):
    book = cb.codebook(d, bits)
    c = book.centroids
    assert np.all(np.diff(c) > 0)
    assert np.max(np.abs(c + c[::-1])) < 1e-15
    assert np.all(book.thresholds == 0.5 * (c[:-1] + c[1:]))
    assert book.centroids32.dtype == np.float32


def test_distortion_matches_turboquant_page(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "turboquant_page_constants.json")))
    for d in (64, 128, 1536):
        f1 = d * cb.codebook(d, 1).mse_per_coord * 4
        # ~1.45 at b=1 (closed form: 4 (1 - d c1^2))
        assert abs(f1 - 4 * (1 - d * closed_form_abs_mean(d) ** 2)) < 1e-10
        assert abs(f1 - g["distortion_factor_b1_about"]) < 0.02
        for bits in (2, 3, 4):
            fb = d * cb.codebook(d, bits).mse_per_coord * 4 ** bits
            # within the ~2.7 factor (Panter-Dite high-rate constant sqrt(3) pi / 2)
            assert fb < math.sqrt(3) * math.pi / 2
            assert fb > f1


def test_gaussian_limit_textbook_levels(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "gaussian_lloyd_max_levels.json")))
    d = 1536
    for bits in (1, 2, 3, 4):
        levels = np.array(g["positive_levels"][str(bits)])
        c = cb.codebook(d, bits).centroids[1 << (bits - 1):] * math.sqrt(d)
        assert np.max(np.abs(c - levels) / levels) < 4e-3, (bits, c, levels)
        mse = d * cb.codebook(d, bits).mse_per_coord
        assert abs(mse - g["mse"][str(bits)]) / g["mse"][str(bits)] < 1e-2


def test_pdf_integrates_to_one_and_second_moment():
    for d in (64, 128, 1536):
        xs = np.linspace(-1, 1, 400001)
        f = cb.coord_pdf(xs, d)
        assert abs(np.trapezoid(f, xs) - 1) < 1e-6
        assert abs(np.trapezoid(xs * xs * f, xs) - 1 / d) < 1e-6 / d
