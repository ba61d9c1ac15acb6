"""Pins for the oracle's FibQuant k = 2 codec (``oracle/fibquant.py``), against
the mathematics of "FibQuant ..." (gist.science 2605.11478) sections 2.1-2.3
and independent computations:
* the block law f_{d,2} is the law of two coordinates of a uniform point on
  S^{d-1} (Monte Carlo on normalised Gaussians; closed-form normalisation);
* the starting radii are the Bennett-Gersho companding quantiles (independent
  numerical integration and root finding with scipy);
* directions advance by the golden angle;
* the refined code is a Lloyd fixed point of the true law (cell means and MSE
  by independent Monte Carlo) and beats the scalar Lloyd-Max product code at
  the same rate (section 3.2, the vector code dominates the scalar product);
* encode, layout and decode against plain loops; rate log2(N)/2 per coordinate.
"""
import math

import numpy as np
import pytest
from scipy import integrate, optimize

from oracle import codebook as ocb
from oracle import fibquant as fq
from rotated_codebook_kv_tq_b200 import synth


def _sphere_pairs(d, n, seed):
    g = np.random.default_rng(seed).standard_normal((n, d))
    g /= np.linalg.norm(g, axis=1, keepdims=True)
    return g.reshape(n * d // 2, 2)


@pytest.mark.parametrize("d", [16, 128])
def test_pair_law_is_the_sphere_marginal(d):
    # closed-form normalisation over the disk, by polar quadrature
    tot, _ = integrate.quad(lambda r: 2 * math.pi * r * fq.pair_density(np.array([r, 0.0]), d), 0, 1)
    assert abs(tot - 1) < 1e-9
    # |x|^2 of Monte Carlo pairs against the Beta(1, (d-2)/2) CDF (KS distance)
    pairs = _sphere_pairs(d, 40000, 1)[::d // 2]           # one pair per vector: independent
    t = np.sort(np.sum(pairs ** 2, axis=1))
    cdf = 1 - (1 - t) ** ((d - 2) / 2)
    ks = np.max(np.abs(cdf - (np.arange(1, len(t) + 1) - 0.5) / len(t)))
    assert ks < 1.63 / math.sqrt(len(t)) + 1e-3


@pytest.mark.parametrize("d", [16, 128])
def test_quadrature_moments(d):
    pts = fq.quadrature(d)
    assert abs(np.mean(np.sum(pts ** 2, axis=1)) / (2.0 / d) - 1) < 1e-12   # E|x|^2 = 2/d
    assert abs(np.mean(pts[:, 0])) < 1e-12 and abs(np.mean(pts[:, 0] * pts[:, 1])) < 1e-12


@pytest.mark.parametrize("d,N", [(16, 8), (128, 16)])
def test_start_radii_are_bennett_gersho_quantiles(d, N):
    dens = lambda r: 2 * math.pi * r * math.sqrt(fq.pair_density(np.array([r, 0.0]), d))
    total, _ = integrate.quad(dens, 0, 1, epsabs=1e-13)
    cb = fq.start_codebook(d, N)
    r = np.linalg.norm(cb, axis=1)
    for n in range(N):
        target = (n + 0.5) / N
        rn = optimize.brentq(lambda x: integrate.quad(dens, 0, x, epsabs=1e-13)[0] / total - target,
                             0, 1, xtol=1e-14)
        assert abs(r[n] - rn) < 1e-8, (n, r[n], rn)
    # golden-angle directions
    th = np.arctan2(cb[:, 1], cb[:, 0])
    step = np.mod(np.diff(th), 2 * math.pi)
    np.testing.assert_allclose(step, fq.GOLDEN_ANGLE, atol=1e-12)


@pytest.mark.parametrize("d,bits", [(64, 3), (128, 4)])
def test_refined_code_is_a_lloyd_fixed_point(d, bits):
    cb = fq.pair_codebook(d, bits)
    c = cb.centroids
    pairs = _sphere_pairs(d, 40000, 7)                     # 40000 * d/2 pairs
    idx, dist = fq._nearest(pairs, c)
    N = 1 << bits
    for n in range(N):
        sel = pairs[idx == n]
        se = np.std(sel, axis=0) / math.sqrt(len(sel))
        assert np.all(np.abs(sel.mean(axis=0) - c[n]) < 5 * se + 2e-4 / math.sqrt(d)), n
    mc = dist.mean()
    assert abs(mc / cb.mse_per_pair - 1) < 0.01
    # refinement lowers the quadrature MSE of the deterministic start
    pts = fq.quadrature(d)
    assert cb.mse_per_pair <= fq.quad_mse(fq.start_codebook(d, N), pts) + 1e-15


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 2), (64, 4), (128, 4), (128, 6)])
def test_vector_code_beats_scalar_product_at_equal_rate(d, bits):
    """m bits per pair = m/2 bits per coordinate; the scalar product code with
    m/2 bits per coordinate is one particular 2^m-point code of the plane.
    At 4 points the square (product) code is already the best one for a
    radially symmetric law, so the two agree up to the quadrature; from 16
    points on the vector code is strictly better (cell shape and density fit,
    section 3.2)."""
    vec = fq.pair_codebook(d, bits).mse_per_pair
    scalar = 2 * ocb.codebook(d, bits // 2).mse_per_coord
    if bits == 2:
        assert abs(vec / scalar - 1) < 1e-3, (vec, scalar)
    else:
        assert vec < 0.95 * scalar, (vec, scalar)


def _codec(d, bk, bv, seed=3):
    return fq.make_codec(d, bk, bv, synth.rotation_signs(d, seed))


def test_encode_is_nearest_codeword_by_loops():
    c = _codec(32, 3, 2)
    x = np.random.default_rng(2).standard_normal((5, 32))
    enc = fq.encode(x, c.Pi, c.cb_k)
    cb = c.cb_k.centroids32.astype(float)
    for r in range(5):
        u = enc["u"][r].astype(np.float32).astype(float)
        for j in range(16):
            best, bd = 0, None
            for n in range(len(cb)):
                dd = (u[2 * j] - cb[n][0]) ** 2 + (u[2 * j + 1] - cb[n][1]) ** 2
                if bd is None or dd < bd:
                    best, bd = n, dd
            assert enc["idx"][r, j] == best


def test_layout_and_rate():
    d, T = 32, 40
    c = _codec(d, 3, 2)
    assert fq.bytes_per_row(c) == (3 * d // 16 + 4, 2 * d // 16 + 2)
    assert c.cb_k.rate == 1.5 and c.cb_v.rate == 1.0
    rng = np.random.default_rng(5)
    K, V = rng.standard_normal((1, 1, T, d)), rng.standard_normal((1, 1, T, d))
    cache = fq.empty_cache(c, 1, 1, 64)
    diag = fq.quantize_into(cache, K, V, c)
    ik, iv = diag["k"][0]["idx"], diag["v"][0]["idx"]
    for t in range(T):
        for j in range(d // 2):
            for p in range(3):
                assert (int(cache["kcode"][0, 0, t, p, j // 8]) >> (j % 8)) & 1 == (ik[t, j] >> p) & 1
            for p in range(2):
                w = int(cache["vcode"][0, 0, t // 32, p, j])
                assert (w >> (t % 32)) & 1 == (iv[t, j] >> p) & 1
    # appends into a partly covered value group keep the other rows
    before = cache["vcode"].copy()
    fq.quantize_into(cache, K[:, :, :3], V[:, :, :3], c, row0=T)
    assert np.array_equal(fq.cache_rows(cache, c, 0, 0, T)[2], iv)
    assert not np.array_equal(before, cache["vcode"])


def test_decode_matches_loops():
    d, T, Hq = 16, 37, 2
    c = _codec(d, 4, 3)
    rng = np.random.default_rng(8)
    K, V = rng.standard_normal((1, 1, T, d)) * 2, rng.standard_normal((1, 1, T, d))
    q = rng.standard_normal((1, Hq, d))
    cos, sin = synth.rope_table(64, d, 100.0)
    cache = fq.empty_cache(c, 1, 1, 64)
    fq.quantize_into(cache, K, V, c, rope=(cos, sin))
    out = fq.decode(q, cache, c, [T], 0.4, rope=(cos, sin))
    ik, nk, iv, nv = fq.cache_rows(cache, c, 0, 0, T)
    Pi = c.Pi
    ck, cv = c.cb_k.centroids32.astype(float), c.cb_v.centroids32.astype(float)

    def recon(idx, nu, cb):
        y = [cb[idx[j // 2]][j % 2] for j in range(d)]
        return [nu * sum(Pi[i][a] * y[i] for i in range(d)) for a in range(d)]
    keys = [recon(ik[t], nk[t], ck) for t in range(T)]
    vals = [recon(iv[t], nv[t], cv) for t in range(T)]
    for h in range(Hq):
        x = list(q[0, h])
        hh = d // 2
        qr = [0.0] * d
        for i in range(hh):
            cc, ss = float(cos[T - 1, i]), float(sin[T - 1, i])
            qr[i] = x[i] * cc - x[i + hh] * ss
            qr[i + hh] = x[i + hh] * cc + x[i] * ss
        lg = [0.4 * sum(qr[a] * keys[t][a] for a in range(d)) for t in range(T)]
        m = max(lg)
        w = [math.exp(l - m) for l in lg]
        expect = [sum(w[t] * vals[t][a] for t in range(T)) / sum(w) for a in range(d)]
        np.testing.assert_allclose(out[0, h], expect, rtol=1e-10, atol=1e-12)
