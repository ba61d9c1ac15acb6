"""Pins for the oracle's dense Haar rotation (``oracle/rotation.haar_rotation``)
and for codecs built on it: orthogonality, the Haar law (moments of one entry,
the sign-fixed first column, and the Beta coordinate law of a rotated fixed
vector, which is the premise of every codebook: "Google presenta TurboQuant
...", "La mecanica geometrica de TurboQuant"; "FibQuant ...", section 2.1),
and that a codec on the dense rotation keeps the estimator's properties."""
import math
from dataclasses import replace

import numpy as np
import pytest

from oracle import codebook as ocb
from oracle import codec as oc
from oracle.rotation import haar_rotation
from rotated_codebook_kv_tq_b200 import synth


@pytest.mark.parametrize("d", [16, 64, 128])
def test_haar_is_orthogonal_and_deterministic(d):
    P = haar_rotation(synth.haar_gaussian(d, 3))
    assert np.max(np.abs(P.T @ P - np.eye(d))) < 1e-13
    assert np.array_equal(P, haar_rotation(synth.haar_gaussian(d, 3)))
    # R has a positive diagonal: Q^T G is upper triangular with positive diagonal
    R = P.T @ synth.haar_gaussian(d, 3).astype(np.float64)
    assert np.all(np.diag(R) > 0) and np.max(np.abs(np.tril(R, -1))) < 1e-9


def test_haar_entry_moments_and_sign_fix():
    """Over many draws: E P_11 = 0, E P_11^2 = 1/d, E P_11^4 = 3/(d(d+2)) (a
    coordinate of a uniform unit vector).  Without the sign fix the first
    column is -G_1/|G_1| or G_1/|G_1| by the QR convention, so E P_11 != 0."""
    d, n = 8, 20000
    a = np.empty(n)
    raw = np.empty(n)
    rng = np.random.default_rng(11)
    for i in range(n):
        G = rng.standard_normal((d, d))
        a[i] = haar_rotation(G)[0, 0]
        raw[i] = np.linalg.qr(G)[0][0, 0]
    se = a.std() / math.sqrt(n)
    assert abs(a.mean()) < 4 * se
    assert abs(np.mean(a ** 2) * d - 1) < 0.03
    assert abs(np.mean(a ** 4) / (3 / (d * (d + 2))) - 1) < 0.06
    assert abs(raw.mean()) > 20 * se        # the unfixed factor is not Haar


def test_rotated_fixed_vector_follows_the_beta_law():
    """u = P x / |x| for one fixed x and many Haar P: each coordinate has the
    density f_d of the codebooks (KS distance against its CDF)."""
    d, n = 16, 6000
    x = np.arange(1, d + 1, dtype=np.float64) ** 2         # strongly anisotropic
    x /= np.linalg.norm(x)
    rng = np.random.default_rng(5)
    u = np.array([(haar_rotation(rng.standard_normal((d, d))) @ x)[3] for _ in range(n)])
    u.sort()
    # CDF of f_d by quadrature of the oracle's density
    grid = np.linspace(-1, 1, 20001)
    pdf = np.array([ocb.coord_pdf(t, d) for t in grid]).ravel()
    cdf_grid = np.concatenate([[0], np.cumsum((pdf[1:] + pdf[:-1]) / 2 * np.diff(grid))])
    F = np.interp(u, grid, cdf_grid)
    ks = np.max(np.abs(F - (np.arange(1, n + 1) - 0.5) / n))
    assert ks < 1.63 / math.sqrt(n) + 2e-3


def test_dense_codec_estimator_unbiased_and_mse():
    """A codec on a Haar rotation: E_S <y, x~> = <y, x>, and the value MSE of
    unit vectors equals d * mse_per_coord as for any uniform direction."""
    d = 64
    P = haar_rotation(synth.haar_gaussian(d, 9))
    base = oc.make_codec(d, 3, True, 3, synth.rotation_signs(d, 9), synth.qjl_matrix_bf16(d, 9), Pi=P)
    assert np.array_equal(base.Pi, P)
    rng = np.random.default_rng(2)
    x = rng.standard_normal(d)
    y = rng.standard_normal(d) + 0.5 * x
    n = 6000
    est = np.empty(n)
    for s in range(n):
        S = synth.bf16_bits_to_f32(synth.qjl_matrix_bf16(d, 2000 + s)).astype(np.float64)
        c = replace(base, S=S)
        e = oc.quantize_keys(x[None, :], c)
        est[s] = y @ oc.dequant_keys(e["idx"], e["sigma"], e["nu"], e["rho"], c)[0]
    assert abs(est.mean() - x @ y) < 4 * est.std() / math.sqrt(n)
    X = rng.standard_normal((20000, d))
    ev = oc.quantize_values(X, base)
    rel = np.sum((oc.dequant_values(ev["idx"], ev["nu"], base) - X) ** 2, axis=1) / np.sum(X * X, axis=1)
    assert abs(rel.mean() / (d * base.cb_v.mse_per_coord) - 1) < 0.02
