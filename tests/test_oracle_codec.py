"""Pins for oracle.rotation, oracle.codec and oracle.attention.

Independent facts used: library Hadamard matrices (scipy), orthogonality,
RoPE invariance (TurboESM, section 2.A), the exact finite-d 2/pi bias law of
the 1-bit MSE quantizer (TurboQuant page, "Eliminacion del sesgo"), Monte-Carlo
unbiasedness and variance of the QJL estimator (same page's unbiasedness
equation), hand-worked bit layout, and brute-force softmax attention."""
import json
import math
import os
from dataclasses import replace

import numpy as np
import pytest
from scipy.linalg import hadamard as scipy_hadamard

from oracle import attention as att
from oracle import codebook as cb
from oracle import codec as oc
from oracle import rotation as rot
from rotated_codebook_kv_tq_b200 import synth


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("d", [64, 128])
def test_sylvester_matches_library(d):
    assert np.array_equal(rot.hadamard(d), scipy_hadamard(d).astype(np.float64))


@pytest.mark.parametrize("d", [64, 128, 1536])
def test_rotation_orthogonal_and_norm_preserving(d):
    D = synth.rotation_signs(d, 7)
    Pi = rot.rotation_matrix(D)
    assert np.max(np.abs(Pi @ Pi.T - np.eye(d))) < 1e-12
    x = np.random.default_rng(1).standard_normal((5, d))
    assert np.allclose(np.linalg.norm(x @ Pi.T, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    if d == 1536:
        h12 = rot.paley_hadamard(11)
        assert np.array_equal(h12 @ h12.T, 12 * np.eye(12))
        assert set(np.unique(rot.hadamard(d))) == {-1.0, 1.0}


def test_rope_then_rotate_invariance():
    """(Pi R_i q)^T (Pi R_j k) = q^T R_i^T R_j k and depends only on i - j."""
    d, theta = 128, 5e5
    cos, sin = synth.rope_table(4096, d, theta)
    g = np.random.default_rng(2)
    q, k = g.standard_normal(d), g.standard_normal(d)
    Pi = rot.rotation_matrix(synth.rotation_signs(d, 3))
    def dot(i, j):
        qi = rot.apply_rope(q, cos, sin, i)
        kj = rot.apply_rope(k, cos, sin, j)
        return (Pi @ qi) @ (Pi @ kj), qi @ kj
    a, b = dot(100, 40)
    assert abs(a - b) < 1e-11
    c, _ = dot(1060, 1000)
    assert abs(a - c) < 1e-4          # fp32 table rounding only
    assert abs(np.linalg.norm(rot.apply_rope(q, cos, sin, 77)) - np.linalg.norm(q)) < 1e-5


# ---------------------------------------------------------------- 2/pi bias

def _haar_pairs(n, d, rho, g):
    """(Pi x, Pi y) for unit x, y with <x, y> = rho and Pi Haar: the first two
    columns of a Haar matrix are a uniform orthonormal pair."""
    a = g.standard_normal((n, d))
    b = g.standard_normal((n, d))
    u = a / np.linalg.norm(a, axis=1, keepdims=True)
    b = b - np.sum(b * u, axis=1, keepdims=True) * u
    w = b / np.linalg.norm(b, axis=1, keepdims=True)
    return u, rho * u + math.sqrt(1 - rho * rho) * w


@pytest.mark.parametrize("d,factor", [(64, 0.6416), (128, 0.6391)])
def test_two_over_pi_bias_haar(d, factor, golden_dir):
    """E<y, x^_{b=1}> = d c1^2 <y, x>, tending to 2/pi (TurboQuant page)."""
    g = json.load(open(os.path.join(golden_dir, "turboquant_page_constants.json")))
    rng = np.random.default_rng(11)
    rho, n = 0.6, 100_000
    u, yr = _haar_pairs(n, d, rho, rng)
    book = cb.codebook(d, 1)
    idx = oc.scalar_codes(u, book.thresholds32)
    xhat = book.centroids32.astype(np.float64)[idx]
    est = np.sum(yr * xhat, axis=1) / rho
    se = est.std() / math.sqrt(n)
    exact = d * book.centroids[1] ** 2
    assert abs(exact - factor) < 1e-4
    assert abs(est.mean() - exact) < 4 * se
    assert exact > g["bias_limit_2_over_pi"] and exact - g["bias_limit_2_over_pi"] < 0.01


def test_two_over_pi_bias_randomized_wht():
    """Gaussian x makes Pi x / |x| exactly uniform on the sphere for the oracle's
    randomized Hadamard Pi, so the exact factor d c1^2 must appear; for one fixed
    x over random sign vectors D the factor is only close to it."""
    d, n = 64, 60_000
    rng = np.random.default_rng(12)
    Pi = rot.rotation_matrix(synth.rotation_signs(d, 21))
    book = cb.codebook(d, 1)
    x = rng.standard_normal((n, d))
    y = 0.6 * x + rng.standard_normal((n, d))
    nu, u = oc.normalize_rotate(x, Pi)
    xhat = book.centroids32.astype(np.float64)[oc.scalar_codes(u, book.thresholds32)]
    xt = nu[:, None] * (xhat @ Pi)
    est = np.sum(y * xt, axis=1) - 0.0
    ref = np.sum(y * x, axis=1)
    # E<y, x~> = d c1^2 E<y, x> (both averaged over the same draws)
    ratio = est.mean() / ref.mean()
    se = (est - d * book.centroids[1] ** 2 * ref).std() / math.sqrt(n) / ref.mean()
    assert abs(ratio - d * book.centroids[1] ** 2) < 4 * se
    # fixed x, random D: Rademacher sums are close to, not exactly, spherical
    H = rot.hadamard(d)
    x0 = rng.standard_normal(d)
    Ds = np.where(rng.integers(0, 2, size=(20000, d)) == 1, 1.0, -1.0)
    nu0, u0 = oc.normalize_rotate((Ds * x0) @ H.T / math.sqrt(d), np.eye(d))
    xh0 = book.centroids32.astype(np.float64)[oc.scalar_codes(u0, book.thresholds32)]
    f0 = np.mean(nu0 * np.sum(u0 * xh0, axis=1)) / np.linalg.norm(x0)
    assert abs(f0 - d * book.centroids[1] ** 2) < 0.01


# ---------------------------------------------------------------- QJL estimator

def _codec(d, bits_k, qjl, bits_v, seed):
    return oc.make_codec(d, bits_k, qjl, bits_v, synth.rotation_signs(d, seed),
                         synth.qjl_matrix_bf16(d, seed) if qjl else None)


@pytest.mark.parametrize("bits_k", [2, 3])
def test_qjl_estimator_unbiased_and_variance(bits_k):
    """E_S <y, x~> = <y, x> (TurboQuant page, unbiasedness equation), and
    Var = (pi/2) rho^2 nu^2 / m (|Pi y|^2 - (2/pi) <r/rho, Pi y>^2)."""
    d, n = 64, 20_000
    base = _codec(d, bits_k, True, 2, seed=5)
    rng = np.random.default_rng(13)
    x = rng.standard_normal(d) * 2.0
    y = rng.standard_normal(d) + 0.5 * x
    est = np.empty(n)
    enc0 = None
    for s in range(n):
        S = synth.bf16_bits_to_f32(synth.qjl_matrix_bf16(d, 1000 + s)).astype(np.float64)
        c = replace(base, S=S)
        enc = oc.quantize_keys(x[None, :], c)
        xt = oc.dequant_keys(enc["idx"], enc["sigma"], enc["nu"], enc["rho"], c)[0]
        est[s] = y @ xt
        enc0 = enc
    se = est.std() / math.sqrt(n)
    assert abs(est.mean() - x @ y) < 4 * se
    r = enc0["r"][0]
    rho, nu = enc0["rho"][0], enc0["nu"][0]
    yp = base.Pi @ y
    var = (math.pi / 2) * rho ** 2 * nu ** 2 / d * (yp @ yp - (2 / math.pi) * (r / rho @ yp) ** 2)
    assert abs(est.var() / var - 1) < 0.05


def test_mse_only_inner_product_is_biased_at_one_bit():
    """Without the QJL stage the 1-bit estimator shrinks <y,x> (contrast to the
    unbiased prod estimator above)."""
    d = 128
    c = _codec(d, 1, False, 1, seed=6)
    rng = np.random.default_rng(14)
    x = rng.standard_normal((4000, d))
    enc = oc.quantize_keys(x, c)
    xt = oc.dequant_keys(enc["idx"], None, enc["nu"], enc["rho"], c)
    ratio = np.sum(xt * x, axis=1) / np.sum(x * x, axis=1)
    assert 0.60 < ratio.mean() < 0.68


# ---------------------------------------------------------------- layout

def test_key_layout_hand_worked(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "layout_example.json")))
    d = g["d"]
    c = _codec(d, 3, True, 2, seed=1)
    idx = np.zeros((1, d), np.int64)
    for k, v in g["idx_nonzero"].items():
        idx[0, int(k)] = v
    sigma = np.zeros((1, d), bool)
    sigma[0, g["sigma_set"]] = True
    enc = dict(idx=idx, sigma=sigma, nu16=np.float16([1.5]), rho16=np.float16([0.25]))
    kcode, kscale = oc.pack_keys(enc, c)
    assert [kcode[0, p].tobytes().hex() for p in range(3)] == g["expected_kcode_hex"]
    i2, s2, n2, r2 = oc.unpack_keys(kcode, kscale, c)
    assert np.array_equal(i2, idx) and np.array_equal(s2, sigma) and n2[0] == 1.5 and r2[0] == 0.25
    ex = g["value_word_example"]
    vidx = np.zeros((ex["rows"], d), np.int64)
    vidx[ex["row_with_code_3_at_coord_5"], 5] = 3
    vcode, _ = oc.pack_values(dict(idx=vidx, nu16=np.zeros(32, np.float16)), c)
    assert vcode[0, 0, 5] == ex["expected_word_plane0_coord5"]
    assert vcode[0, 1, 5] == ex["expected_word_plane1_coord5"]
    assert np.count_nonzero(vcode) == 2


def test_layout_roundtrip_and_bytes_per_row():
    c = _codec(128, 4, True, 4, seed=2)
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 8, (64, 128))
    sig = rng.integers(0, 2, (64, 128)).astype(bool)
    kc, ks = oc.pack_keys(dict(idx=idx, sigma=sig, nu16=np.ones(64, np.float16),
                               rho16=np.ones(64, np.float16)), c)
    i2, s2, _, _ = oc.unpack_keys(kc, ks, c)
    assert np.array_equal(i2, idx) and np.array_equal(s2, sig)
    vidx = rng.integers(0, 16, (64, 128))
    vc, vn = oc.pack_values(dict(idx=vidx, nu16=np.ones(64, np.float16)), c)
    assert np.array_equal(oc.unpack_values(vc, vn, c)[0], vidx)
    assert oc.bytes_per_row(c) == (68, 66)                      # 134 B per token-head
    assert oc.bytes_per_row(_codec(128, 2, True, 2, 1)) == (36, 34)
    assert oc.bytes_per_row(_codec(64, 3, True, 3, 1)) == (28, 26)


def test_zero_and_nonfinite_rows():
    c = _codec(128, 3, True, 3, seed=4)
    x = np.random.default_rng(5).standard_normal((4, 128))
    x[1] = 0.0
    x[2, 7] = np.nan
    x[3, 0] = 1e6      # norm overflows fp16
    ek = oc.quantize_keys(x, c)
    assert list(ek["bad"]) == [False, False, True, True]
    for r in (1, 2, 3):
        assert ek["nu16"][r] == 0
        # zero vector: u = 0 sits on the middle threshold (exactly 0) -> upper cell
        assert np.all(ek["idx"][r] == (1 << (c.mse_bits_k - 1)))
    xt = oc.dequant_keys(ek["idx"], ek["sigma"], ek["nu16"].astype(float), ek["rho16"].astype(float), c)
    assert np.all(xt[1:] == 0)


def test_quantization_error_in_expected_range():
    """Reconstruction MSE of unit vectors matches d * mse_per_coord (values)."""
    d = 128
    c = _codec(d, 2, True, 3, seed=8)
    x = np.random.default_rng(9).standard_normal((20000, d))
    ev = oc.quantize_values(x, c)
    vt = oc.dequant_values(ev["idx"], ev["nu"], c)
    rel = np.sum((vt - x) ** 2, axis=1) / np.sum(x * x, axis=1)
    expect = d * c.cb_v.mse_per_coord
    assert abs(rel.mean() / expect - 1) < 0.02


# ---------------------------------------------------------------- attention

def test_estimator_equals_dequant_form_and_brute_force_softmax():
    d, T, G = 64, 37, 2
    c = _codec(d, 3, True, 3, seed=10)
    rng = np.random.default_rng(15)
    K = rng.standard_normal((1, 1, T, d)) * 3
    V = rng.standard_normal((1, 1, T, d))
    q = rng.standard_normal((1, G, d))
    cos, sin = synth.rope_table(64, d, 1e4)
    cache = oc.empty_cache(c, 1, 1, 64)
    oc.quantize_into(cache, K, V, c, rope=(cos, sin))
    scale = 1 / math.sqrt(d)
    out, logits = att.decode(q, cache, c, [T], scale, rope=(cos, sin), want_logits=True)
    rows = oc.cache_rows(cache, c, 0, 0, T)
    keys = oc.dequant_keys(*rows[:4], c)
    vals = oc.dequant_values(rows[4], rows[5], c)
    for h in range(G):
        qr = rot.apply_rope(q[0, h], cos, sin, T - 1)
        lg2 = att.dequant_logits(qr[None], rows, c, scale)[0]
        assert np.max(np.abs(lg2 - logits[(0, h)])) < 1e-12 * np.max(np.abs(lg2))
        # brute force: plain loops over keys and coordinates
        lg = [scale * sum(qr[i] * keys[j, i] for i in range(d)) for j in range(T)]
        m = max(lg)
        w = [math.exp(l - m) for l in lg]
        o = [sum(w[j] * vals[j, i] for j in range(T)) / sum(w) for i in range(d)]
        assert np.max(np.abs(np.array(o) - out[0, h])) < 1e-12


def test_attention_degenerate_cases():
    d, T = 128, 64
    c = _codec(d, 2, True, 2, seed=12)
    rng = np.random.default_rng(16)
    K = np.repeat(rng.standard_normal((1, 1, 1, d)), T, axis=2)
    V = rng.standard_normal((1, 1, T, d))
    cache = oc.empty_cache(c, 1, 1, T)
    oc.quantize_into(cache, K, V, c)
    q = rng.standard_normal((1, 4, d))
    out = att.decode(q, cache, c, [T], 0.1)
    vals = oc.dequant_values(*oc.cache_rows(cache, c, 0, 0, T)[4:], c)
    # identical keys -> uniform weights -> mean of the dequantized values
    assert np.max(np.abs(out[0] - vals.mean(axis=0))) < 1e-12
    # single key -> its value
    out1 = att.decode(q, cache, c, [1], 0.1)
    assert np.max(np.abs(out1[0] - vals[0])) < 1e-12


# ---------------------------------------------------------------- vector search (d = 1536)

def test_scan_scores_equal_dequantized_inner_products_d1536():
    """Scores of the oracle scan equal <q, x~_j> with x~ the dequantized rows
    (identity of the estimator form), and top-k matches a brute-force sort."""
    from oracle import scan
    d = 1536
    c = oc.make_codec(d, 4, True, 4, synth.rotation_signs(d, 4), synth.qjl_matrix_bf16(d, 4))
    x = synth.unit_rows(40, d, 4, 0).astype(np.float64)
    q = synth.unit_rows(3, d, 4, 2).astype(np.float64)
    enc = oc.quantize_keys(x, c)
    kcode, kscale = oc.pack_keys(enc, c)
    s = scan.scores(q, kcode, kscale, c)
    ik, sg, nk, rk = oc.unpack_keys(kcode, kscale, c)
    xt = oc.dequant_keys(ik, sg, nk, rk, c)
    assert np.max(np.abs(s - q @ xt.T)) < 1e-12
    idx, val = scan.topk(s, 5)
    for i in range(3):
        brute = sorted(range(40), key=lambda j: (-s[i, j], j))[:5]
        assert list(idx[i]) == brute
    # the estimator tracks the true inner products (unit rows, 3+1 bits)
    assert np.corrcoef(s.ravel(), (q @ x.T).ravel())[0, 1] > 0.9
