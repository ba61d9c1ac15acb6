"""Pins for the oracle's outlier-channel split (``oracle/split.py``).

Expected values come from plain loops written from the definitions, from the
already pinned single-codec oracle (``oracle/codec.py``), from invariants and
from Monte-Carlo laws -- never from ``split.decode`` itself:
* rotate-half RoPE over the whole head vector ("TurboESM ...", section 2.A),
  then each channel set coded by its own codec;
* logit = scale * sum over all channels of q_c * k~_c with each key half
  dequantized by its codec and put back at its channels; softmax and the
  value average in plain loops;
* the split estimator is unbiased over the two QJL sketches ("Google presenta
  TurboQuant ...", "Eliminacion del sesgo interno del producto"), with each
  codec's own constant sqrt(pi/2)/m, m = d/2;
* rates 2.5 = (3 + 2) / 2 and 3.5 = (4 + 3) / 2 bits per channel ("Google
  presenta TurboQuant ...", "Desempeno teorico y empirico").
"""
import math
from dataclasses import replace

import numpy as np
import pytest

from oracle import codec as oc
from oracle import split as osp
from rotated_codebook_kv_tq_b200 import synth


def _codec(d, bits_k, qjl, bits_v, seed):
    return oc.make_codec(d, bits_k, qjl, bits_v, synth.rotation_signs(d, seed),
                         synth.qjl_matrix_bf16(d, seed) if qjl else None)


def _rope_loop(x, cos, sin, pos):
    d = len(x)
    h = d // 2
    y = [0.0] * d
    for i in range(h):
        c, s = float(cos[pos, i]), float(sin[pos, i])
        y[i] = x[i] * c - x[i + h] * s
        y[i + h] = x[i + h] * c + x[i] * s
    return y


def _random_channels(rng, Hkv, d):
    return np.stack([np.stack([rng.permutation(d), rng.permutation(d)]) for _ in range(Hkv)])


def test_outlier_channels_hand_worked():
    got = osp.outlier_channels(np.array([3, 1, 4, 1, 5, 9, 2, 6], float))
    # top four scores 9 (ch 5), 6 (ch 7), 5 (ch 4), 4 (ch 2), ascending
    assert got.tolist() == [2, 4, 5, 7, 0, 1, 3, 6]
    # ties go to the lower channel
    assert osp.outlier_channels(np.ones(4)).tolist() == [0, 1, 2, 3]
    assert osp.outlier_channels(np.array([0, 2, 2, 2], float)).tolist() == [1, 2, 0, 3]


@pytest.mark.parametrize("bits", [((3, 3), (2, 2)), ((4, 4), (3, 3))])
def test_rates_are_the_pages_examples(bits):
    (bk_hi, bv_hi), (bk_lo, bv_lo) = bits
    sc = osp.make_split_codec(_codec(64, bk_hi, True, bv_hi, 1), _codec(64, bk_lo, True, bv_lo, 2),
                              _random_channels(np.random.default_rng(0), 1, 128))
    rk, rv = osp.rate_bits(sc)
    assert rk == rv == (bk_hi + bk_lo) / 2 and rk in (2.5, 3.5)
    kb, vb = osp.bytes_per_row(sc)
    # code bits of both halves plus one (nu, rho) pair and one nu per half
    assert kb == (bk_hi + bk_lo) * 64 // 8 + 8
    assert vb == (bv_hi + bv_lo) * 64 // 8 + 4


def test_make_split_codec_rejects_bad_maps():
    hi, lo = _codec(8, 3, True, 3, 1), _codec(8, 2, True, 2, 2)
    ok = _random_channels(np.random.default_rng(1), 2, 16)
    osp.make_split_codec(hi, lo, ok)
    bad = ok.copy()
    bad[1, 0, 3] = bad[1, 0, 4]
    with pytest.raises(ValueError):
        osp.make_split_codec(hi, lo, bad)
    with pytest.raises(ValueError):
        osp.make_split_codec(hi, _codec(16, 2, True, 2, 2), ok)


def _tiny_split(seed=3, d=16, Hkv=2):
    rng = np.random.default_rng(seed)
    hi = _codec(d // 2, 3, True, 3, 11)     # 2 MSE bits + QJL
    lo = _codec(d // 2, 2, True, 2, 12)     # 1 MSE bit + QJL
    return osp.make_split_codec(hi, lo, _random_channels(rng, Hkv, d)), rng


def test_quantize_gathers_after_full_rope():
    """Each half cache equals the single-codec encoding of the channels picked
    from the RoPE'd (over all d channels) key, built here by loops."""
    d, Hkv, T, pos0 = 16, 2, 40, 7
    sc, rng = _tiny_split(d=d, Hkv=Hkv)
    K = rng.standard_normal((1, Hkv, T, d)) * np.linspace(0.5, 3.0, d)
    V = rng.standard_normal((1, Hkv, T, d))
    cos, sin = synth.rope_table(64, d, 100.0)
    caches = osp.empty_caches(sc, 1, Hkv, 64)
    osp.quantize_into(caches, K, V, sc, rope=(cos, sin), pos0=pos0)
    for h in range(Hkv):
        kr = [_rope_loop(list(K[0, h, t]), cos, sin, pos0 + t) for t in range(T)]
        for part, codec in ((0, sc.hi), (1, sc.lo)):
            ck = sc.channels[h, 0][part * d // 2:(part + 1) * d // 2]
            cv = sc.channels[h, 1][part * d // 2:(part + 1) * d // 2]
            ks = np.array([[kr[t][c] for c in ck] for t in range(T)])[None, None]
            vs = np.array([[V[0, h, t, c] for c in cv] for t in range(T)])[None, None]
            ref = oc.empty_cache(codec, 1, 1, 64)
            oc.quantize_into(ref, ks, vs, codec)
            for key in ("kcode", "kscale", "vcode", "vnorm"):
                np.testing.assert_array_equal(caches[part][key][:, h], ref[key][:, 0], err_msg=key)


def test_decode_matches_brute_force_loops():
    """GQA (Hq = 4, Hkv = 2), RoPE at position T - 1, two lengths."""
    d, Hkv, Hq, T = 16, 2, 4, 45
    sc, rng = _tiny_split(d=d, Hkv=Hkv)
    K = rng.standard_normal((2, Hkv, T, d)) * np.linspace(3.0, 0.5, d)
    V = rng.standard_normal((2, Hkv, T, d))
    q = rng.standard_normal((2, Hq, d))
    cos, sin = synth.rope_table(64, d, 100.0)
    caches = osp.empty_caches(sc, 2, Hkv, 64)
    osp.quantize_into(caches, K, V, sc, rope=(cos, sin))
    seq = [T, 33]
    scale = 0.3
    out, lg = osp.decode(q, caches, sc, seq, scale, rope=(cos, sin), want_logits=True)
    for b in range(2):
        n = seq[b]
        for h in range(Hq):
            kvh = h // (Hq // Hkv)
            keys = [[0.0] * d for _ in range(n)]
            vals = [[0.0] * d for _ in range(n)]
            for part, codec in ((0, sc.hi), (1, sc.lo)):
                ik, sg, nk, rk, iv, nv = oc.cache_rows(caches[part], codec, b, kvh, n)
                kt = oc.dequant_keys(ik, sg, nk, rk, codec)
                vt = oc.dequant_values(iv, nv, codec)
                for j in range(d // 2):
                    ckj = sc.channels[kvh, 0][part * d // 2 + j]
                    cvj = sc.channels[kvh, 1][part * d // 2 + j]
                    for t in range(n):
                        keys[t][ckj] = kt[t, j]
                        vals[t][cvj] = vt[t, j]
            qr = _rope_loop(list(q[b, h]), cos, sin, n - 1)
            logit = [scale * sum(qr[c] * keys[t][c] for c in range(d)) for t in range(n)]
            m = max(logit)
            w = [math.exp(x - m) for x in logit]
            expect = [sum(w[t] * vals[t][c] for t in range(n)) / sum(w) for c in range(d)]
            np.testing.assert_allclose(lg[(b, h)], logit, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(out[b, h], expect, rtol=1e-11, atol=1e-12)


def test_channel_relabelling_invariance():
    """Relabelling the channels of q, K, V and of the maps together (no RoPE)
    leaves every code unchanged and relabels the output the same way."""
    d, Hkv, T = 16, 2, 32
    sc, rng = _tiny_split(d=d, Hkv=Hkv)
    K = rng.standard_normal((1, Hkv, T, d))
    V = rng.standard_normal((1, Hkv, T, d))
    q = rng.standard_normal((1, 2 * Hkv, d))
    perm = rng.permutation(d)
    inv = np.argsort(perm)
    sc2 = osp.make_split_codec(sc.hi, sc.lo, inv[sc.channels])
    c1, c2 = osp.empty_caches(sc, 1, Hkv, 32), osp.empty_caches(sc2, 1, Hkv, 32)
    osp.quantize_into(c1, K, V, sc)
    osp.quantize_into(c2, K[..., perm], V[..., perm], sc2)
    for part in range(2):
        for key in ("kcode", "kscale", "vcode", "vnorm"):
            np.testing.assert_array_equal(c1[part][key], c2[part][key])
    o1 = osp.decode(q, c1, sc, [T], 0.5)
    o2 = osp.decode(q[..., perm], c2, sc2, [T], 0.5)
    np.testing.assert_array_equal(o2, o1[..., perm])


def test_split_estimator_unbiased_over_both_sketches():
    """E over S_hi, S_lo of the split logit = scale <q, k>; a constant built
    from the full d (m = 16 instead of 8) would shrink both QJL terms."""
    d, n = 16, 3000
    sc0, rng = _tiny_split(d=d, Hkv=1)
    k = rng.standard_normal((1, 1, 1, d)) * np.linspace(0.5, 2.0, d)
    v = rng.standard_normal((1, 1, 1, d))
    q = k[0, :, 0] + 0.7 * rng.standard_normal((1, 1, d))
    est = np.empty(n)
    for s in range(n):
        S_hi = synth.bf16_bits_to_f32(synth.qjl_matrix_bf16(d // 2, 5000 + s)).astype(np.float64)
        S_lo = synth.bf16_bits_to_f32(synth.qjl_matrix_bf16(d // 2, 9000 + s)).astype(np.float64)
        sc = replace(sc0, hi=replace(sc0.hi, S=S_hi), lo=replace(sc0.lo, S=S_lo))
        caches = osp.empty_caches(sc, 1, 1, 32)
        osp.quantize_into(caches, k, v, sc)
        _, lg = osp.decode(q, caches, sc, [1], 1.0, want_logits=True)
        est[s] = lg[(0, 0)][0]
    truth = float(q[0, 0] @ k[0, 0, 0])
    se = est.std() / math.sqrt(n)
    assert abs(est.mean() - truth) < 4 * se
    # the QJL terms carry enough here that halving them (a constant built from
    # the full d) would move the mean by more than 6 standard errors
    mse_only = 0.0
    for part, codec in ((0, sc0.hi), (1, sc0.lo)):
        ck = sc0.channels[0, 0][part * d // 2:(part + 1) * d // 2]
        e = oc.quantize_keys(k[0, 0, 0][ck][None, :], codec)
        c = codec.cb_k.centroids32.astype(np.float64)[e["idx"][0]]
        mse_only += e["nu"][0] * float((codec.Pi @ q[0, 0][ck]) @ c)
    assert abs(truth - mse_only) / 2 > 6 * se


def test_half_distortion_follows_each_codebook():
    """Value halves: E||x_half - x~_half||^2 / ||x_half||^2 = (d/2) mse_per_coord
    of that half's codebook (dimension d/2, its own bit width)."""
    d, n = 64, 8000
    rng = np.random.default_rng(21)
    hi, lo = _codec(d // 2, 3, True, 3, 31), _codec(d // 2, 2, True, 2, 32)
    sc = osp.make_split_codec(hi, lo, _random_channels(rng, 1, d))
    # isotropic rows, so each half's direction is uniform on its sphere
    V = rng.standard_normal((1, 1, n, d))
    K = rng.standard_normal((1, 1, n, d))
    caches = osp.empty_caches(sc, 1, 1, n)
    osp.quantize_into(caches, K, V, sc)
    vt = osp.dequantize(caches, sc, 1, 0, 0, n)
    for part, codec in ((0, hi), (1, lo)):
        ch = sc.channels[0, 1][part * d // 2:(part + 1) * d // 2]
        x, y = V[0, 0][:, ch], vt[:, ch]
        rel = np.sum((y - x) ** 2, axis=1) / np.sum(x * x, axis=1)
        assert abs(rel.mean() / (d // 2 * codec.cb_v.mse_per_coord) - 1) < 0.03
