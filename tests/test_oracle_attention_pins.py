"""Brute-force pins for the parts of the oracle that the GPU parity tests lean
on most: grouped-query decode, the bidirectional pass and appends that cover a
32-token value group only partly.

Every expected value here comes from plain Python loops written from the
definitions, not from ``attention.estimator_logits`` or
``attention.softmax_average``:
* rotate-half RoPE ("TurboESM ...", section 2.A: RoPE is applied first, then
  the rotation) from the shared cos/sin table, one coordinate pair at a time;
* the logit of key j is scale * <RoPE(q), x~_j> with x~_j the dequantized key
  (the prod estimator's dequantized form, "Google presenta TurboQuant ...",
  "Eliminacion del sesgo interno del producto");
* softmax with max subtraction, output = sum_j p_j v~_j / sum_j p_j;
* query head h reads KV head h // (H / Hkv); the decode query of a sequence of
  length T sits at position T - 1; bidirectional query i sits at position i and
  attends to every key with no mask ("TurboESM ...", section 2.E).
"""
import math

import numpy as np
import pytest

from oracle import attention as att
from oracle import codec as oc
from rotated_codebook_kv_tq_b200 import synth


def _codec(d, bits_k, qjl, bits_v, seed):
    return oc.make_codec(d, bits_k, qjl, bits_v, synth.rotation_signs(d, seed),
                         synth.qjl_matrix_bf16(d, seed) if qjl else None)


def _rope_loop(x, cos, sin, pos):
    """Rotate-half RoPE of one vector at one position, pair (i, i + d/2)."""
    d = len(x)
    h = d // 2
    y = [0.0] * d
    for i in range(h):
        c, s = float(cos[pos, i]), float(sin[pos, i])
        y[i] = x[i] * c - x[i + h] * s
        y[i + h] = x[i + h] * c + x[i] * s
    return y


def _attend_loop(qv, keys, vals, scale):
    """Softmax attention of one query over dequantized rows, in plain loops."""
    T, d = len(keys), len(qv)
    lg = [scale * sum(qv[i] * keys[j][i] for i in range(d)) for j in range(T)]
    m = max(lg)
    w = [math.exp(l - m) for l in lg]
    tot = sum(w)
    return [sum(w[j] * vals[j][i] for j in range(T)) / tot for i in range(d)], lg


def _dequant_rows(cache, c, b, kvh, T):
    ik, sg, nk, rk, iv, nv = oc.cache_rows(cache, c, b, kvh, T)
    return oc.dequant_keys(ik, sg, nk, rk, c).tolist(), oc.dequant_values(iv, nv, c).tolist()


@pytest.mark.parametrize("qjl", [True, False])
def test_gqa_decode_brute_force(qjl):
    """B = 2 with different lengths, Hkv = 2, G = 4: every query head must read
    its own KV head, at its own batch's length, with the query at T_b - 1."""
    d, B, Hkv, G = 64, 2, 2, 4
    Hq = Hkv * G
    c = _codec(d, 3, qjl, 3, seed=21)
    rng = np.random.default_rng(22)
    rows_cap = 64
    lens = [41, 23]
    K = rng.standard_normal((B, Hkv, rows_cap, d)) * 2
    V = rng.standard_normal((B, Hkv, rows_cap, d))
    # make KV heads distinguishable: shift head 1's values
    V[:, 1] += 3.0
    q = rng.standard_normal((B, Hq, d))
    cos, sin = synth.rope_table(rows_cap, d, 1e4)
    cache = oc.empty_cache(c, B, Hkv, rows_cap)
    oc.quantize_into(cache, K, V, c, rope=(cos, sin))
    scale = 1 / math.sqrt(d)
    out, logits = att.decode(q, cache, c, lens, scale, rope=(cos, sin), want_logits=True)
    for b in range(B):
        T = lens[b]
        for h in range(Hq):
            keys, vals = _dequant_rows(cache, c, b, h // G, T)
            qv = _rope_loop(q[b, h].tolist(), cos, sin, T - 1)
            o, lg = _attend_loop(qv, keys, vals, scale)
            assert np.max(np.abs(np.array(lg) - logits[(b, h)])) < 1e-11 * max(1.0, max(map(abs, lg)))
            assert np.max(np.abs(np.array(o) - out[b, h])) < 1e-11


def test_bidirectional_brute_force():
    """Lq != T, query i RoPE'd at position i, no mask, Hkv = 2 < H = 4."""
    d, B, H, Hkv, T, Lq = 64, 1, 4, 2, 29, 11
    c = _codec(d, 3, True, 3, seed=23)
    rng = np.random.default_rng(24)
    K = rng.standard_normal((B, Hkv, 32, d)) * 2
    V = rng.standard_normal((B, Hkv, 32, d))
    V[:, 1] -= 2.0
    q = rng.standard_normal((B, H, Lq, d))
    cos, sin = synth.rope_table(32, d, 1e4)
    cache = oc.empty_cache(c, B, Hkv, 32)
    oc.quantize_into(cache, K[:, :, :T], V[:, :, :T], c, rope=(cos, sin))
    scale = 0.125
    out = att.bidirectional(q, cache, c, T, scale, rope=(cos, sin))
    for h in range(H):
        keys, vals = _dequant_rows(cache, c, 0, h // (H // Hkv), T)
        for i in range(Lq):
            qv = _rope_loop(q[0, h, i].tolist(), cos, sin, i)
            o, _ = _attend_loop(qv, keys, vals, scale)
            assert np.max(np.abs(np.array(o) - out[0, h, i])) < 1e-11


def test_bidirectional_equals_decode_at_last_position():
    """Query Lq - 1 of the bidirectional pass over T = Lq keys is the decode
    query of a length-T sequence (same position T - 1, same keys)."""
    d, T = 64, 20
    c = _codec(d, 3, True, 2, seed=25)
    rng = np.random.default_rng(26)
    K = rng.standard_normal((1, 1, T, d))
    V = rng.standard_normal((1, 1, T, d))
    q = rng.standard_normal((1, 2, T, d))
    cos, sin = synth.rope_table(32, d, 1e4)
    cache = oc.empty_cache(c, 1, 1, 32)
    oc.quantize_into(cache, K, V, c, rope=(cos, sin))
    bi = att.bidirectional(q, cache, c, T, 0.2, rope=(cos, sin))
    de = att.decode(q[:, :, T - 1], cache, c, [T], 0.2, rope=(cos, sin))
    assert np.max(np.abs(bi[0, :, T - 1] - de[0])) < 1e-12


@pytest.mark.parametrize("qjl", [True, False])
def test_appends_match_one_shot_encode(qjl):
    """Appending rows [0, 37), [37, 42), [42, 72) (partial 32-token value
    groups on both sides of each call) gives the same cache as one call over
    [0, 72): every plane, every byte."""
    d, B, Hkv, T = 64, 2, 2, 72
    c = _codec(d, 3, qjl, 3, seed=27)
    rng = np.random.default_rng(28)
    K = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d))
    cos, sin = synth.rope_table(96, d, 1e4)
    one = oc.empty_cache(c, B, Hkv, 96)
    oc.quantize_into(one, K, V, c, rope=(cos, sin))
    app = oc.empty_cache(c, B, Hkv, 96)
    for r0, r1 in [(0, 37), (37, 42), (42, 72)]:
        oc.quantize_into(app, K[:, :, r0:r1], V[:, :, r0:r1], c, rope=(cos, sin), pos0=r0, row0=r0)
    for key in ("kcode", "kscale", "vcode", "vnorm"):
        assert np.array_equal(one[key], app[key]), key
    # and the value planes hold each row's codes at bit (row % 32) of group row // 32
    enc = oc.quantize_values(V[1, 0], c)
    for r in (0, 31, 32, 37, 41, 42, 63, 64, 71):
        g, t = divmod(r, 32)
        for i in (0, 5, 63):
            code = sum((((int(one["vcode"][1, 0, g, p, i]) >> t) & 1) << p) for p in range(c.bits_v))
            assert code == enc["idx"][r, i]
    # rows beyond the last append stay zero
    assert not np.any(one["vcode"][:, :, 2] >> np.uint32(8))


def test_append_preserves_other_rows_of_group():
    """A later append into the middle of a 32-token group must not touch the
    rows of that group written by earlier calls, nor rows after it."""
    d = 64
    c = _codec(d, 2, True, 2, seed=29)
    rng = np.random.default_rng(30)
    K = rng.standard_normal((1, 1, 64, d))
    V = rng.standard_normal((1, 1, 64, d))
    cache = oc.empty_cache(c, 1, 1, 64)
    oc.quantize_into(cache, K[:, :, :10], V[:, :, :10], c)
    oc.quantize_into(cache, K[:, :, 20:30], V[:, :, 20:30], c, pos0=20, row0=20)
    before = cache["vcode"].copy()
    oc.quantize_into(cache, K[:, :, 10:20], V[:, :, 10:20], c, pos0=10, row0=10)
    mask = np.uint32(((1 << 10) - 1) << 10)       # bits 10..19 may change
    assert np.array_equal(cache["vcode"] & ~mask, before & ~mask)
    enc = oc.quantize_values(V[0, 0, :30], c)
    iv, _ = oc.unpack_values(cache["vcode"][0, 0, :1], cache["vnorm"][0, 0, :32], c)
    assert np.array_equal(iv[:30], enc["idx"])
