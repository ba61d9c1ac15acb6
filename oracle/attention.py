"""Attention over the compressed cache (oracle side).

Sources:
* "TurboESM ..." (gist.science 2603.26110), section 2.E "Kernel Fuso Triton":
  attention is computed in one pass straight from the compressed cache
  (unpack, residual correction, inverse rotation Pi^T, attention with online
  softmax), with no intermediate dequantized buffer; section 2.A: RoPE is
  applied before the rotation and Pi^T Pi = I keeps q.k unchanged.
* "Google presenta TurboQuant..." (7minutos.es), "Eliminacion del sesgo interno
  del producto": the prod estimator of <y, x> is unbiased.

The logit of key j for a query q (after RoPE) is computed in the estimator form
    l_j = s * nu_j * ( <Pi q, c[idx_j]> + sqrt(pi/2)/m * rho_j * <S Pi q, 2 sigma_j - 1> ),
which equals s * <q, x~_j> with x~_j the dequantized key; ``dequant_logits``
computes that second form so tests can check the identity.  Softmax uses max
subtraction in fp64; the output is sum_j p_j v~_j / sum_j p_j.  Readings: the
decode query of a sequence of length T sits at position T-1; query head h reads
KV head floor(h / G); the bidirectional pass gives query i position i and
attends to every key with no mask.
"""
from __future__ import annotations

import numpy as np

from .codec import Codec, cache_rows, dequant_keys, dequant_values
from .rotation import apply_rope


def estimator_logits(qr: np.ndarray, rows, codec: Codec, scale: float) -> np.ndarray:
    """qr: [n_q, d] queries after RoPE.  rows: unpacked cache rows."""
    ik, sg, nk, rk, _, _ = rows
    q1 = qr @ codec.Pi.T                                         # Pi q
    ck = codec.cb_k.centroids32.astype(np.float64)[ik]           # [T, d]
    mse = q1 @ ck.T                                              # [n_q, T]
    if codec.qjl_k:
        q2 = q1 @ codec.S.T                                      # S Pi q
        qj = q2 @ (2.0 * sg - 1.0).T
        mse = mse + codec.qjl_coef * rk[None, :] * qj
    return scale * nk[None, :] * mse


def dequant_logits(qr: np.ndarray, rows, codec: Codec, scale: float) -> np.ndarray:
    ik, sg, nk, rk, _, _ = rows
    return scale * (qr @ dequant_keys(ik, sg, nk, rk, codec).T)


def softmax_average(logits: np.ndarray, vals: np.ndarray) -> np.ndarray:
    m = np.max(logits, axis=-1, keepdims=True)
    p = np.exp(logits - m)
    return (p @ vals) / np.sum(p, axis=-1, keepdims=True)


def decode(q: np.ndarray, cache: dict, codec: Codec, seq_lens, scale: float,
           rope=None, heads=None, want_logits: bool = False):
    """One decode step.  q: [B, Hq, d] (pre-RoPE).  Returns out [B, Hq, d]
    (rows not in ``heads`` are NaN) and optionally the logits per (b, h)."""
    B, Hq, d = q.shape
    Hkv = cache["kcode"].shape[1]
    G = Hq // Hkv
    out = np.full((B, Hq, d), np.nan)
    logits = {}
    heads = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else heads
    by_kv = {}
    for b, h in heads:
        by_kv.setdefault((b, h // G), []).append(h)
    for (b, kvh), hs in by_kv.items():
        T = int(seq_lens[b])
        rows = cache_rows(cache, codec, b, kvh, T)
        vals = dequant_values(rows[4], rows[5], codec)
        qb = np.asarray(q[b, hs], np.float64)
        if rope is not None:
            qb = apply_rope(qb, rope[0], rope[1], np.full(len(hs), T - 1))
        lg = estimator_logits(qb, rows, codec, scale)
        o = softmax_average(lg, vals)
        for i, h in enumerate(hs):
            out[b, h] = o[i]
            if want_logits:
                logits[(b, h)] = lg[i]
    return (out, logits) if want_logits else out


def bidirectional(q: np.ndarray, cache: dict, codec: Codec, T: int, scale: float,
                  rope=None, heads=None) -> np.ndarray:
    """Full bidirectional pass: q [B, H, Lq, d], query i at position i, every
    query attends to keys 0..T-1 with no mask.  Returns [B, H, Lq, d]."""
    B, H, Lq, d = q.shape
    Hkv = cache["kcode"].shape[1]
    G = H // Hkv
    out = np.full((B, H, Lq, d), np.nan)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in heads:
        rows = cache_rows(cache, codec, b, h // G, T)
        vals = dequant_values(rows[4], rows[5], codec)
        qb = np.asarray(q[b, h], np.float64)
        if rope is not None:
            qb = apply_rope(qb, rope[0], rope[1], np.arange(Lq))
        out[b, h] = softmax_average(estimator_logits(qb, rows, codec, scale), vals)
    return out
