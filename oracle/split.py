"""Outlier-channel mixed precision: two codecs over two channel sets (oracle side).

Source: "Google presenta TurboQuant ..." (7minutos.es), "Desempeno teorico y
empirico": for bit widths that are not integers, specific outlier channels get
more bits (e.g. 3) and the other channels fewer (e.g. 2), for effective rates
such as 2.5 or 3.5 bits per channel.

Readings (the page gives only the rates and the two bit widths):
* The outlier channels are channels of the head vector as the model produces
  it, before the rotation: a rotation spreads every channel over all
  coordinates, so a per-channel bit map means something only before it.
* Each channel set is coded by its own TurboQuant codec (own norm, own
  randomized Walsh-Hadamard rotation, own Beta codebook, own QJL sketch for
  keys), so the sets never mix.  The page's two examples, 2.5 = (3 + 2) / 2 and
  3.5 = (4 + 3) / 2, are what equal halves give: each set holds d/2 channels,
  which also keeps each rotation a power-of-two transform.
* Which channels are the outliers is the caller's input, per KV head and
  separately for keys and values: ``channels[h][0]`` (keys) and
  ``channels[h][1]`` (values) are permutations of 0..d-1 whose first d/2
  entries are the outlier channels (coded by ``hi``) and whose last d/2 are
  the rest (coded by ``lo``).  ``outlier_channels`` gives one such choice: the
  d/2 channels with the largest score (ties to the lower index), each half in
  ascending channel order.
* RoPE acts on the whole head vector before the split ("TurboESM ...",
  section 2.A: RoPE first, then the rotation).
* The logit of a key is the sum of the two codecs' estimates of their halves'
  inner products, ``<q, k> = <q[O], k[O]> + <q[R], k[R]>``; the output puts
  each value half, reconstructed by its codec, back at its channels.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import attention as att
from . import codec as oc
from .rotation import apply_rope


@dataclass
class SplitCodec:
    d: int
    hi: oc.Codec          # outlier channels
    lo: oc.Codec          # the other channels
    channels: np.ndarray  # int64 [Hkv, 2, d]


def outlier_channels(score: np.ndarray) -> np.ndarray:
    """score [..., d] -> permutation [..., d]: the d/2 highest-scoring channels
    (ties to the lower index) in ascending order, then the rest ascending."""
    score = np.asarray(score, dtype=np.float64)
    d = score.shape[-1]
    flat = score.reshape(-1, d)
    out = np.empty(flat.shape, dtype=np.int64)
    for r, s in enumerate(flat):
        order = sorted(range(d), key=lambda i: (-s[i], i))
        top = sorted(order[:d // 2])
        rest = sorted(order[d // 2:])
        out[r] = top + rest
    return out.reshape(score.shape)


def make_split_codec(hi: oc.Codec, lo: oc.Codec, channels: np.ndarray) -> SplitCodec:
    if hi.d != lo.d:
        raise ValueError("both codecs code d/2 channels")
    ch = np.asarray(channels, dtype=np.int64)
    d = 2 * hi.d
    if ch.ndim != 3 or ch.shape[1:] != (2, d):
        raise ValueError("channels must be [Hkv, 2, d]")
    for row in ch.reshape(-1, d):
        if sorted(row.tolist()) != list(range(d)):
            raise ValueError("each channel list must be a permutation of 0..d-1")
    return SplitCodec(d, hi, lo, ch)


def rate_bits(sc: SplitCodec) -> tuple[float, float]:
    """Bits per channel of keys and values (norm words excluded)."""
    return (sc.hi.bits_k + sc.lo.bits_k) / 2.0, (sc.hi.bits_v + sc.lo.bits_v) / 2.0


def bytes_per_row(sc: SplitCodec) -> tuple[int, int]:
    """Compressed bytes per (token, head) of both halves: keys, values."""
    kh, vh = oc.bytes_per_row(sc.hi)
    kl, vl = oc.bytes_per_row(sc.lo)
    return kh + kl, vh + vl


def empty_caches(sc: SplitCodec, B: int, Hkv: int, rows_cap: int):
    return oc.empty_cache(sc.hi, B, Hkv, rows_cap), oc.empty_cache(sc.lo, B, Hkv, rows_cap)


def quantize_into(caches, K: np.ndarray, V: np.ndarray, sc: SplitCodec, rope=None,
                  pos0: int = 0, row0: int = 0) -> dict:
    """Encode K, V [B, Hkv, T, d] into rows [row0, row0 + T) of both caches.
    RoPE (if given) turns K at positions pos0.. over all d channels first; then
    each KV head's channel sets go to their codecs.  Returns the bad-row count
    and the per-row encodings enc[(half, b, h)] = (keys, values)."""
    B, H, T, d = K.shape
    K = np.asarray(K, np.float64)
    if rope is not None:
        K = apply_rope(K, rope[0], rope[1], np.arange(pos0, pos0 + T))
    V = np.asarray(V, np.float64)
    half = d // 2
    bad = 0
    enc = {}
    for h in range(H):
        ck, cv = sc.channels[h, 0], sc.channels[h, 1]
        for part, codec, sel in ((0, sc.hi, slice(0, half)), (1, sc.lo, slice(half, d))):
            kh = K[:, h:h + 1][..., ck[sel]]
            vh = V[:, h:h + 1][..., cv[sel]]
            # views of KV head h: the codec writes through them
            sub = {key: (val[:, h:h + 1] if isinstance(val, np.ndarray) else val)
                   for key, val in caches[part].items()}
            diag = oc.quantize_into(sub, kh, vh, codec, rope=None, row0=row0)
            bad += diag["bad_rows"]
            for b in range(B):
                enc[(part, b, h)] = (diag["k"][b], diag["v"][b])
    return dict(bad_rows=bad, enc=enc)


def decode(q: np.ndarray, caches, sc: SplitCodec, seq_lens, scale: float, rope=None,
           heads=None, want_logits: bool = False):
    """One decode step over the split cache.  q: [B, Hq, d] (pre-RoPE)."""
    B, Hq, d = q.shape
    Hkv = caches[0]["kcode"].shape[1]
    G = Hq // Hkv
    half = d // 2
    out = np.full((B, Hq, d), np.nan)
    logits = {}
    heads = [(b, h) for b in range(B) for h in range(Hq)] if heads is None else heads
    for b, h in heads:
        kvh = h // G
        T = int(seq_lens[b])
        qv = np.asarray(q[b, h], np.float64)[None, :]
        if rope is not None:
            qv = apply_rope(qv, rope[0], rope[1], np.array([T - 1]))
        ck, cv = sc.channels[kvh, 0], sc.channels[kvh, 1]
        lg = np.zeros((1, T))
        vals = np.zeros((T, d))
        for part, codec, sel in ((0, sc.hi, slice(0, half)), (1, sc.lo, slice(half, d))):
            rows = oc.cache_rows(caches[part], codec, b, kvh, T)
            lg = lg + att.estimator_logits(qv[:, ck[sel]], rows, codec, scale)
            vals[:, cv[sel]] = oc.dequant_values(rows[4], rows[5], codec)
        out[b, h] = att.softmax_average(lg, vals)[0]
        if want_logits:
            logits[(b, h)] = lg[0]
    return (out, logits) if want_logits else out


def dequantize(caches, sc: SplitCodec, which: int, b: int, h: int, n: int) -> np.ndarray:
    """Rows 0..n-1 of (b, KV head h) with every half back at its channels."""
    d, half = sc.d, sc.d // 2
    ch = sc.channels[h, which]
    out = np.zeros((n, d))
    for part, codec, sel in ((0, sc.hi, slice(0, half)), (1, sc.lo, slice(half, d))):
        ik, sg, nk, rk, iv, nv = oc.cache_rows(caches[part], codec, b, h, n)
        if which == 0:
            out[:, ch[sel]] = oc.dequant_keys(ik, sg, nk, rk, codec)
        else:
            out[:, ch[sel]] = oc.dequant_values(iv, nv, codec)
    return out
