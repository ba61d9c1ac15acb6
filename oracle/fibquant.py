"""FibQuant k = 2: a shared two-dimensional vector codebook for the rotated
coordinates (oracle side).

Source: "FibQuant: Quantizzazione Vettoriale Universale per la Compressione della
KV-Cache ad Accesso Casuale" (gist.science 2605.11478):
* section 2.1 "La Sorgente Canonica": after normalisation and a Haar rotation
  any block of k consecutive coordinates follows one spherical-Beta density
  f_{d,k} on the unit ball B^k, so one offline code serves every head;
* section 2.2 "Costruzione del Codice": radii fitted to the radial law by
  Bennett-Gersho companding (for k = 2 a closed form in Beta quantiles),
  directions on the planar Fibonacci (golden-angle) spiral, then a multi-restart
  Lloyd-Max refinement of that deterministic start for the finite size N;
* section 2.3 "Codifica e Decodifica": store nu, rotate x / nu, cut it into d/k
  blocks, code each by its nearest codeword; decode by codeword lookup,
  concatenation, inverse rotation and scaling by nu; rate b = log2(N) / k bits
  per coordinate.

Readings (the page names the parts without formulas):
* f_{d,2}(x) = (d - 2)/(2 pi) (1 - |x|^2)^((d - 4)/2) on the unit disk, the
  law of two coordinates of a uniform point on S^{d-1}; |x|^2 ~ Beta(1, (d-2)/2).
* Bennett-Gersho point density ~ f^(k/(k+2)) = f^(1/2); in the plane its radial
  CDF is 1 - (1 - r^2)^(d/4), so codeword n of N sits at the radius whose
  CDF is (n + delta)/N: r_n^2 = 1 - (1 - (n + delta)/N)^(4/d) (a Beta(1, d/4)
  quantile), delta = 1/2 for the deterministic start.
* Directions theta_n = n * pi (3 - sqrt 5) (golden angle).
* Lloyd-Max on a fixed quadrature of f: NU shells of |x|^2 of equal
  probability under its Beta law, each at its conditional mean of |x|^2,
  angles at 2 pi (j + 1/2)/NA, equal weights;
  a fixed number of steps (nearest codeword, ties to the lower index; each
  codeword moves to the mean of its points, an empty cell keeps its codeword).
  Restarts: delta in {1/4, 1/2, 3/4} (rotating a start changes nothing, f is
  radially symmetric); the restart with the smallest quadrature MSE wins, an
  earlier one unless a later one is lower by more than a relative 1e-9 (so
  restarts that reach the same code keep the earlier labels).  Codewords
  stored as fp32.
* N = 2^m with m bits per block (fixed-address planes); blocks are the
  coordinate pairs (2j, 2j + 1) of the rotated unit vector (the randomized
  Walsh-Hadamard rotation of the TurboQuant codec stands in for Haar).
* The nearest-codeword decision is taken on fp32 values (the kernel's
  precision); squared distances in fp64 here.
* Both keys and values use the code (no QJL stage); the attention logit is
  s * nu * sum_j <q'_(2j, 2j+1), c[idx_j]>.

Layout: keys kcode[row][plane][d/16] bytes (plane p holds bit p of each
block's code; block j in byte j // 8, bit j % 8), kscale[row] = (nu, 0) fp16;
values vcode[row // 32][plane][d/2] uint32 words (bit row % 32 of word
(row // 32, p, j) is bit p of block j's code), vnorm[row] fp16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from .codec import _bits_to_bytes, _bytes_to_bits, _sanitize, _to_f16, normalize_rotate
from .rotation import apply_rope, rotation_matrix

GOLDEN_ANGLE = math.pi * (3.0 - math.sqrt(5.0))
RESTART_DELTAS = (0.25, 0.5, 0.75)
GRID_NU = 256
GRID_NA = 256
LLOYD_STEPS = 100
RESTART_MARGIN = 1e-9


def pair_density(x: np.ndarray, d: int) -> np.ndarray:
    """f_{d,2} at points x [..., 2] (zero outside the unit disk)."""
    r2 = np.sum(np.asarray(x, np.float64) ** 2, axis=-1)
    inside = r2 < 1.0
    out = np.zeros(r2.shape)
    out[inside] = (d - 2) / (2 * math.pi) * (1.0 - r2[inside]) ** ((d - 4) / 2.0)
    return out


def start_codebook(d: int, N: int, delta: float = 0.5) -> np.ndarray:
    """Companded radii on the golden-angle spiral: [N, 2] fp64."""
    n = np.arange(N, dtype=np.float64)
    r = np.sqrt(1.0 - (1.0 - (n + delta) / N) ** (4.0 / d))
    th = n * GOLDEN_ANGLE
    return np.stack([r * np.cos(th), r * np.sin(th)], axis=1)


def quadrature(d: int, nu: int = GRID_NU, na: int = GRID_NA) -> np.ndarray:
    """Equal-weight points of f_{d,2}: [nu * na, 2].  |x|^2 = T ~ Beta(1, b),
    b = (d-2)/2, is cut into nu shells of equal probability; shell i is
    represented by its conditional mean of T (closed form), so E|x|^2 = 2/d
    holds exactly on the grid."""
    b = (d - 2) / 2.0
    a = np.arange(nu + 1, dtype=np.float64) / nu          # CDF values of the shell edges
    t = 1.0 - (1.0 - a) ** (1.0 / b)
    e = (t[:-1] * (1.0 - a[:-1]) - t[1:] * (1.0 - a[1:])
         + ((1.0 - a[:-1]) ** ((b + 1) / b) - (1.0 - a[1:]) ** ((b + 1) / b)) / (b + 1))
    r = np.sqrt(e * nu)
    ph = 2 * math.pi * (np.arange(na) + 0.5) / na
    return np.stack([(r[:, None] * np.cos(ph)[None, :]).ravel(),
                     (r[:, None] * np.sin(ph)[None, :]).ravel()], axis=1)


def _nearest(pts: np.ndarray, cb: np.ndarray, chunk: int = 16384):
    """Index of the nearest codeword (ties to the lower index) and the squared
    distance, fp64."""
    idx = np.empty(len(pts), np.int64)
    dist = np.empty(len(pts))
    for a in range(0, len(pts), chunk):
        p = pts[a:a + chunk]
        d2 = (p[:, None, 0] - cb[None, :, 0]) ** 2 + (p[:, None, 1] - cb[None, :, 1]) ** 2
        i = np.argmin(d2, axis=1)
        idx[a:a + chunk] = i
        dist[a:a + chunk] = d2[np.arange(len(p)), i]
    return idx, dist


def lloyd(cb: np.ndarray, pts: np.ndarray, steps: int = LLOYD_STEPS) -> np.ndarray:
    cb = np.array(cb, np.float64, copy=True)
    N = len(cb)
    for _ in range(steps):
        idx, _ = _nearest(pts, cb)
        cnt = np.bincount(idx, minlength=N)
        sx = np.bincount(idx, weights=pts[:, 0], minlength=N)
        sy = np.bincount(idx, weights=pts[:, 1], minlength=N)
        nz = cnt > 0
        cb[nz, 0] = sx[nz] / cnt[nz]
        cb[nz, 1] = sy[nz] / cnt[nz]
    return cb


def quad_mse(cb: np.ndarray, pts: np.ndarray) -> float:
    """Mean squared distance per block (two coordinates) on the quadrature."""
    return float(np.mean(_nearest(pts, cb)[1]))


@dataclass(frozen=True)
class PairCodebook:
    d: int
    bits: int                 # m: bits per block, N = 2^m
    centroids: np.ndarray     # fp64 [N, 2]
    mse_per_pair: float       # quadrature MSE per block at the solution
    restart: int

    @property
    def centroids32(self) -> np.ndarray:
        return self.centroids.astype(np.float32)

    @property
    def rate(self) -> float:
        return self.bits / 2.0


_CACHE: dict = {}


def pair_codebook(d: int, bits: int) -> PairCodebook:
    key = (d, bits)
    if key not in _CACHE:
        if d < 4 or bits < 1:
            raise ValueError("need d >= 4 and at least one bit per block")
        pts = quadrature(d)
        best = None
        for j, delta in enumerate(RESTART_DELTAS):
            cb = lloyd(start_codebook(d, 1 << bits, delta), pts)
            m = quad_mse(cb, pts)
            # a later restart wins only by a clear margin, so restarts that
            # reach the same code (up to rounding) keep the earlier labels
            if best is None or m < best[1] * (1.0 - RESTART_MARGIN):
                best = (cb, m, j)
        _CACHE[key] = PairCodebook(d, bits, best[0], best[1], best[2])
    return _CACHE[key]


# ---------------------------------------------------------------------------
# Codec
# ---------------------------------------------------------------------------

@dataclass
class FqCodec:
    d: int
    bits_k: int               # bits per block of keys
    bits_v: int
    D: np.ndarray
    Pi: np.ndarray
    cb_k: PairCodebook
    cb_v: PairCodebook


def make_codec(d: int, bits_k: int, bits_v: int, D: np.ndarray) -> FqCodec:
    if d % 2:
        raise ValueError("d must be even")
    return FqCodec(d, bits_k, bits_v, np.asarray(D, np.int8), rotation_matrix(D),
                   pair_codebook(d, bits_k), pair_codebook(d, bits_v))


def encode(x: np.ndarray, Pi: np.ndarray, cb: PairCodebook) -> dict:
    """nu, the rotated unit vector u and the block codes of rows x [n, d]."""
    x, bad = _sanitize(x)
    nu, u = normalize_rotate(x, Pi)
    nu16 = _to_f16(nu)
    over = ~np.isfinite(nu16)
    if over.any():
        x[over] = 0.0
        bad = bad | over
        nu, u = normalize_rotate(x, Pi)
        nu16 = _to_f16(nu)
    n, d = u.shape
    pairs = u.astype(np.float32).astype(np.float64).reshape(n * d // 2, 2)
    idx, _ = _nearest(pairs, cb.centroids32.astype(np.float64))
    return dict(idx=idx.reshape(n, d // 2), nu=nu, nu16=nu16, u=u, bad=bad)


def decode_rows(idx: np.ndarray, nu: np.ndarray, codec: FqCodec, cb: PairCodebook) -> np.ndarray:
    """x~ = nu Pi^T concat_j c[idx_j]."""
    n = idx.shape[0]
    y = cb.centroids32.astype(np.float64)[idx].reshape(n, codec.d)
    return nu[:, None] * (y @ codec.Pi)


def empty_cache(codec: FqCodec, B: int, Hkv: int, rows_cap: int) -> dict:
    if rows_cap % 32 or codec.d % 16:
        raise ValueError("rows_cap must be a multiple of 32 and d of 16")
    d = codec.d
    return dict(kcode=np.zeros((B, Hkv, rows_cap, codec.bits_k, d // 16), np.uint8),
                kscale=np.zeros((B, Hkv, rows_cap, 2), np.float16),
                vcode=np.zeros((B, Hkv, rows_cap // 32, codec.bits_v, d // 2), np.uint32),
                vnorm=np.zeros((B, Hkv, rows_cap), np.float16),
                rows_cap=rows_cap)


def _pack_values(idx: np.ndarray, bits: int) -> np.ndarray:
    n, nb = idx.shape
    g = idx.reshape(n // 32, 32, nb)
    out = np.zeros((n // 32, bits, nb), np.uint32)
    for p in range(bits):
        bit = ((g >> p) & 1).astype(np.uint64)
        out[:, p, :] = np.sum(bit << np.arange(32, dtype=np.uint64)[None, :, None], axis=1).astype(np.uint32)
    return out


def _unpack_values(vcode: np.ndarray) -> np.ndarray:
    ng, P, nb = vcode.shape
    sh = np.arange(32, dtype=np.uint32)
    idx = np.zeros((ng, 32, nb), np.int64)
    for p in range(P):
        idx |= (((vcode[:, p, None, :] >> sh[None, :, None]) & 1).astype(np.int64)) << p
    return idx.reshape(ng * 32, nb)


def quantize_into(cache: dict, K: np.ndarray, V: np.ndarray, codec: FqCodec, rope=None,
                  pos0: int = 0, row0: int = 0) -> dict:
    """Encode K, V [B, Hkv, T, d] into rows [row0, row0 + T); RoPE on K first."""
    B, H, T, d = K.shape
    diag = dict(bad_rows=0, k=[], v=[])
    for b in range(B):
        for h in range(H):
            k = np.asarray(K[b, h], np.float64)
            if rope is not None:
                k = apply_rope(k, rope[0], rope[1], np.arange(pos0, pos0 + T))
            ek = encode(k, codec.Pi, codec.cb_k)
            ev = encode(np.asarray(V[b, h], np.float64), codec.Pi, codec.cb_v)
            planes = [_bits_to_bytes((ek["idx"] >> p) & 1) for p in range(codec.bits_k)]
            cache["kcode"][b, h, row0:row0 + T] = np.stack(planes, axis=1)
            cache["kscale"][b, h, row0:row0 + T, 0] = ek["nu16"]
            cache["kscale"][b, h, row0:row0 + T, 1] = 0
            cache["vnorm"][b, h, row0:row0 + T] = ev["nu16"]
            g0, g1 = row0 // 32, (row0 + T + 31) // 32
            iv = _unpack_values(cache["vcode"][b, h, g0:g1])
            iv[row0 - g0 * 32: row0 - g0 * 32 + T] = ev["idx"]
            cache["vcode"][b, h, g0:g1] = _pack_values(iv, codec.bits_v)
            diag["bad_rows"] += int(ek["bad"].sum() + ev["bad"].sum())
            diag["k"].append(ek)
            diag["v"].append(ev)
    return diag


def cache_rows(cache: dict, codec: FqCodec, b: int, h: int, n: int):
    """(key block codes, nu_k, value block codes, nu_v) of rows 0..n-1."""
    bits = _bytes_to_bits(cache["kcode"][b, h, :n])           # [n, P, d/2]
    ik = np.zeros((n, codec.d // 2), np.int64)
    for p in range(codec.bits_k):
        ik |= bits[:, p, :] << p
    nk = cache["kscale"][b, h, :n, 0].astype(np.float64)
    ng = (n + 31) // 32
    iv = _unpack_values(cache["vcode"][b, h, :ng])[:n]
    nv = cache["vnorm"][b, h, :n].astype(np.float64)
    return ik, nk, iv, nv


def decode(q: np.ndarray, cache: dict, codec: FqCodec, seq_lens, scale: float, rope=None):
    """One decode step: q [B, Hq, d] (pre-RoPE) -> out [B, Hq, d]."""
    B, Hq, d = q.shape
    Hkv = cache["kcode"].shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        T = int(seq_lens[b])
        for kvh in range(Hkv):
            ik, nk, iv, nv = cache_rows(cache, codec, b, kvh, T)
            ck = codec.cb_k.centroids32.astype(np.float64)[ik].reshape(T, d)   # rotated domain
            vals = decode_rows(iv, nv, codec, codec.cb_v)
            qs = np.asarray(q[b, kvh * G:(kvh + 1) * G], np.float64)
            if rope is not None:
                qs = apply_rope(qs, rope[0], rope[1], np.full(G, T - 1))
            lg = scale * nk[None, :] * ((qs @ codec.Pi.T) @ ck.T)
            m = np.max(lg, axis=1, keepdims=True)
            p = np.exp(lg - m)
            out[b, kvh * G:(kvh + 1) * G] = (p @ vals) / np.sum(p, axis=1, keepdims=True)
    return out


def bytes_per_row(codec: FqCodec) -> tuple[int, int]:
    return codec.bits_k * codec.d // 16 + 4, codec.bits_v * codec.d // 16 + 2
