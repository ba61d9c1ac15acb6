"""TurboQuant_mse / TurboQuant_prod encode, bit layout and dequantize (oracle side).

Sources:
* "FibQuant ..." (gist.science 2605.11478), section 1: a deployable cache codec
  stores each token at a fixed address so that any token decodes on its own by
  address arithmetic (fixed rate, no variable-length codes); section 2.3
  "Codifica e Decodifica": store nu = ||x||, rotate x / nu, quantize, and decode
  by looking the code up, rotating back and scaling by nu.
* "Google presenta TurboQuant..." (7minutos.es), "La mecanica geometrica de
  TurboQuant": per-coordinate scalar codebook (vectorised compares, no binary
  search); "Eliminacion del sesgo interno del producto": TURBOQUANT_prod spends
  b-1 bits on TURBOQUANT_mse, then a 1-bit QJL transform of the residual, and the
  result is an unbiased inner-product estimator E<y, Q^-1(Q(x))> = <y, x>.
* "TurboQuant: Jak rozwiazac ..." (securhub.pl), "Blad sredniokwadratowy to
  pulapka": the same two-stage construction.

Readings (the pages leave these open):
* Zero row: nu = 0 and u = 0; codes are those of u = 0 and dequantize gives 0.
* Threshold ties go to the upper cell: idx_i = #{k : u_i >= t_k}.
* QJL: S is m x d (m = d) i.i.d. N(0,1) stored as bf16 (the bf16 matrix is the
  sketch); it acts on the rotated-domain residual r = u - c[idx];
  sigma_i = [ (S r)_i >= 0 ]; the dequantized key is
  nu Pi^T (c[idx] + sqrt(pi/2)/m * rho * S^T (2 sigma - 1)), rho = ||r||.
* Integer decisions (codes, signs) are taken in fp32, the kernel's precision:
  the fp64 value is rounded to fp32 before it is compared.
* nu and rho are stored as fp16 (round to nearest even).
* Rows with a non-finite element, or whose fp16 norm overflows, are encoded as
  zero rows and counted.

Bit layout (this library's specification -- parity unpinned by the pages):
* keys  kcode[row][plane][d/8] bytes, planes 0..mse_bits-1 hold bit p of the
  code, the last plane (QJL) holds sigma; coordinate i sits in byte i//8,
  bit i%8 (little-endian 32-bit words).  kscale[row] = (nu, rho) fp16.
* values vcode[row//32][plane][i] uint32 words: bit (row % 32) of word
  (row//32, p, i) is bit p of coordinate i's code ("32-token column groups");
  vnorm[row] fp16.  Every token still sits at fixed addresses.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np

from rotated_codebook_kv_tq_b200 import synth
from . import codebook as cbmod
from .rotation import apply_rope, rotation_matrix


@dataclass
class Codec:
    d: int
    bits_k: int
    qjl_k: bool
    bits_v: int
    D: np.ndarray          # int8 +-1
    S: Optional[np.ndarray]  # fp64 (m x d), values of the bf16 sketch
    Pi: np.ndarray         # fp64 d x d
    cb_k: cbmod.Codebook
    cb_v: cbmod.Codebook

    @property
    def mse_bits_k(self) -> int:
        return self.bits_k - 1 if self.qjl_k else self.bits_k

    @property
    def planes_k(self) -> int:
        return self.mse_bits_k + (1 if self.qjl_k else 0)

    @property
    def qjl_coef(self) -> float:
        """sqrt(pi/2)/m: scale of the QJL term in the estimator."""
        return math.sqrt(math.pi / 2.0) / self.S.shape[0]


def make_codec(d: int, bits_k: int, qjl_k: bool, bits_v: int, D: np.ndarray,
               S_bf16: Optional[np.ndarray], Pi: Optional[np.ndarray] = None) -> Codec:
    """Pi (optional): a dense orthogonal rotation used instead of the
    randomized Walsh-Hadamard H diag(D) / sqrt(d) (e.g. rotation.haar_rotation)."""
    mse_k = bits_k - 1 if qjl_k else bits_k
    if mse_k < 1 or bits_v < 1:
        raise ValueError("each codebook needs at least one bit")
    S = synth.bf16_bits_to_f32(S_bf16).astype(np.float64) if qjl_k else None
    P = rotation_matrix(D) if Pi is None else np.asarray(Pi, np.float64)
    return Codec(d, bits_k, qjl_k, bits_v, np.asarray(D, np.int8), S,
                 P, cbmod.codebook(d, mse_k), cbmod.codebook(d, bits_v))


# ---------------------------------------------------------------------------
# Encode
# ---------------------------------------------------------------------------

def _finite_rows(x: np.ndarray) -> np.ndarray:
    return np.all(np.isfinite(x), axis=-1)


def normalize_rotate(x: np.ndarray, Pi: np.ndarray):
    """nu = ||x||, u = Pi x / nu (u = 0 for a zero row)."""
    nu = np.sqrt(np.sum(x * x, axis=-1))
    safe = np.where(nu > 0, nu, 1.0)
    u = (x @ Pi.T) / safe[:, None]
    u[nu == 0] = 0.0
    return nu, u


def scalar_codes(u: np.ndarray, thresholds32: np.ndarray) -> np.ndarray:
    """idx_i = #{k : fp32(u_i) >= t_k} against fp32 thresholds."""
    u32 = u.astype(np.float32)
    return np.sum(u32[..., None] >= thresholds32[None, None, :], axis=-1).astype(np.int64)


def _to_f16(v: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return v.astype(np.float16)


def _sanitize(x: np.ndarray):
    x = np.array(x, dtype=np.float64, copy=True)
    bad = ~_finite_rows(x)
    x[bad] = 0.0
    return x, bad


def quantize_values(x: np.ndarray, codec: Codec) -> dict:
    """TurboQuant_mse at bits_v bits."""
    x, bad = _sanitize(x)
    nu, u = normalize_rotate(x, codec.Pi)
    nu16 = _to_f16(nu)
    over = ~np.isfinite(nu16)
    if over.any():
        x[over] = 0.0
        bad = bad | over
        nu, u = normalize_rotate(x, codec.Pi)
        nu16 = _to_f16(nu)
    idx = scalar_codes(u, codec.cb_v.thresholds32)
    return dict(idx=idx, nu=nu, nu16=nu16, u=u, bad=bad)


def quantize_keys(x: np.ndarray, codec: Codec) -> dict:
    """TurboQuant_prod: (bits_k - 1)-bit MSE stage plus a 1-bit QJL sketch of the
    residual (or the plain MSE stage at bits_k bits when QJL is off)."""
    x, bad = _sanitize(x)
    nu, u = normalize_rotate(x, codec.Pi)
    nu16 = _to_f16(nu)
    over = ~np.isfinite(nu16)
    if over.any():
        x[over] = 0.0
        bad = bad | over
        nu, u = normalize_rotate(x, codec.Pi)
        nu16 = _to_f16(nu)
    idx = scalar_codes(u, codec.cb_k.thresholds32)
    out = dict(idx=idx, nu=nu, nu16=nu16, u=u, bad=bad)
    if codec.qjl_k:
        r = u - codec.cb_k.centroids32.astype(np.float64)[idx]
        rho = np.sqrt(np.sum(r * r, axis=-1))
        z = r @ codec.S.T
        out.update(r=r, rho=rho, rho16=_to_f16(rho), z=z,
                   sigma=z.astype(np.float32) >= 0)
    else:
        out.update(rho=np.zeros_like(nu), rho16=np.zeros(nu.shape, np.float16))
    return out


# ---------------------------------------------------------------------------
# Bit layout
# ---------------------------------------------------------------------------

def _bits_to_bytes(bits: np.ndarray) -> np.ndarray:
    """[..., d] of 0/1 -> [..., d/8] bytes, coordinate i in byte i//8 bit i%8."""
    d = bits.shape[-1]
    b = bits.reshape(bits.shape[:-1] + (d // 8, 8)).astype(np.uint16)
    weights = (1 << np.arange(8)).astype(np.uint16)
    return np.sum(b * weights, axis=-1).astype(np.uint8)


def _bytes_to_bits(by: np.ndarray) -> np.ndarray:
    sh = np.arange(8, dtype=np.uint8)
    bits = (by[..., None] >> sh) & 1
    return bits.reshape(by.shape[:-1] + (by.shape[-1] * 8,)).astype(np.int64)


def pack_keys(enc: dict, codec: Codec):
    """-> kcode [N, planes_k, d/8] uint8, kscale [N, 2] float16 (nu, rho)."""
    idx = enc["idx"]
    planes = [(idx >> p) & 1 for p in range(codec.mse_bits_k)]
    if codec.qjl_k:
        planes.append(enc["sigma"].astype(np.int64))
    kcode = np.stack([_bits_to_bytes(p) for p in planes], axis=1)
    kscale = np.stack([enc["nu16"], enc["rho16"]], axis=-1).astype(np.float16)
    return kcode, kscale


def unpack_keys(kcode: np.ndarray, kscale: np.ndarray, codec: Codec):
    planes = _bytes_to_bits(kcode)                       # [N, P, d]
    idx = np.zeros(planes.shape[::2], dtype=np.int64)    # [N, d]
    for p in range(codec.mse_bits_k):
        idx |= planes[:, p, :] << p
    sigma = planes[:, codec.mse_bits_k, :].astype(bool) if codec.qjl_k else None
    return idx, sigma, kscale[:, 0].astype(np.float64), kscale[:, 1].astype(np.float64)


def pack_values(enc: dict, codec: Codec):
    """-> vcode [N/32, bits_v, d] uint32 (32-token column groups), vnorm [N] f16.
    N must be a multiple of 32."""
    idx = enc["idx"]
    n, d = idx.shape
    if n % 32:
        raise ValueError("value rows must come in groups of 32")
    g = idx.reshape(n // 32, 32, d)
    vcode = np.zeros((n // 32, codec.bits_v, d), dtype=np.uint32)
    for p in range(codec.bits_v):
        bit = ((g >> p) & 1).astype(np.uint64)                   # [G, 32, d]
        word = np.sum(bit << np.arange(32, dtype=np.uint64)[None, :, None], axis=1)
        vcode[:, p, :] = word.astype(np.uint32)
    return vcode, enc["nu16"].astype(np.float16)


def unpack_values(vcode: np.ndarray, vnorm: np.ndarray, codec: Codec):
    ng, P, d = vcode.shape
    sh = np.arange(32, dtype=np.uint32)
    idx = np.zeros((ng, 32, d), dtype=np.int64)
    for p in range(P):
        bits = (vcode[:, p, None, :] >> sh[None, :, None]) & 1    # [G, 32, d]
        idx |= bits.astype(np.int64) << p
    return idx.reshape(ng * 32, d), vnorm.astype(np.float64)


# ---------------------------------------------------------------------------
# Decode (dequantize)
# ---------------------------------------------------------------------------

def dequant_keys(idx, sigma, nu, rho, codec: Codec) -> np.ndarray:
    """x~ = nu Pi^T (c[idx] + sqrt(pi/2)/m rho S^T (2 sigma - 1))."""
    y = codec.cb_k.centroids32.astype(np.float64)[idx]
    if codec.qjl_k:
        y = y + codec.qjl_coef * rho[:, None] * ((2.0 * sigma - 1.0) @ codec.S)
    return nu[:, None] * (y @ codec.Pi)


def dequant_values(idx, nu, codec: Codec) -> np.ndarray:
    """v~ = nu Pi^T c_v[idx]."""
    return nu[:, None] * (codec.cb_v.centroids32.astype(np.float64)[idx] @ codec.Pi)


# ---------------------------------------------------------------------------
# Whole-cache helpers ([B, Hkv, T, d] inputs)
# ---------------------------------------------------------------------------

def empty_cache(codec: Codec, B: int, Hkv: int, rows_cap: int) -> dict:
    if rows_cap % 32:
        raise ValueError("rows_cap must be a multiple of 32")
    d = codec.d
    return dict(
        kcode=np.zeros((B, Hkv, rows_cap, codec.planes_k, d // 8), np.uint8),
        kscale=np.zeros((B, Hkv, rows_cap, 2), np.float16),
        vcode=np.zeros((B, Hkv, rows_cap // 32, codec.bits_v, d), np.uint32),
        vnorm=np.zeros((B, Hkv, rows_cap), np.float16),
        rows_cap=rows_cap)


def quantize_into(cache: dict, K: np.ndarray, V: np.ndarray, codec: Codec,
                  rope=None, pos0: int = 0, row0: int = 0) -> dict:
    """Encode K, V [B, Hkv, T, d] (fp64 values) into cache rows
    [row0, row0 + T).  RoPE (if given) is applied to K at positions
    pos0 .. pos0+T-1 before encoding.  Returns per-row diagnostics."""
    B, H, T, d = K.shape
    diag = dict(bad_rows=0, k=[], v=[])
    for b in range(B):
        for h in range(H):
            k = np.asarray(K[b, h], np.float64)
            if rope is not None:
                k = apply_rope(k, rope[0], rope[1], np.arange(pos0, pos0 + T))
            ek = quantize_keys(k, codec)
            ev = quantize_values(np.asarray(V[b, h], np.float64), codec)
            kc, ks = pack_keys(ek, codec)
            cache["kcode"][b, h, row0:row0 + T] = kc
            cache["kscale"][b, h, row0:row0 + T] = ks
            cache["vnorm"][b, h, row0:row0 + T] = ev["nu16"]
            # values: read-modify-write of the 32-token groups touched
            g0, g1 = row0 // 32, (row0 + T + 31) // 32
            idx_all, _ = unpack_values(cache["vcode"][b, h, g0:g1],
                                       cache["vnorm"][b, h, g0 * 32:g1 * 32], codec)
            idx_all[row0 - g0 * 32: row0 - g0 * 32 + T] = ev["idx"]
            vc, _ = pack_values(dict(idx=idx_all, nu16=np.zeros(len(idx_all), np.float16)), codec)
            cache["vcode"][b, h, g0:g1] = vc
            diag["bad_rows"] += int(ek["bad"].sum() + ev["bad"].sum())
            diag["k"].append(ek)
            diag["v"].append(ev)
    return diag


def cache_rows(cache: dict, codec: Codec, b: int, h: int, n: int):
    """Unpacked (idx_k, sigma, nu_k, rho, idx_v, nu_v) of rows 0..n-1."""
    ik, sg, nk, rk = unpack_keys(cache["kcode"][b, h, :n], cache["kscale"][b, h, :n], codec)
    ng = (n + 31) // 32
    iv, nv = unpack_values(cache["vcode"][b, h, :ng], cache["vnorm"][b, h, :ng * 32], codec)
    return ik, sg, nk, rk, iv[:n], nv[:n]


def bytes_per_row(codec: Codec) -> tuple[int, int]:
    """Compressed bytes per (token, head): keys, values."""
    kb = codec.planes_k * codec.d // 8 + 4
    vb = codec.bits_v * codec.d // 8 + 2
    return kb, vb
