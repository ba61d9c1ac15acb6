"""Seeded synthetic inputs shared by the CUDA path and the CPU oracle.

This module draws random numbers and lays them out; it holds none of the
codec's arithmetic (no norms, rotations, codebooks, codes or attention).
Everything the codec draws at random (the rotation's sign vector D and the
QJL Gaussian matrix S) is produced here and passed in as an input, so that the
oracle and the library see the same bits.

Generator: numpy PCG64 seeded with ``SeedSequence([seed, stream])``; the
ablation page (gist.science 2607.09683, "Validazione") runs its oracle on
PCG64 as well.  Streams: 0 = keys, 1 = values, 2 = queries,
3 = channel scales / outlier channels, 4 = rotation signs D, 5 = QJL matrix S,
6 = the Gaussian matrix behind a dense Haar rotation.
Draw order is row-major over [B, H, T, d].

Workload recipes (shapes follow the pages' workloads; values are synthetic
stand-ins because no model weights or datasets are available):

* ``tiny``      - 1 head, d=128, 1024 keys/values, fp32 N(0,1), seed 0; keys
                  2-bit MSE + 1-bit QJL, values 3-bit.
* ``llama_decode`` - Llama-3.1-8B-shaped decode layer: B=1, 32 query / 8 KV
                  heads, d=128, context 32768, bf16 N(0,1) x lognormal(0,1)
                  channel scales with 4 outlier channels x20 per head; RoPE
                  theta 5e5 on K and q; keys 3+QJL bits, values 4 bits.
* ``esm_prefill`` - ESM-2-650M-shaped prefill: B=16, 20 heads, d=64, T=1024,
                  same channel law, RoPE theta 1e4; keys 2+QJL, values 3 bits.
* ``long_decode`` - B=4, 32 query / 8 KV heads, d=128, T=131072, lognormal
                  sigma 1.5 channel scales, no outliers, no RoPE; keys 1+QJL,
                  values 2 bits; 128 split-K chunks.
* ``vector_search`` - 10^6 unit-norm d=1536 fp32 database rows, 1024 unit
                  queries, TurboQuant_prod at 4 bits (3 + QJL).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

STREAM_K, STREAM_V, STREAM_Q, STREAM_SCALES, STREAM_D, STREAM_S, STREAM_HAAR = range(7)


def generator(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


# ----------------------------------------------------------------------------
# bf16 representation helpers (storage format of inputs, not codec math)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).reshape(-1)
    out = np.empty(b.shape, dtype=np.uint16)
    step = 1 << 24
    for a in range(0, b.size, step):      # finite inputs: no uint32 overflow
        c = b[a:a + step]
        out[a:a + step] = ((c + np.uint32(0x7FFF) + ((c >> 16) & 1)) >> 16).astype(np.uint16)
    return out.reshape(np.shape(x))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# Codec randomness
# ----------------------------------------------------------------------------

def rotation_signs(d: int, seed: int) -> np.ndarray:
    """i.i.d. Rademacher vector D (int8, +-1) of the randomized Hadamard rotation."""
    g = generator(seed, STREAM_D)
    return np.where(g.integers(0, 2, size=d) == 1, 1, -1).astype(np.int8)


def qjl_matrix_bf16(d: int, seed: int, m: Optional[int] = None) -> np.ndarray:
    """QJL sketch S (m x d, default m = d), i.i.d. N(0,1) drawn in fp32, stored as
    bf16.  The bf16 matrix IS the sketch for every consumer.  Returns uint16 bits."""
    m = d if m is None else m
    g = generator(seed, STREAM_S)
    return f32_to_bf16_bits(g.standard_normal((m, d), dtype=np.float32))


# ----------------------------------------------------------------------------
# RoPE angle table (positional-encoding input of the model, computed in fp64
# and handed to both sides as fp32)
# ----------------------------------------------------------------------------

def haar_gaussian(d: int, seed: int) -> np.ndarray:
    """d x d i.i.d. N(0,1) fp32 (row-major): the random input of a dense Haar
    rotation (its QR factorisation is the method's arithmetic, not done here)."""
    return generator(seed, STREAM_HAAR).standard_normal((d, d), dtype=np.float32)


def rope_table(t_max: int, d: int, theta: float) -> tuple[np.ndarray, np.ndarray]:
    """cos/sin tables [t_max, d/2] fp32 for rotate-half RoPE with base theta."""
    half = d // 2
    inv_freq = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = np.arange(t_max, dtype=np.float64)[:, None] * inv_freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


# ----------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    bits_k: int          # total key bits (MSE bits + 1 when qjl)
    qjl_k: bool
    bits_v: int
    dtype: str           # "fp32" | "bf16"
    rope_theta: Optional[float]
    sigma_scale: Optional[float]   # lognormal sigma of channel scales (None: unit)
    n_outliers: int
    outlier_gain: float
    num_splits: int      # split-K chunks per (batch, KV head); 0 = the library's default
    Lq: int = 1          # queries per head (1 = decode, T = bidirectional)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 0, 1, 1, 1, 128, 1024, 3, True, 3, "fp32", None, None, 0, 1.0, 8),
    "llama_decode": Workload("llama_decode", 1, 1, 32, 8, 128, 32768, 4, True, 4, "bf16",
                             500000.0, 1.0, 4, 20.0, 0),
    "esm_prefill": Workload("esm_prefill", 2, 16, 20, 20, 64, 1024, 3, True, 3, "bf16",
                            10000.0, 1.0, 4, 20.0, 8, Lq=1024),
    "long_decode": Workload("long_decode", 3, 4, 32, 8, 128, 131072, 2, True, 2, "bf16",
                            None, 1.5, 0, 1.0, 128),
}


@dataclasses.dataclass(frozen=True)
class SearchWorkload:
    """Vector-search recipe: ``n`` database rows and ``nq`` queries, unit-norm
    N(0,1) fp32 of dimension d (streams 0 and 2 of ``seed``), TurboQuant_prod
    at ``bits`` total bits, top-``k`` per query."""
    name: str
    seed: int
    n: int
    nq: int
    d: int
    bits: int
    k: int

    def scaled(self, **kw) -> "SearchWorkload":
        return dataclasses.replace(self, **kw)


VECTOR_SEARCH = SearchWorkload("vector_search", 4, 1_000_000, 1024, 1536, 4, 10)


def search_inputs(w: SearchWorkload):
    """(database [n, d], queries [nq, d]) fp32 unit rows."""
    return unit_rows(w.n, w.d, w.seed, STREAM_K), unit_rows(w.nq, w.d, w.seed, STREAM_Q)


def channel_scales(w: Workload) -> tuple[np.ndarray, np.ndarray]:
    """Per (KV head, channel) scales for K and V: lognormal(0, sigma) with
    ``n_outliers`` random channels per head multiplied by ``outlier_gain``."""
    if w.sigma_scale is None:
        one = np.ones((w.Hkv, w.d), dtype=np.float64)
        return one, one.copy()
    g = generator(w.seed, STREAM_SCALES)
    out = []
    for _ in range(2):  # K then V
        s = g.lognormal(0.0, w.sigma_scale, size=(w.Hkv, w.d))
        for h in range(w.Hkv):
            if w.n_outliers:
                ch = g.choice(w.d, size=w.n_outliers, replace=False)
                s[h, ch] *= w.outlier_gain
        out.append(s)
    return out[0], out[1]


def _normal_rows(g: np.random.Generator, shape, chunk_rows: int = 1 << 16) -> np.ndarray:
    """fp32 N(0,1) of ``shape`` drawn sequentially (row-major), chunked so the
    bit stream does not depend on memory limits."""
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.float32)
    step = chunk_rows * shape[-1]
    for a in range(0, total, step):
        b = min(total, a + step)
        out[a:b] = g.standard_normal(b - a, dtype=np.float32)
    return out.reshape(shape)


def kv_inputs(w: Workload, T: Optional[int] = None):
    """K, V of shape [B, Hkv, T, d].  fp32 workloads return float32 arrays;
    bf16 workloads return uint16 bf16 bits.  ``T`` defaults to the workload's."""
    T = w.T if T is None else T
    if w.name == "tiny":
        g = generator(w.seed, 0)
        k = g.standard_normal((w.B, w.Hkv, T, w.d), dtype=np.float32)
        v = g.standard_normal((w.B, w.Hkv, T, w.d), dtype=np.float32)
        return k, v
    sk, sv = channel_scales(w)
    k = _normal_rows(generator(w.seed, STREAM_K), (w.B, w.Hkv, T, w.d))
    v = _normal_rows(generator(w.seed, STREAM_V), (w.B, w.Hkv, T, w.d))
    k *= sk[None, :, None, :].astype(np.float32)
    v *= sv[None, :, None, :].astype(np.float32)
    if w.dtype == "bf16":
        return f32_to_bf16_bits(k), f32_to_bf16_bits(v)
    return k, v


def query_inputs(w: Workload, Lq: Optional[int] = None):
    """Queries [B, Hq, Lq, d] (N(0,1); bf16 bits for bf16 workloads)."""
    Lq = w.Lq if Lq is None else Lq
    if w.name == "tiny":
        g = generator(w.seed, 0)
        g.standard_normal((w.B, w.Hkv, w.T, w.d), dtype=np.float32)  # K
        g.standard_normal((w.B, w.Hkv, w.T, w.d), dtype=np.float32)  # V
        return g.standard_normal((w.B, w.Hq, Lq, w.d), dtype=np.float32)
    q = _normal_rows(generator(w.seed, STREAM_Q), (w.B, w.Hq, Lq, w.d))
    if w.dtype == "bf16":
        return f32_to_bf16_bits(q)
    return q


def as_float64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored inputs (fp32 or bf16 bits) to float64."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def unit_rows(n: int, d: int, seed: int, stream: int) -> np.ndarray:
    """n rows of N(0,1) fp32 normalised to unit length (vector-search inputs).
    The norm is taken in fp64 row by row; rows are processed in chunks so a
    10^6 x 1536 database needs no fp64 copy of itself."""
    x = _normal_rows(generator(seed, stream), (n, d))
    step = 1 << 16
    for a in range(0, n, step):
        c = x[a:a + step].astype(np.float64)
        c /= np.linalg.norm(c, axis=1, keepdims=True)
        x[a:a + step] = c.astype(np.float32)
    return x


def rope_for(w: Workload, t_max: Optional[int] = None):
    if w.rope_theta is None:
        return None
    return rope_table(w.T if t_max is None else t_max, w.d, w.rope_theta)


def kv_inputs_torch(w: Workload, T: Optional[int] = None, device: str = "cuda", seed_salt: int = 0):
    """Same recipe as ``kv_inputs`` drawn on the device with torch's generator
    (used where only timing matters, e.g. the benchmark; values differ from the
    numpy stream).  Returns bf16 (or fp32) tensors [B, Hkv, T, d]."""
    import torch
    T = w.T if T is None else T
    sk, sv = channel_scales(w)
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1000 + seed_salt)
    out = []
    for s in (sk, sv):
        x = torch.randn((w.B, w.Hkv, T, w.d), generator=g, device=device, dtype=torch.float32)
        x *= torch.as_tensor(s, dtype=torch.float32, device=device)[None, :, None, :]
        out.append(x.to(torch.bfloat16) if w.dtype == "bf16" else x)
    return out[0], out[1]


def query_inputs_torch(w: Workload, Lq: int = 1, device: str = "cuda", seed_salt: int = 0):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1000 + 500 + seed_salt)
    q = torch.randn((w.B, w.Hq, Lq, w.d), generator=g, device=device, dtype=torch.float32)
    return q.to(torch.bfloat16) if w.dtype == "bf16" else q
