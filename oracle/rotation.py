"""Shared random rotation Pi and rotary position embedding (oracle side).

Sources:
* "Ablazione, Inferenza Statistica e Validazione per la Compressione della
  KV-Cache" (gist.science 2607.09683), "Configurazione Sperimentale": TurboQuant
  spreads each token's energy with a randomized Walsh-Hadamard transform.
* "FibQuant ..." (gist.science 2605.11478), section 1: one shared rotation for
  every vector.
* "TurboESM ..." (gist.science 2603.26110), section 2.A "Pipeline di Rotazione
  Invariante a RoPE": RoPE first, then Pi; since Pi^T Pi = I the query-key inner
  product is unchanged, (Pi R_i q)^T (Pi R_j k) = q^T R_i^T R_j k.

Readings: Pi = H_d diag(D) / sqrt(d) with H_d the Sylvester Hadamard matrix in
natural order and D an i.i.d. +-1 vector (one round).  For d = 1536, which is
not a power of two, H = H_12 (Paley construction I over GF(11)) kron H_128.
RoPE uses the rotate-half pairing (i, i + d/2) with the fp32 cos/sin table
passed in; the arithmetic is fp64.
"""
from __future__ import annotations

import numpy as np


def sylvester_hadamard(n: int) -> np.ndarray:
    if n < 1 or n & (n - 1):
        raise ValueError("Sylvester order must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def paley_hadamard(q: int) -> np.ndarray:
    """Paley construction I for a prime q = 3 (mod 4): order q + 1."""
    if q % 4 != 3:
        raise ValueError("Paley I needs q = 3 mod 4")
    residues = {(x * x) % q for x in range(1, q)}

    def chi(a: int) -> int:
        a %= q
        return 0 if a == 0 else (1 if a in residues else -1)

    jac = np.array([[chi(j - i) for j in range(q)] for i in range(q)], dtype=np.float64)
    s = np.zeros((q + 1, q + 1), dtype=np.float64)
    s[0, 1:] = 1.0
    s[1:, 0] = -1.0
    s[1:, 1:] = jac
    return np.eye(q + 1) + s


def hadamard(d: int) -> np.ndarray:
    if d & (d - 1) == 0:
        return sylvester_hadamard(d)
    if d == 1536:
        return np.kron(paley_hadamard(11), sylvester_hadamard(128))
    raise ValueError(f"no Hadamard construction for d={d}")


def rotation_matrix(D: np.ndarray) -> np.ndarray:
    """Pi = H diag(D) / sqrt(d) as a dense fp64 matrix."""
    D = np.asarray(D, dtype=np.float64)
    d = D.shape[0]
    return hadamard(d) * D[None, :] / np.sqrt(d)


def haar_rotation(G: np.ndarray) -> np.ndarray:
    """A Haar-distributed orthogonal matrix from a square matrix G of i.i.d.
    N(0,1) entries: the Q factor of G = QR with every diagonal entry of R made
    positive (Q's columns scaled by sign(R_kk)); without that step the law of Q
    depends on the QR routine's sign convention and is not Haar.  Source: the
    shared random rotation of the theory ("Google presenta TurboQuant ...",
    "La mecanica geometrica de TurboQuant"; "FibQuant ...", section 2.1, Haar
    rotation)."""
    G = np.asarray(G, dtype=np.float64)
    q, r = np.linalg.qr(G)
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s[None, :]


def apply_rope(x: np.ndarray, cos: np.ndarray, sin: np.ndarray, pos) -> np.ndarray:
    """Rotate-half RoPE: for i < d/2,
    x'_i = x_i cos - x_{i+d/2} sin,  x'_{i+d/2} = x_{i+d/2} cos + x_i sin,
    with cos/sin taken at the (broadcastable) positions ``pos``."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    c = np.asarray(cos, dtype=np.float64)[pos]
    s = np.asarray(sin, dtype=np.float64)[pos]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
