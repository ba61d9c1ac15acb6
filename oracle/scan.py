"""Inner-product scan with top-k over a TurboQuant_prod-encoded database (oracle side).

Sources: "Google presenta TurboQuant..." (7minutos.es), "Velocidad y eficiencia
de indexacion": nearest-neighbour search over data-oblivious TurboQuant codes
(indexing needs no training); "Eliminacion del sesgo interno del producto": the
prod estimator of <q, x> is unbiased.  "TurboQuant: Jak rozwiazac ..."
(securhub.pl), "Zaskakujace przyspieszenie baz wektorowych": the same use for
vector databases.

Readings: database rows are encoded exactly like keys (TURBOQUANT_prod, no
RoPE); the score of row j for query q is the estimator
    s_j = nu_j ( <Pi q, c[idx_j]> + sqrt(pi/2)/m rho_j <S Pi q, 2 sigma_j - 1> ),
and the top-k list is ordered by (-score, index).
"""
from __future__ import annotations

import numpy as np

from .attention import estimator_logits
from .codec import Codec, unpack_keys


def scores(q: np.ndarray, kcode: np.ndarray, kscale: np.ndarray, codec: Codec) -> np.ndarray:
    """q [nq, d] fp64, kcode [n, planes, d/8], kscale [n, 2] -> scores [nq, n]."""
    ik, sg, nk, rk = unpack_keys(kcode, kscale, codec)
    return estimator_logits(np.asarray(q, np.float64), (ik, sg, nk, rk, None, None), codec, 1.0)


def topk(s: np.ndarray, k: int):
    """Per query: indices and scores of the k largest, ties to the lower index."""
    n = s.shape[1]
    idx = np.empty((s.shape[0], k), np.int64)
    val = np.empty((s.shape[0], k), np.float64)
    for i in range(s.shape[0]):
        order = np.lexsort((np.arange(n), -s[i]))[:k]
        idx[i] = order
        val[i] = s[i, order]
    return idx, val
