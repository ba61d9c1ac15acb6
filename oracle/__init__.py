"""CPU oracle for the rotated-codebook KV codec -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 numpy restatement of what the hot path computes, written
from the pages' descriptions of TurboQuant (normalize -> shared random rotation
-> per-coordinate Lloyd-Max codebook for the Beta coordinate law -> 1-bit QJL
sketch of the residual -> inner-product estimator) and of compressed-domain
attention.  Each function cites the passage it follows.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  It shares no code with the CUDA
library (``rotated_codebook_kv_tq_b200``); the only module both sides use is
``rotated_codebook_kv_tq_b200.synth``, which draws the seeded inputs and holds
none of the method's arithmetic.

Modules: ``codebook`` (scalar Lloyd-Max codes), ``rotation`` (randomized
Walsh-Hadamard and dense Haar rotations, RoPE), ``codec`` (TurboQuant_mse /
_prod encode, layout, dequantize), ``attention`` (decode and bidirectional
attention over the compressed cache), ``scan`` (vector-search scores and
top-k), ``split`` (outlier-channel mixed precision), ``fibquant`` (FibQuant
k = 2 pair codes).

Parity status: every function here is pinned by a ``-m "not gpu"`` test against
closed forms, textbook values, invariants, Monte-Carlo laws or brute force,
except the two items listed as "parity unpinned" in ``codec.py``'s header
(the bit layout, which is this library's own specification, and the RoPE
base/convention, which the pages do not fix); the FibQuant block layout is
likewise this library's specification, checked against plain loops.
"""
