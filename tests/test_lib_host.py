"""CPU tests of the C-ABI library: it loads, exports every function declared in
include/tq.h, its host Lloyd-Max solver (incomplete-Beta method) agrees with
the oracle's (quadrature method), and argument validation rejects bad input
before any device work."""
import ctypes
import os
import re

import numpy as np
import pytest

from rotated_codebook_kv_tq_b200 import native, synth
from oracle import codebook as ocb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from rotated_codebook_kv_tq_b200.build import build
    build()
    return native.lib()


def declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\s*\**\s*(tq_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(native.EXPORTS)


@pytest.mark.parametrize("d,bits", [(64, 2), (64, 3), (128, 1), (128, 2), (128, 3), (128, 4)])
def test_host_codebook_matches_oracle(L, d, bits):
    c, t, mse = native.build_codebook(d, bits)
    ref = ocb.codebook(d, bits)
    assert np.array_equal(c, ref.centroids32)
    assert np.array_equal(t, ref.thresholds32)
    assert abs(mse - ref.mse_per_coord) < 1e-10 * ref.mse_per_coord + 1e-16


def test_host_codebook_fp64_agreement(L):
    # the fp64 fixed points of the two independent solvers agree closely
    for d, bits in [(128, 3), (1536, 3), (1536, 4)]:
        c, _, mse = native.build_codebook(d, bits)
        ref = ocb.codebook(d, bits)
        assert np.max(np.abs(c.astype(np.float64) - ref.centroids)) < 6e-8 * np.max(ref.centroids)
        assert abs(mse - ref.mse_per_coord) < 1e-9 * ref.mse_per_coord


def test_codebook_rejects_bad_args(L):
    c = np.zeros(16, np.float32)
    t = np.zeros(15, np.float32)
    assert L.tq_build_codebook(2, 3, c.ctypes.data, t.ctypes.data, None) == native.TQ_ERR_INVALID_ARG
    assert L.tq_build_codebook(128, 0, c.ctypes.data, t.ctypes.data, None) == native.TQ_ERR_INVALID_ARG
    assert L.tq_build_codebook(128, 3, None, t.ctypes.data, None) == native.TQ_ERR_INVALID_ARG
    assert b"codebook" in L.tq_last_error()


def test_codec_create_validation(L):
    signs = synth.rotation_signs(128, 0)
    S = synth.qjl_matrix_bf16(128, 0)
    for d, bk, q, bv, s, code in [
        (96, 3, 1, 3, S, native.TQ_ERR_UNSUPPORTED),
        (128, 1, 1, 3, S, native.TQ_ERR_UNSUPPORTED),     # no MSE bit left
        (128, 6, 1, 3, S, native.TQ_ERR_UNSUPPORTED),
        (128, 3, 1, 5, S, native.TQ_ERR_UNSUPPORTED),
        (128, 3, 1, 3, None, native.TQ_ERR_INVALID_ARG),  # QJL needs S
    ]:
        desc = native.CodecDesc(d, bk, q, bv, signs.ctypes.data,
                                None if s is None else s.ctypes.data)
        h = ctypes.c_void_p()
        assert L.tq_codec_create(ctypes.byref(desc), ctypes.byref(h)) == code
        assert h.value is None
    bad = signs.copy()
    bad[3] = 0
    desc = native.CodecDesc(128, 3, 1, 3, bad.ctypes.data, S.ctypes.data)
    h = ctypes.c_void_p()
    assert L.tq_codec_create(ctypes.byref(desc), ctypes.byref(h)) == native.TQ_ERR_INVALID_ARG


def test_cache_bytes_formula(L):
    # bytes per (token, head) of the proposed layouts: 68 + 66 (4-bit), 36 + 34 (2-bit)
    from oracle import codec as oc
    c = oc.make_codec(128, 4, True, 4, synth.rotation_signs(128, 0), synth.qjl_matrix_bf16(128, 0))
    kb, vb = oc.bytes_per_row(c)
    assert kb + vb == 134
