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


def test_every_call_has_a_ctypes_signature(L):
    # without argtypes, ctypes cannot pass a Python float as a C float
    for n in native.EXPORTS:
        if n != "tq_last_error":
            assert getattr(L, n).argtypes is not None, n


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


def test_split_channels_matches_oracle(L):
    """tq_split_channels (host C) against the oracle's choice of outlier
    channels, ties included."""
    from oracle import split as osp
    rng = np.random.default_rng(4)
    score = rng.lognormal(0.0, 1.0, size=(8, 2, 128)).astype(np.float32)
    score[0, 0, :10] = 7.0          # ties straddling the cut
    score[1, 1] = 1.0               # all equal
    got = native.split_channels(score)
    np.testing.assert_array_equal(got.astype(np.int64), osp.outlier_channels(score))
    assert got.dtype == np.int16 and got.shape == score.shape
    bad = score.copy()
    bad[2, 0, 5] = np.nan
    with pytest.raises(native.TqError):
        native.split_channels(bad)
    assert L.tq_split_channels(score.ctypes.data, 1, 7, got.ctypes.data) == native.TQ_ERR_INVALID_ARG


def test_split_calls_validate_before_device_work(L):
    sz = ctypes.c_size_t(0)
    assert L.tq_attention_split_workspace(None, 1, 8, 0, ctypes.byref(sz)) == native.TQ_ERR_INVALID_ARG
    empty = native.SplitDesc(None, None, None)
    cd = native.CacheDesc(None, None, None, None, 1, 1, 32)
    assert L.tq_quantize_kv_split(ctypes.byref(empty), None, None, 0, 1, 1, 1, 0, 0, 0, None, None,
                                  0, ctypes.byref(cd), ctypes.byref(cd), 0, None,
                                  None) == native.TQ_ERR_INVALID_ARG
    assert L.tq_dequantize_split(ctypes.byref(empty), ctypes.byref(cd), ctypes.byref(cd), 0, 0, 1,
                                 None, None) == native.TQ_ERR_INVALID_ARG
    assert b"split" in L.tq_last_error()


@pytest.mark.parametrize("d,bits", [(64, 1), (64, 3), (128, 2), (128, 4), (128, 6)])
def test_fq_host_codebook_matches_oracle(L, d, bits):
    """tq_fq_build_codebook (host C++) against the oracle's FibQuant k = 2 code:
    same start, quadrature, Lloyd steps and restart rule, written separately."""
    from oracle import fibquant as ofq
    c, mse = native.fq_build_codebook(d, bits)
    ref = ofq.pair_codebook(d, bits)
    np.testing.assert_allclose(c.astype(np.float64), ref.centroids, rtol=0, atol=1e-7)
    assert abs(mse / ref.mse_per_pair - 1) < 1e-9


def test_decode_step_host_validates_before_device_work(L):
    cd = native.CacheDesc(None, None, None, None, 1, 1, 32)
    f = L.tq_decode_step_host
    # no codec
    assert f(None, 1, 2, 16, native.TQ_BF16, native.TQ_BF16, 1, 1, 1, ctypes.byref(cd), 4, 0.1, None,
             None, 0, 3, 64, 5, 6, None) == native.TQ_ERR_INVALID_ARG
    assert b"codec" in L.tq_last_error()
    # a NULL host or device buffer is rejected before the codec is read
    fake = ctypes.create_string_buffer(256)
    for bufs in [(None, 2, 5, 6), (1, None, 5, 6), (1, 2, None, 6), (1, 2, 5, None)]:
        ih, idv, od, oh = bufs
        assert f(ctypes.addressof(fake), ih, idv, 16, native.TQ_BF16, native.TQ_BF16, 1, 1, 1,
                 ctypes.byref(cd), 4, 0.1, None, None, 0, 3, 64, od, oh, None) == native.TQ_ERR_INVALID_ARG
        assert b"NULL buffer" in L.tq_last_error()


def test_fq_codec_is_host_only_and_validates(L):
    signs = synth.rotation_signs(128, 0)
    c = native.FqCodec(128, 4, 3, signs)
    ck, cv = c.codebooks()
    ref_k, _ = native.fq_build_codebook(128, 4)
    assert np.array_equal(ck, ref_k) and cv.shape == (8, 2)
    assert native.fq_cache_bytes(c, 1, 2, 64) == [2 * 64 * 4 * 8, 2 * 64 * 4, 2 * 2 * 3 * 64 * 4, 2 * 64 * 2]
    c.close()
    for d, bk, bv, code in [(96, 2, 2, native.TQ_ERR_UNSUPPORTED), (128, 0, 2, native.TQ_ERR_UNSUPPORTED),
                            (128, 2, 7, native.TQ_ERR_UNSUPPORTED)]:
        with pytest.raises(native.TqError) as e:
            native.FqCodec(d, bk, bv, synth.rotation_signs(d, 0))
        assert e.value.code == code
    bad = signs.copy()
    bad[5] = 0
    with pytest.raises(native.TqError):
        native.FqCodec(128, 2, 2, bad)


@pytest.mark.parametrize("d", [8, 64, 128])
def test_haar_rotation_matches_oracle(L, d):
    """tq_haar_rotation (host Householder QR) against the oracle's sign-fixed
    numpy QR of the same Gaussian matrix."""
    from oracle.rotation import haar_rotation
    G = synth.haar_gaussian(d, 4)
    got = native.haar_rotation(G).astype(np.float64)
    ref = haar_rotation(G)
    assert np.max(np.abs(got - ref)) < 1e-6
    assert np.max(np.abs(got @ got.T - np.eye(d))) < 1e-5


def test_dense_rotation_validation(L):
    bad = np.eye(64, dtype=np.float32)
    bad[3, 3] = 0.5
    S = synth.qjl_matrix_bf16(64, 0)
    desc = native.CodecDesc(64, 3, 1, 3, None, S.ctypes.data, bad.ctypes.data)
    h = ctypes.c_void_p()
    assert L.tq_codec_create(ctypes.byref(desc), ctypes.byref(h)) == native.TQ_ERR_INVALID_ARG
    assert b"orthogonal" in L.tq_last_error()
    big = np.eye(1536, dtype=np.float32)
    desc = native.CodecDesc(1536, 3, 1, 3, None, None, big.ctypes.data)
    assert L.tq_codec_create(ctypes.byref(desc), ctypes.byref(h)) == native.TQ_ERR_UNSUPPORTED
    g = synth.haar_gaussian(16, 0)
    g[2, 2] = np.nan
    with pytest.raises(native.TqError):
        native.haar_rotation(g)
