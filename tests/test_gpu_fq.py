"""GPU-vs-oracle parity of the FibQuant k = 2 codec ("FibQuant ...", sections
2.1-2.3) through the C ABI: quantize, dequantize and decode.

Codes: every block's code equals the oracle's nearest codeword except blocks
whose rotated pair lies within 1e-5 (unit-variance scale, sqrt(d) times the
distance to the bisector of the two nearest codewords) of a cell boundary;
such mismatches may be at most 1e-4 of the blocks.  nu within one fp16 ulp.
Dequantized rows within 1e-3 relative and decode outputs within 2e-3 max-abs
after the per-channel scale, on the same codes."""
import math

import numpy as np
import pytest
import torch

from oracle import fibquant as ofq
from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


LLAMA = synth.WORKLOADS["llama_decode"]
ESM = synth.WORKLOADS["esm_prefill"]
CASES = {
    # name: (workload, bits per block of keys and values, quantize segments, decode lengths, splits)
    "llama_2bit": (LLAMA.scaled(B=2, Hq=8, Hkv=2, T=700), (4, 4), [(0, 700)], [700, 311], 4),
    "llama_appends_1.5bit": (LLAMA.scaled(B=1, Hq=8, Hkv=2, T=300), (3, 3), [(0, 250), (250, 1), (251, 49)],
                             [300], 0),
    "llama_3bit_g8": (LLAMA.scaled(B=1, Hq=16, Hkv=2, T=400, dtype="fp32"), (6, 6), [(0, 400)], [400], 5),
    "llama_half_bit": (LLAMA.scaled(B=1, Hq=4, Hkv=4, T=200), (1, 2), [(0, 200)], [200], 2),
    "esm_d64": (ESM.scaled(B=2, Hq=3, Hkv=3, T=150), (4, 3), [(0, 150)], [150, 97], 3),
}


def _setup(case):
    w, (bk, bv), segments, lens, splits = CASES[case]
    D = synth.rotation_signs(w.d, w.seed + 7)
    oc = ofq.make_codec(w.d, bk, bv, D)
    nc = native.FqCodec(w.d, bk, bv, D)
    K, V = synth.kv_inputs(w)
    return w, oc, nc, K, V, segments, lens, splits, (w.T + 31) // 32 * 32


def _in_window(u, cb):
    """Blocks whose pair lies within 1e-5 (sqrt(d) times the distance to the
    bisector of its two nearest codewords) of a cell boundary."""
    d = u.shape[-1]
    p = u.astype(np.float32).astype(np.float64).reshape(-1, 2)
    c = cb.astype(np.float64)
    d2 = np.sum((p[:, None, :] - c[None, :, :]) ** 2, axis=-1)
    o = np.argsort(d2, axis=1, kind="stable")
    i1, i2 = o[:, 0], o[:, 1]
    r = np.arange(len(p))
    sep = np.linalg.norm(c[i1] - c[i2], axis=-1)
    dist = (d2[r, i2] - d2[r, i1]) / (2 * np.maximum(sep, 1e-30))
    return (math.sqrt(d) * dist < 1e-5).reshape(u.shape[0], d // 2)


def _window(u, idx_gpu, idx_ref, cb):
    """sqrt(d) * distance of each mismatching pair to the bisector of the two
    codewords involved (fp64 on the fp32 pair)."""
    d = u.shape[-1]
    p = u.astype(np.float32).astype(np.float64).reshape(u.shape[0], d // 2, 2)
    c = cb.astype(np.float64)
    a, b = c[idx_gpu], c[idx_ref]
    da = np.sum((p - a) ** 2, axis=-1)
    db = np.sum((p - b) ** 2, axis=-1)
    sep = np.linalg.norm(a - b, axis=-1)
    return math.sqrt(d) * np.abs(da - db) / (2 * np.maximum(sep, 1e-30))


@pytest.mark.parametrize("case", list(CASES))
def test_fq_quantize_parity(case):
    w, oc, nc, K, V, segments, _, _, rows_cap = _setup(case)
    K64, V64 = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
    rope = synth.rope_for(w, rows_cap)
    ocache = ofq.empty_cache(oc, w.B, w.Hkv, rows_cap)
    ncache = native.fq_alloc_cache(nc, w.B, w.Hkv, rows_cap)
    kd, vd = tl.to_device(K, w.dtype), tl.to_device(V, w.dtype)
    rd = tl.rope_device(rope)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    encs = []
    for row0, T in segments:
        sl = slice(row0, row0 + T)
        diag = ofq.quantize_into(ocache, K64[:, :, sl], V64[:, :, sl], oc, rope=rope, pos0=row0,
                                 row0=row0)
        native.fq_quantize_kv(nc, kd[:, :, sl], vd[:, :, sl], ncache, row0=row0, rope=rd, pos0=row0,
                              status=status)
        encs.append((row0, T, diag))
    torch.cuda.synchronize()
    gpu = tl.download_cache(ncache)
    mism = blocks = inwin = 0
    for row0, T, diag in encs:
        i = 0
        for b in range(w.B):
            for h in range(w.Hkv):
                ek, ev = diag["k"][i], diag["v"][i]
                i += 1
                ik, nk, iv, nv = ofq.cache_rows(gpu, oc, b, h, row0 + T)
                for got, ref, nu_got, enc, cb in ((ik[row0:], ek["idx"], nk[row0:], ek, oc.cb_k),
                                                  (iv[row0:], ev["idx"], nv[row0:], ev, oc.cb_v)):
                    bad = got != ref
                    if bad.any():
                        win = _window(enc["u"], got, ref, cb.centroids32)
                        assert np.all(win[bad] < 1e-5), (case, np.max(win[bad]))
                    mism += int(bad.sum())
                    blocks += bad.size
                    inwin += int(_in_window(enc["u"], cb.centroids32).sum())
                    assert np.all(tl.fp16_close(nu_got, enc["nu16"]))
    tl.MISMATCH_REPORT.append(dict(test=f"fq_quantize[{case}]", code_mism=mism, sign_mism=0,
                                   code_window=inwin, sign_window=0, coords=blocks,
                                   fraction=mism / blocks))
    assert mism <= 1e-4 * blocks
    assert int(status.item()) == 0


def _upload(ocache, nc, w):
    c = native.fq_alloc_cache(nc, w.B, w.Hkv, ocache["rows_cap"])
    c.kcode.copy_(torch.from_numpy(ocache["kcode"]))
    c.kscale.copy_(torch.from_numpy(ocache["kscale"]))
    c.vcode.copy_(torch.from_numpy(ocache["vcode"].view(np.int32)))
    c.vnorm.copy_(torch.from_numpy(ocache["vnorm"]))
    return c


def _oracle_cache(w, oc, K, V, rows_cap):
    rope = synth.rope_for(w, rows_cap)
    ocache = ofq.empty_cache(oc, w.B, w.Hkv, rows_cap)
    ofq.quantize_into(ocache, synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype), oc, rope=rope)
    return ocache, rope


@pytest.mark.parametrize("case", list(CASES))
def test_fq_dequantize_parity(case):
    w, oc, nc, K, V, _, _, _, rows_cap = _setup(case)
    ocache, _ = _oracle_cache(w, oc, K, V, rows_cap)
    cache = _upload(ocache, nc, w)
    row0, rows = 3, w.T - 7
    for which in (0, 1):
        out = torch.full((w.B, w.Hkv, rows, w.d), float("nan"), device="cuda")
        native.fq_dequantize(nc, cache, which, row0, rows, out)
        got = out.cpu().numpy().astype(np.float64)
        cb = oc.cb_k if which == 0 else oc.cb_v
        for b in range(w.B):
            for h in range(w.Hkv):
                ik, nk, iv, nv = ofq.cache_rows(ocache, oc, b, h, row0 + rows)
                idx, nu = (ik, nk) if which == 0 else (iv, nv)
                ref = ofq.decode_rows(idx[row0:], nu[row0:], oc, cb)
                err = np.linalg.norm(got[b, h] - ref, axis=1) / np.linalg.norm(ref, axis=1)
                assert np.max(err) <= 1e-3, (which, b, h, np.max(err))


@pytest.mark.parametrize("case", list(CASES))
def test_fq_decode_parity(case):
    w, oc, nc, K, V, _, lens, splits, rows_cap = _setup(case)
    ocache, rope = _oracle_cache(w, oc, K, V, rows_cap)
    cache = _upload(ocache, nc, w)
    q = synth.query_inputs(w, Lq=1)[:, :, 0]
    scale = 1.0 / math.sqrt(w.d)
    ref = ofq.decode(synth.as_float64(q, w.dtype), ocache, oc, lens, scale, rope=rope)
    out = torch.full((w.B, w.Hq, w.d), float("nan"), device="cuda")
    ws = torch.empty(native.fq_attention_workspace(nc, w.B, w.Hq, splits), dtype=torch.uint8,
                     device="cuda")
    native.fq_attention_decode(nc, tl.to_device(np.ascontiguousarray(q), w.dtype), cache, max(lens),
                               scale, out, ws, seq_lens=torch.tensor(lens, dtype=torch.int32,
                                                                     device="cuda"),
                               rope=tl.rope_device(rope), num_splits=splits)
    got = out.cpu().numpy().astype(np.float64)
    vscale = tl.channel_scale_of_values(w)
    for b in range(w.B):
        for h in range(w.Hq):
            err = np.abs(got[b, h] - ref[b, h]) / vscale[h // w.G]
            assert np.max(err) <= 2e-3, (b, h, np.max(err))


def test_fq_bad_rows_and_arguments():
    w = LLAMA.scaled(B=1, Hq=2, Hkv=1, T=40, dtype="fp32")
    nc = native.FqCodec(128, 4, 4, synth.rotation_signs(128, 1))
    K = torch.randn((1, 1, 40, 128), device="cuda")
    V = torch.randn((1, 1, 40, 128), device="cuda")
    K[0, 0, 5, 7] = float("nan")
    V[0, 0, 9, 0] = float("inf")
    cache = native.fq_alloc_cache(nc, 1, 1, 64)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.fq_quantize_kv(nc, K, V, cache, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 2
    assert float(cache.kscale[0, 0, 5, 0]) == 0.0 and float(cache.vnorm[0, 0, 9]) == 0.0
    out = torch.empty((1, 1, 40, 128), device="cuda")
    native.fq_dequantize(nc, cache, 0, 0, 40, out)
    assert torch.all(out[0, 0, 5] == 0)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(native.TqError) as e:
        native.fq_attention_decode(nc, torch.zeros((1, 2, 128), device="cuda"), cache, 40, 0.1,
                                   torch.empty((1, 2, 128), device="cuda"), small, num_splits=2)
    assert e.value.code == native.TQ_ERR_WORKSPACE
    with pytest.raises(native.TqError):
        native.fq_quantize_kv(nc, torch.zeros((1, 1, 70, 128), device="cuda"),
                              torch.zeros((1, 1, 70, 128), device="cuda"), cache)
