"""GPU-vs-oracle parity of codecs on a dense Haar rotation (the theory's
shared random rotation: "Google presenta TurboQuant ...", "La mecanica
geometrica de TurboQuant"; "FibQuant ...", section 2.1) through the C ABI.

Each side factorises the same Gaussian matrix itself (oracle: numpy QR in
fp64; library: tq_haar_rotation, Householder in fp64, stored fp32).  The
tolerances are those of the Walsh-Hadamard codecs: codes bit-exact outside
the 1e-5 boundary window, dequantized rows within 1e-3, logits within
1e-3 RMS, outputs within 2e-3 after the per-channel scale."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import codec as oc
from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


LLAMA = synth.WORKLOADS["llama_decode"]
ESM = synth.WORKLOADS["esm_prefill"]

QUANT_CASES = {
    "llama_appends": (LLAMA.scaled(T=138), [(0, 100), (100, 1), (101, 37)]),
    # >= 256 token groups: the tile kernel with the rotation on the tensor
    # cores (with and without the sketch; "simt" takes the CUDA-core kernels)
    "llama_tc_sketch": (LLAMA.scaled(T=1100), [(0, 1037), (1037, 63)]),
    "llama_large_mse_fp32": (LLAMA.scaled(T=1100, qjl_k=False, bits_k=3, dtype="fp32"), [(0, 1100)]),
    "esm_d64": (ESM.scaled(B=2, Hq=3, Hkv=3, T=100), [(0, 100)]),
    # >= 256 token groups with d = 64, starting mid-group (row 45)
    "esm_large_d64": (ESM.scaled(B=4, Hq=20, Hkv=20, T=300), [(0, 45), (45, 255)]),
}


@pytest.mark.parametrize("impl", ["default", "simt"])
@pytest.mark.parametrize("case", list(QUANT_CASES))
def test_haar_quantize_parity(case, impl, monkeypatch):
    if impl == "simt":
        monkeypatch.setenv("TQ_QUANT_IMPL", "simt")
    else:
        monkeypatch.delenv("TQ_QUANT_IMPL", raising=False)
    w, segments = QUANT_CASES[case]
    ocodec, ncodec = tl.codecs(w, haar=True)
    K, V = synth.kv_inputs(w)
    K64, V64 = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
    rows_cap = (w.T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    ncache = native.alloc_cache(ncodec, w.B, w.Hkv, rows_cap)
    kd, vd, rd = tl.to_device(K, w.dtype), tl.to_device(V, w.dtype), tl.rope_device(rope)
    stats = tl.new_stats()
    for row0, T in segments:
        sl = slice(row0, row0 + T)
        diag = oc.quantize_into(ocache, K64[:, :, sl], V64[:, :, sl], ocodec, rope=rope, pos0=row0,
                                row0=row0)
        native.quantize_kv(ncodec, kd[:, :, sl], vd[:, :, sl], ncache, row0=row0, rope=rd, pos0=row0)
        torch.cuda.synchronize()
        gpu = tl.download_cache(ncache)
        i = 0
        for b in range(w.B):
            for h in range(w.Hkv):
                tl.compare_rows(gpu, ocache, ocodec, b, h, np.arange(row0, row0 + T), diag["k"][i],
                                diag["v"][i], stats)
                i += 1
    tl.assert_mismatch_budget(stats)


@pytest.mark.parametrize("case", ["llama_appends", "esm_d64"])
def test_haar_dequantize_parity(case):
    w, _ = QUANT_CASES[case]
    ocodec, ncodec = tl.codecs(w, haar=True)
    K, V = synth.kv_inputs(w)
    rows_cap = (w.T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    oc.quantize_into(ocache, synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype), ocodec,
                     rope=rope)
    ncache = tl.upload_cache(ocache, ncodec, w.B, w.Hkv)
    for which in (0, 1):
        out = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.float32, device="cuda")
        native.dequantize(ncodec, ncache, which, 0, w.T, out)
        got = out.cpu().numpy().astype(np.float64)
        for b in range(w.B):
            for h in range(w.Hkv):
                ik, sg, nk, rk, iv, nv = oc.cache_rows(ocache, ocodec, b, h, w.T)
                ref = (oc.dequant_keys(ik, sg, nk, rk, ocodec) if which == 0
                       else oc.dequant_values(iv, nv, ocodec))
                err = np.linalg.norm(got[b, h] - ref, axis=1) / np.linalg.norm(ref, axis=1)
                assert np.max(err) <= 1e-3, (which, b, h, np.max(err))


DECODE_CASES = {
    "llama_g4": (LLAMA.scaled(B=2, Hq=8, Hkv=2, T=1000), [1000, 411], 7),
    "llama_mse_keys": (LLAMA.scaled(B=1, Hq=8, Hkv=2, T=700, qjl_k=False, bits_k=4), None, 3),
    "esm_d64": (ESM.scaled(B=2, Hq=3, Hkv=3, T=300, Lq=1), None, 4),
}


@pytest.mark.parametrize("impl", ["default", "simt"])
@pytest.mark.parametrize("case", list(DECODE_CASES))
def test_haar_decode_parity(case, impl, monkeypatch):
    if impl == "simt":
        monkeypatch.setenv("TQ_DECODE_IMPL", "simt")
    else:
        monkeypatch.delenv("TQ_DECODE_IMPL", raising=False)
    w, lens, splits = DECODE_CASES[case]
    ocodec, ncodec = tl.codecs(w, haar=True)
    K, V = synth.kv_inputs(w)
    rows_cap = (w.T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    oc.quantize_into(ocache, synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype), ocodec,
                     rope=rope)
    ncache = tl.upload_cache(ocache, ncodec, w.B, w.Hkv)
    q = synth.query_inputs(w, Lq=1)[:, :, 0]
    scale = 1.0 / math.sqrt(w.d)
    lens = [w.T] * w.B if lens is None else lens
    ref, ref_logits = oatt.decode(synth.as_float64(q, w.dtype), ocache, ocodec, lens, scale,
                                  rope=rope, want_logits=True)
    ws = torch.empty(native.attention_workspace(ncodec, w.B, w.Hq, splits), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    logits = torch.full((w.B, w.Hq, w.T), float("nan"), dtype=torch.float32, device="cuda")
    native.attention_logits(ncodec, tl.to_device(np.ascontiguousarray(q), w.dtype), ncache, w.T,
                            scale, out, logits, ws,
                            seq_lens=torch.tensor(lens, dtype=torch.int32, device="cuda"),
                            rope=tl.rope_device(rope), num_splits=splits)
    got, gl = out.cpu().numpy().astype(np.float64), logits.cpu().numpy()
    vscale = tl.channel_scale_of_values(w)
    for b in range(w.B):
        for h in range(w.Hq):
            lr = ref_logits[(b, h)]
            rms = math.sqrt(np.mean(lr * lr))
            assert np.max(np.abs(gl[b, h, :lens[b]] - lr)) <= 1e-3 * rms
            err = np.abs(got[b, h] - ref[b, h]) / vscale[h // w.G]
            assert np.max(err) <= 2e-3, (b, h, np.max(err))


def test_haar_codec_rejected_where_not_built():
    w = ESM.scaled(B=1, Hq=2, Hkv=2, T=64, Lq=64)
    _, ncodec = tl.codecs(w, haar=True)
    cache = native.alloc_cache(ncodec, 1, 2, 64)
    q = torch.zeros((1, 2, 64, 64), device="cuda")
    out = torch.empty((1, 2, 64, 64), device="cuda")
    ws = torch.empty(native.attention_bidir_workspace(ncodec, 1, 2, 64), dtype=torch.uint8,
                     device="cuda")
    with pytest.raises(native.TqError) as e:
        native.attention_bidir(ncodec, q, cache, 64, 0.125, out, ws)
    assert e.value.code == native.TQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("T", [40, 1100])
def test_haar_quantize_nonfinite_rows(T):
    """Rows with a NaN or Inf are stored as zero rows and counted once per row,
    in the warp-per-group kernels (T = 40) and the tensor-core rotation kernel
    (T = 1100, >= 256 token groups)."""
    w = LLAMA.scaled(B=1, Hq=8, Hkv=8, T=T, dtype="fp32")
    ocodec, ncodec = tl.codecs(w, haar=True)
    K = torch.randn((1, 8, T, 128), device="cuda")
    V = torch.randn((1, 8, T, 128), device="cuda")
    K[0, 3, 17, 5] = float("nan")
    V[0, 6, T - 1, 100] = float("inf")
    rows_cap = (T + 31) // 32 * 32
    cache = native.alloc_cache(ncodec, 1, 8, rows_cap)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.quantize_kv(ncodec, K, V, cache, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 2
    assert float(cache.kscale[0, 3, 17, 0]) == 0.0 and float(cache.vnorm[0, 6, T - 1]) == 0.0
    # the zero rows decode to zero vectors; a finite row next to them is intact
    out = torch.empty((1, 8, T, 128), device="cuda")
    native.dequantize(ncodec, cache, 0, 0, T, out)
    assert torch.all(out[0, 3, 17] == 0)
    ref = K[0, 3, 18].double().cpu().numpy()
    got = out[0, 3, 18].double().cpu().numpy()
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 0.5
