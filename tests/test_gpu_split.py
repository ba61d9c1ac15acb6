"""GPU-vs-oracle parity of the outlier-channel split ("Google presenta
TurboQuant ...", "Desempeno teorico y empirico": outlier channels at more bits
than the rest, 2.5 and 3.5 bits per channel) through the C ABI: quantize into
both caches, dequantize back onto the channels, decode over both caches.

The channel lists are the oracle's choice of outlier channels (largest mean
square per KV head in the prefill, keys and values separately).  Codes follow
the boundary-window rule of the other parity tests; dequantized rows are within
1e-3 relative and decode outputs within 2e-3 max-abs after the per-channel
scale, on the same codes."""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from oracle import split as osp
from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


# (hi bits_k, hi qjl, hi bits_v), (lo ...): 2.5 and 3.5 bits per channel
RATES = {
    "r2.5": ((3, True, 3), (2, True, 2)),
    "r3.5": ((4, True, 4), (3, True, 3)),
    "r2.5_mse": ((3, False, 3), (2, False, 2)),
    "r1.5_mse": ((2, False, 2), (1, False, 1)),
}

LLAMA = synth.WORKLOADS["llama_decode"]
CASES = {
    # name: (workload, rate, quantize segments, decode lengths, splits)
    "llama_g4": (LLAMA.scaled(B=2, Hq=8, Hkv=2, T=700), "r2.5", [(0, 700)], [700, 333], 4),
    "llama_appends": (LLAMA.scaled(B=1, Hq=8, Hkv=2, T=300), "r3.5", [(0, 250), (250, 1), (251, 49)],
                      [300], 0),
    "llama_mse_g2": (LLAMA.scaled(B=1, Hq=4, Hkv=2, T=400), "r2.5_mse", [(0, 400)], [400], 5),
    # key codebooks of at most 2 bits without QJL, GQA group 1 (table path)
    "llama_mse_lin_g1": (LLAMA.scaled(B=2, Hq=2, Hkv=2, T=500), "r1.5_mse", [(0, 500)], [500, 129], 3),
    # >= 256 token groups per call: the tensor-core sketch kernel with the map
    "llama_tc_sketch": (LLAMA.scaled(B=2, Hq=16, Hkv=8, T=600), "r2.5", [(0, 600)], [600, 411], 0),
    # halves of 128 channels, GQA group 8, fp32 inputs
    "d256_g8": (LLAMA.scaled(B=1, Hq=8, Hkv=1, d=256, T=300, dtype="fp32"), "r2.5", [(0, 300)],
                [300], 3),
}


def _codecs(w, rate, seed):
    out = []
    for i, (bk, qjl, bv) in enumerate(RATES[rate]):
        ds = w.d // 2
        D = synth.rotation_signs(ds, seed + 100 * (i + 1))
        S = synth.qjl_matrix_bf16(ds, seed + 100 * (i + 1)) if qjl else None
        out.append((oc.make_codec(ds, bk, qjl, bv, D, S), native.Codec(ds, bk, qjl, bv, D, S)))
    return out


def _setup(case):
    w, rate, segments, lens, splits = CASES[case]
    (ohi, nhi), (olo, nlo) = _codecs(w, rate, w.seed)
    K, V = synth.kv_inputs(w)
    K64, V64 = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
    score = np.stack([np.mean(K64 ** 2, axis=(0, 2)), np.mean(V64 ** 2, axis=(0, 2))], axis=1)
    chan = osp.outlier_channels(score)                                   # [Hkv, 2, d]
    sc = osp.make_split_codec(ohi, olo, chan)
    ns = native.Split(nhi, nlo, torch.from_numpy(chan.astype(np.int16)).cuda())
    rows_cap = (w.T + 31) // 32 * 32
    return w, sc, ns, K, V, K64, V64, segments, lens, splits, rows_cap


@pytest.mark.parametrize("impl", ["default", "simt"])
@pytest.mark.parametrize("case", list(CASES))
def test_split_quantize_parity(case, impl, monkeypatch):
    if impl == "simt":
        monkeypatch.setenv("TQ_QUANT_IMPL", "simt")
    else:
        monkeypatch.delenv("TQ_QUANT_IMPL", raising=False)
    w, sc, ns, K, V, K64, V64, segments, _, _, rows_cap = _setup(case)
    rope = synth.rope_for(w, rows_cap)
    ocaches = osp.empty_caches(sc, w.B, w.Hkv, rows_cap)
    nhi = native.alloc_cache(ns.hi, w.B, w.Hkv, rows_cap)
    nlo = native.alloc_cache(ns.lo, w.B, w.Hkv, rows_cap)
    kd, vd = tl.to_device(K, w.dtype), tl.to_device(V, w.dtype)
    rd = tl.rope_device(rope)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    encs = []
    for row0, T in segments:
        sl = slice(row0, row0 + T)
        diag = osp.quantize_into(ocaches, K64[:, :, sl], V64[:, :, sl], sc, rope=rope, pos0=row0,
                                 row0=row0)
        native.quantize_kv_split(ns, kd[:, :, sl], vd[:, :, sl], nhi, nlo, row0=row0, rope=rd,
                                 pos0=row0, status=status)
        encs.append((np.arange(row0, row0 + T), diag["enc"]))
    torch.cuda.synchronize()
    gpus = (tl.download_cache(nhi), tl.download_cache(nlo))
    codecs = (sc.hi, sc.lo)
    stats = tl.new_stats()
    for rows, enc in encs:
        for (part, b, h), (ek, ev) in enc.items():
            tl.compare_rows(gpus[part], ocaches[part], codecs[part], b, h, rows, ek, ev, stats)
    tl.assert_mismatch_budget(stats)
    assert int(status.item()) == 0


def _upload(sc, ns, ocaches, w):
    return (tl.upload_cache(ocaches[0], ns.hi, w.B, w.Hkv),
            tl.upload_cache(ocaches[1], ns.lo, w.B, w.Hkv))


@pytest.mark.parametrize("case", list(CASES))
def test_split_dequantize_parity(case):
    w, sc, ns, K, V, K64, V64, _, _, _, rows_cap = _setup(case)
    rope = synth.rope_for(w, rows_cap)
    ocaches = osp.empty_caches(sc, w.B, w.Hkv, rows_cap)
    osp.quantize_into(ocaches, K64, V64, sc, rope=rope)
    chi, clo = _upload(sc, ns, ocaches, w)
    row0, rows = 5, w.T - 9
    for which in (0, 1):
        out = torch.full((w.B, w.Hkv, rows, w.d), float("nan"), device="cuda")
        native.dequantize_split(ns, chi, clo, which, row0, rows, out)
        got = out.cpu().numpy().astype(np.float64)
        for b in range(w.B):
            for h in range(w.Hkv):
                ref = osp.dequantize(ocaches, sc, which, b, h, row0 + rows)[row0:]
                err = np.linalg.norm(got[b, h] - ref, axis=1) / np.linalg.norm(ref, axis=1)
                assert np.max(err) <= 1e-3, (which, b, h, np.max(err))


@pytest.mark.parametrize("case", list(CASES))
def test_split_decode_parity(case):
    w, sc, ns, K, V, K64, V64, _, lens, splits, rows_cap = _setup(case)
    rope = synth.rope_for(w, rows_cap)
    ocaches = osp.empty_caches(sc, w.B, w.Hkv, rows_cap)
    osp.quantize_into(ocaches, K64, V64, sc, rope=rope)
    chi, clo = _upload(sc, ns, ocaches, w)
    q = synth.query_inputs(w, Lq=1)[:, :, 0]
    q64 = synth.as_float64(q, w.dtype)
    scale = 1.0 / np.sqrt(w.d)
    ref = osp.decode(q64, ocaches, sc, lens, scale, rope=rope)
    qd = tl.to_device(np.ascontiguousarray(q), w.dtype)
    out = torch.full((w.B, w.Hq, w.d), float("nan"), device="cuda")
    ws = torch.empty(native.attention_split_workspace(ns, w.B, w.Hq, splits), dtype=torch.uint8,
                     device="cuda")
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    native.attention_decode_split(ns, qd, chi, clo, max(lens), scale, out, ws, seq_lens=seq,
                                  rope=tl.rope_device(rope), num_splits=splits)
    got = out.cpu().numpy().astype(np.float64)
    vscale = tl.channel_scale_of_values(w)
    for b in range(w.B):
        for h in range(w.Hq):
            err = np.abs(got[b, h] - ref[b, h]) / vscale[h // w.G]
            assert np.max(err) <= 2e-3, (b, h, np.max(err))


def test_split_rejects_bad_arguments():
    w, sc, ns, *_ = _setup("llama_mse_g2")
    chi = native.alloc_cache(ns.hi, 1, 2, 64)
    clo = native.alloc_cache(ns.lo, 1, 2, 96)        # rows_cap differs
    q = torch.zeros((1, 4, 128), device="cuda")
    out = torch.empty((1, 4, 128), device="cuda")
    ws = torch.empty(native.attention_split_workspace(ns, 1, 4, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(native.TqError) as e:
        native.attention_decode_split(ns, q, chi, clo, 64, 0.1, out, ws, num_splits=2)
    assert e.value.code == native.TQ_ERR_INVALID_ARG
    clo = native.alloc_cache(ns.lo, 1, 2, 64)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(native.TqError) as e:
        native.attention_decode_split(ns, q, chi, clo, 64, 0.1, out, small, num_splits=2)
    assert e.value.code == native.TQ_ERR_WORKSPACE
    # codecs of different widths cannot form a split
    other = native.Codec(128, 3, True, 3, synth.rotation_signs(128, 1), synth.qjl_matrix_bf16(128, 1))
    bad = native.Split(ns.hi, other, ns.channels)
    with pytest.raises(native.TqError) as e:
        native.attention_decode_split(bad, q, chi, clo, 64, 0.1, out, ws, num_splits=2)
    assert e.value.code == native.TQ_ERR_UNSUPPORTED


def test_split_quantize_nonfinite_rows():
    """A NaN in an outlier channel spoils only the half that holds it: that
    half row is stored as a zero row and counted, the other half is coded."""
    w, sc, ns, *_ = _setup("llama_mse_g2")
    T = 64
    K = torch.randn((1, 2, T, 128), device="cuda")
    V = torch.randn((1, 2, T, 128), device="cuda")
    ch = sc.channels[0, 0]
    K[0, 0, 10, int(ch[3])] = float("nan")          # an outlier (hi) key channel of head 0
    chi = native.alloc_cache(ns.hi, 1, 2, T)
    clo = native.alloc_cache(ns.lo, 1, 2, T)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.quantize_kv_split(ns, K, V, chi, clo, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    assert float(chi.kscale[0, 0, 10, 0]) == 0.0
    assert float(clo.kscale[0, 0, 10, 0]) > 0.0
