"""GPU-vs-oracle parity through the C ABI (quantize, dequantize, decode).

Sizes are small enough for the oracle to finish in seconds but span several
tiles, ragged tails, partially covered 32-token value groups and empty split-K
chunks.  Full-size checks (the launch configuration bench.py times) live in
test_gpu_fullsize.py."""
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


def _inputs(w):
    K, V = synth.kv_inputs(w)
    return K, V, synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)


QUANT_CASES = {
    "tiny": (synth.WORKLOADS["tiny"], [(0, 1024)]),
    "llama_ragged": (synth.WORKLOADS["llama_decode"].scaled(T=200), [(0, 200)]),
    "llama_appends": (synth.WORKLOADS["llama_decode"].scaled(T=138), [(0, 100), (100, 1), (101, 37)]),
    "esm_d64": (synth.WORKLOADS["esm_prefill"].scaled(B=2, Hq=3, Hkv=3, T=100), [(0, 100)]),
    "long_2bit": (synth.WORKLOADS["long_decode"].scaled(B=2, Hq=8, Hkv=2, T=300), [(0, 300)]),
    # >= 256 groups of 32 tokens: large calls take the tcgen05 sketch kernel
    "llama_tc_sketch": (synth.WORKLOADS["llama_decode"].scaled(T=1100), [(0, 1037), (1037, 63)]),
    "esm_tc_sketch_d64": (synth.WORKLOADS["esm_prefill"].scaled(B=4, T=100), [(0, 100)]),
    # large call, fp32 input, MSE-only keys (no sketch)
    "llama_lanes_fp32_mse": (synth.WORKLOADS["llama_decode"].scaled(T=1100, dtype="fp32", qjl_k=False,
                                                                     bits_k=3), [(0, 1100)]),
    # large bf16 calls take the one-thread-per-row tile kernel; the second call
    # starts mid-tile and mid value group (row 600)
    "llama_tile_offset": (synth.WORKLOADS["llama_decode"].scaled(B=2, T=1100), [(0, 600), (600, 500)]),
    "llama_tile_mse4": (synth.WORKLOADS["llama_decode"].scaled(T=1100, qjl_k=False, bits_k=4), [(0, 1100)]),
    "esm_tile_mse3_d64": (synth.WORKLOADS["esm_prefill"].scaled(B=4, T=100, qjl_k=False, bits_k=3),
                          [(0, 100)]),
    "esm_tile_offset_d64": (synth.WORKLOADS["esm_prefill"].scaled(B=4, T=300), [(0, 45), (45, 255)]),
    # an odd number of (batch, head) rows: the tile kernel's last step holds one tile
    "esm_tile_odd_heads_d64": (synth.WORKLOADS["esm_prefill"].scaled(B=1, Hq=3, Hkv=3, T=2800),
                               [(0, 2800)]),
    "llama_tile_odd_heads": (synth.WORKLOADS["llama_decode"].scaled(B=1, Hq=20, Hkv=5, T=3600),
                             [(0, 1700), (1700, 1900)]),
}


def _quantize_both(w, segments, rows_cap=None):
    ocodec, ncodec = tl.codecs(w)
    K, V, K64, V64 = _inputs(w)
    rows_cap = rows_cap or (w.T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    ncache = native.alloc_cache(ncodec, w.B, w.Hkv, rows_cap)
    kd, vd = tl.to_device(K, w.dtype), tl.to_device(V, w.dtype)
    rd = tl.rope_device(rope)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    encs = {}
    for row0, T in segments:
        sl = slice(row0, row0 + T)
        diag = oc.quantize_into(ocache, K64[:, :, sl], V64[:, :, sl], ocodec, rope=rope,
                                pos0=row0, row0=row0)
        native.quantize_kv(ncodec, kd[:, :, sl], vd[:, :, sl], ncache, row0=row0, rope=rd,
                           pos0=row0, status=status)
        i = 0
        for b in range(w.B):
            for h in range(w.Hkv):
                encs.setdefault((b, h), []).append((np.arange(row0, row0 + T), diag["k"][i], diag["v"][i]))
                i += 1
    torch.cuda.synchronize()
    return ocodec, ncodec, ocache, ncache, encs, int(status.item())


@pytest.mark.parametrize("impl", ["default", "simt"])
@pytest.mark.parametrize("case", list(QUANT_CASES))
def test_quantize_parity(case, impl, monkeypatch):
    # "default": tensor-core sketch for calls of >= 256 token groups with QJL;
    # "simt": the CUDA-core sketch everywhere
    if impl == "simt":
        monkeypatch.setenv("TQ_QUANT_IMPL", "simt")
    else:
        monkeypatch.delenv("TQ_QUANT_IMPL", raising=False)
    w, segments = QUANT_CASES[case]
    ocodec, ncodec, ocache, ncache, encs, bad = _quantize_both(w, segments)
    gpu = tl.download_cache(ncache)
    stats = tl.new_stats()
    for (b, h), parts in encs.items():
        for rows, ek, ev in parts:
            tl.compare_rows(gpu, ocache, ocodec, b, h, rows, ek, ev, stats)
    tl.assert_mismatch_budget(stats)
    assert bad == 0
    # rows outside the written ranges stay zero
    written = max(r0 + T for r0, T in segments)
    assert not gpu["kcode"][:, :, written:].any()
    assert not gpu["vnorm"][:, :, written:].any()


@pytest.mark.parametrize("T,dtype", [(64, "fp32"), (4096, "fp32"), (4096, "bf16")])
def test_quantize_zero_and_nonfinite_rows(T, dtype):
    # 4096 rows: 256 token groups, the large-call kernels (bf16: one thread per row)
    w = synth.WORKLOADS["llama_decode"].scaled(B=1, Hkv=2, Hq=8, T=T)
    ocodec, ncodec = tl.codecs(w)
    K, V, K64, V64 = _inputs(w)
    Kf = synth.bf16_bits_to_f32(K).copy()
    Vf = synth.bf16_bits_to_f32(V).copy()
    Kf[0, 0, 3] = 0.0
    Kf[0, 1, 5, 17] = np.nan
    Vf[0, 0, 9, 2] = np.inf
    Vf[0, 1, 10] = 0.0
    Kf[0, 1, 40, 0] = 1e6          # key norm overflows fp16
    if dtype == "bf16":            # every value above is exact in bf16
        Kf = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.nan_to_num(Kf, nan=0.0, posinf=0.0)))
        Kf[0, 1, 5, 17] = np.nan
        Vf = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.nan_to_num(Vf, nan=0.0, posinf=0.0)))
        Vf[0, 0, 9, 2] = np.inf
    w32 = w.scaled(dtype="fp32")
    rope = synth.rope_for(w32, T)
    ocache = oc.empty_cache(ocodec, 1, 2, T)
    diag = oc.quantize_into(ocache, Kf.astype(np.float64), Vf.astype(np.float64), ocodec, rope=rope)
    ncache = native.alloc_cache(ncodec, 1, 2, T)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if dtype == "bf16":
        kd = torch.from_numpy(Kf).cuda().to(torch.bfloat16)
        vd = torch.from_numpy(Vf).cuda().to(torch.bfloat16)
    else:
        kd, vd = tl.to_device(Kf, "fp32"), tl.to_device(Vf, "fp32")
    native.quantize_kv(ncodec, kd, vd, ncache, rope=tl.rope_device(rope), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == diag["bad_rows"] == 3
    gpu = tl.download_cache(ncache)
    stats = tl.new_stats()
    for i, (b, h) in enumerate([(0, 0), (0, 1)]):
        tl.compare_rows(gpu, ocache, ocodec, b, h, np.arange(T), diag["k"][i], diag["v"][i], stats)
    tl.assert_mismatch_budget(stats)
    assert gpu["kscale"][0, 1, 5, 0] == 0 and gpu["vnorm"][0, 0, 9] == 0


DEQUANT_CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "llama_ragged": synth.WORKLOADS["llama_decode"].scaled(T=200),
    "esm_d64": synth.WORKLOADS["esm_prefill"].scaled(B=2, Hq=3, Hkv=3, T=100),
    "long_2bit": synth.WORKLOADS["long_decode"].scaled(B=2, Hq=8, Hkv=2, T=300),
    "tiny_mse_keys": synth.WORKLOADS["tiny"].scaled(qjl_k=False, bits_k=3),
    "llama_mse_keys": synth.WORKLOADS["llama_decode"].scaled(T=200, qjl_k=False, bits_k=4),
    "long_mse_keys": synth.WORKLOADS["long_decode"].scaled(B=2, Hq=8, Hkv=2, T=300, qjl_k=False,
                                                          bits_k=2),
}


@pytest.mark.parametrize("case", list(DEQUANT_CASES))
def test_dequantize_parity(case):
    w = DEQUANT_CASES[case]
    ocodec, ncodec = tl.codecs(w)
    K, V, K64, V64 = _inputs(w)
    rows_cap = (w.T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    oc.quantize_into(ocache, K64, V64, ocodec, rope=rope)
    ncache = tl.upload_cache(ocache, ncodec, w.B, w.Hkv)
    row0, rows = 3, w.T - 3
    for which in (0, 1):
        out = torch.empty((w.B, w.Hkv, rows, w.d), dtype=torch.float32, device="cuda")
        native.dequantize(ncodec, ncache, which, row0, rows, out)
        got = out.cpu().numpy().astype(np.float64)
        for b in range(w.B):
            for h in range(w.Hkv):
                ik, sg, nk, rk, iv, nv = oc.cache_rows(ocache, ocodec, b, h, w.T)
                ref = (oc.dequant_keys(ik, sg, nk, rk, ocodec) if which == 0
                       else oc.dequant_values(iv, nv, ocodec))[row0:]
                err = np.linalg.norm(got[b, h] - ref, axis=1)
                nrm = np.linalg.norm(ref, axis=1)
                assert np.all(err <= 1e-3 * nrm + 1e-30), (which, b, h, np.max(err / np.maximum(nrm, 1e-30)))


DECODE_CASES = {
    "tiny": (synth.WORKLOADS["tiny"], None, 8),
    "llama_splits7": (synth.WORKLOADS["llama_decode"].scaled(T=1000), None, 7),
    "llama_one_split": (synth.WORKLOADS["llama_decode"].scaled(B=1, Hq=8, Hkv=2, T=3000), None, 1),
    "long_empty_splits": (synth.WORKLOADS["long_decode"].scaled(B=2, Hq=8, Hkv=2, T=3000), None, 128),
    "esm_mha_d64": (synth.WORKLOADS["esm_prefill"].scaled(B=2, Hq=3, Hkv=3, T=300, Lq=1), None, 4),
    "ragged_lens": (synth.WORKLOADS["llama_decode"].scaled(B=3, Hq=8, Hkv=2, T=300), [1, 77, 300], 5),
    "gqa8": (synth.WORKLOADS["long_decode"].scaled(B=1, Hq=16, Hkv=2, T=500), None, 3),
    "gqa2_multi_sub": (synth.WORKLOADS["llama_decode"].scaled(B=1, Hq=4, Hkv=2, T=2500), None, 1),
    "tiny_two_chunks": (synth.WORKLOADS["tiny"].scaled(T=1000), None, 2),
    # MSE-only keys (TQ-KV, no QJL plane): all key bits on the Lloyd-Max stage
    "tiny_mse_keys": (synth.WORKLOADS["tiny"].scaled(qjl_k=False, bits_k=3), None, 8),
    "llama_mse_keys": (synth.WORKLOADS["llama_decode"].scaled(T=1000, qjl_k=False, bits_k=4), None, 7),
    "long_mse_keys": (synth.WORKLOADS["long_decode"].scaled(B=2, Hq=8, Hkv=2, T=3000, qjl_k=False,
                                                           bits_k=2), None, 128),
    "esm_mse_keys_d64": (synth.WORKLOADS["esm_prefill"].scaled(B=2, Hq=4, Hkv=2, T=300, Lq=1,
                                                               qjl_k=False, bits_k=3), None, 4),
}


def _decode_case(w, lens, splits):
    ocodec, ncodec = tl.codecs(w)
    K, V, K64, V64 = _inputs(w)
    rows_cap = (w.T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    oc.quantize_into(ocache, K64, V64, ocodec, rope=rope)
    ncache = tl.upload_cache(ocache, ncodec, w.B, w.Hkv)
    q = synth.query_inputs(w, Lq=1)[:, :, 0]
    q64 = synth.as_float64(q, w.dtype)
    scale = 1.0 / math.sqrt(w.d)
    lens = [w.T] * w.B if lens is None else lens
    ref, ref_logits = oatt.decode(q64, ocache, ocodec, lens, scale, rope=rope, want_logits=True)
    ws = torch.empty(native.attention_workspace(ncodec, w.B, w.Hq, splits) // 4 + 4,
                     dtype=torch.float32, device="cuda")
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    logits = torch.full((w.B, w.Hq, w.T), float("nan"), dtype=torch.float32, device="cuda")
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    native.attention_logits(ncodec, tl.to_device(q, w.dtype), ncache, w.T, scale, out, logits, ws,
                            seq_lens=sl, rope=tl.rope_device(rope), num_splits=splits)
    torch.cuda.synchronize()
    return ref, ref_logits, out.cpu().numpy().astype(np.float64), logits.cpu().numpy(), lens


@pytest.mark.parametrize("impl", ["default", "simt"])
@pytest.mark.parametrize("case", list(DECODE_CASES))
def test_decode_parity(case, impl, monkeypatch):
    # "default" takes the tensor-core kernels where they are built (d=128,
    # group size 1/2/4, the bit widths of the workloads) and the CUDA-core
    # kernels elsewhere; "simt" forces the CUDA-core kernels everywhere.
    if impl == "simt":
        monkeypatch.setenv("TQ_DECODE_IMPL", "simt")
    else:
        monkeypatch.delenv("TQ_DECODE_IMPL", raising=False)
    w, lens, splits = DECODE_CASES[case]
    ref, ref_logits, got, got_logits, lens = _decode_case(w, lens, splits)
    vscale = tl.channel_scale_of_values(w)
    for b in range(w.B):
        for h in range(w.Hq):
            lr = ref_logits[(b, h)]
            lg = got_logits[b, h, :lens[b]].astype(np.float64)
            rms = math.sqrt(np.mean(lr * lr))
            assert np.max(np.abs(lg - lr)) <= 1e-3 * rms, (b, h, np.max(np.abs(lg - lr)) / rms)
            err = np.abs(got[b, h] - ref[b, h]) / vscale[h // w.G]
            assert np.max(err) <= 2e-3, (b, h, np.max(err))


def test_decode_rejects_bad_arguments():
    w = synth.WORKLOADS["tiny"]
    _, ncodec = tl.codecs(w)
    cache = native.alloc_cache(ncodec, 1, 1, 64)
    q = torch.zeros((1, 1, 128), device="cuda")
    out = torch.empty((1, 1, 128), device="cuda")
    small = torch.empty(4, device="cuda")
    with pytest.raises(native.TqError) as e:
        native.attention_decode(ncodec, q, cache, 64, 0.1, out, small, num_splits=4)
    assert e.value.code == native.TQ_ERR_WORKSPACE
    ws = torch.empty(native.attention_workspace(ncodec, 1, 1, 4), dtype=torch.uint8, device="cuda")
    with pytest.raises(native.TqError) as e:
        native.attention_decode(ncodec, q, cache, 65, 0.1, out, ws, num_splits=4)
    assert e.value.code == native.TQ_ERR_INVALID_ARG
    with pytest.raises(native.TqError):
        native.quantize_kv(ncodec, torch.zeros((1, 1, 70, 128), device="cuda"),
                           torch.zeros((1, 1, 70, 128), device="cuda"), cache)


def test_decode_step_equals_append_then_decode():
    """tq_decode_step is tq_quantize_kv at row T - 1 followed by
    tq_attention_decode over T rows: same cache bytes, same output bits; so is
    tq_decode_step_host, fed from and read back to host memory."""
    w = synth.WORKLOADS["llama_decode"].scaled(B=2, Hq=8, Hkv=2, T=333)
    _, ncodec = tl.codecs(w)
    K, V = synth.kv_inputs(w)
    kd, vd = tl.to_device(K, w.dtype), tl.to_device(V, w.dtype)
    q = tl.to_device(np.ascontiguousarray(synth.query_inputs(w, Lq=1)[:, :, 0]), w.dtype)
    rope = tl.rope_device(synth.rope_for(w, 352))
    caches, outs = [], []
    for mode in ("separate", "fused", "host"):
        c = native.alloc_cache(ncodec, w.B, w.Hkv, 352)
        native.quantize_kv(ncodec, kd[:, :, :w.T - 1], vd[:, :, :w.T - 1], c, rope=rope)
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
        ws = torch.empty(native.attention_workspace(ncodec, w.B, w.Hq, 5), dtype=torch.uint8,
                         device="cuda")
        kn, vn = kd[:, :, w.T - 1:].contiguous(), vd[:, :, w.T - 1:].contiguous()
        if mode == "fused":
            native.decode_step(ncodec, kn, vn, q, c, w.T, 0.088, out, ws, rope=rope, num_splits=5)
        elif mode == "host":
            # the three parts back to back in one pinned host buffer, the
            # output read back into pinned host memory by the call itself
            hin = torch.cat([kn.reshape(-1), vn.reshape(-1), q.reshape(-1)]).cpu().pin_memory()
            din = torch.empty_like(hin, device="cuda")
            hout = torch.full((w.B, w.Hq, w.d), float("nan")).pin_memory()
            native.decode_step_host(ncodec, hin, din, kn.dtype, q.dtype, w.B, w.Hq, w.Hkv, c, w.T, 0.088,
                                    out, hout, ws, rope=rope, num_splits=5)
            assert torch.equal(hout, out.cpu())
        else:
            native.quantize_kv(ncodec, kn, vn, c, row0=w.T - 1, rope=rope, pos0=w.T - 1)
            native.attention_decode(ncodec, q, c, w.T, 0.088, out, ws, rope=rope, num_splits=5)
        torch.cuda.synchronize()
        caches.append(tl.download_cache(c))
        outs.append(out.cpu().numpy())
    for i in (1, 2):
        for key in ("kcode", "kscale", "vcode", "vnorm"):
            assert np.array_equal(caches[0][key], caches[i][key]), (i, key)
        assert np.array_equal(outs[0], outs[i]), i
    # the input size must be the parts' total
    with pytest.raises(native.TqError) as e:
        native.decode_step_host(ncodec, hin[:-8], din, kn.dtype, q.dtype, w.B, w.Hq, w.Hkv, c, w.T,
                                0.088, out, hout, ws, rope=rope, num_splits=5)
    assert e.value.code == native.TQ_ERR_INVALID_ARG
