"""Quality report of the compressed cache (relMSE_K, relMSE_V, cosine of the
attention output), as bench.py's ``--only quality`` prints it for the tiny,
Llama-shaped, ESM-2-shaped and long-context workloads, for keys with the QJL
sketch (TQ-QKV) and keys spent wholly on the MSE stage (TQ-KV).

The pin: on the same seeded inputs, the relative MSE of the GPU's
tq_dequantize output equals the oracle's (the codes agree except at decision
boundaries, whose effect on a sum over 10^5 coordinates is far below the
tolerance); the report itself is then checked for sane ranges."""
import os
import sys

import numpy as np
import pytest
import torch

from oracle import codec as oc
from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


def _rel(xh: np.ndarray, x: np.ndarray) -> float:
    return float(((xh - x) ** 2).sum() / (x ** 2).sum())


@pytest.mark.parametrize("name,qjl", [("tiny", True), ("tiny", False),
                                      ("llama_small", True), ("llama_small", False)])
def test_relmse_matches_oracle(name, qjl):
    w = (synth.WORKLOADS["tiny"] if name == "tiny"
         else synth.WORKLOADS["llama_decode"].scaled(Hq=8, Hkv=2, T=500))
    w = w.scaled(qjl_k=qjl)
    ocodec, ncodec = tl.codecs(w)
    K, V = synth.kv_inputs(w)
    K64, V64 = synth.as_float64(K, w.dtype), synth.as_float64(V, w.dtype)
    rows_cap = (w.T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    # oracle: quantize, then dequantize every row
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    oc.quantize_into(ocache, K64, V64, ocodec, rope=rope)
    ok_, ov_ = [], []
    for b in range(w.B):
        for h in range(w.Hkv):
            ik, sg, nk, rk, iv, nv = oc.cache_rows(ocache, ocodec, b, h, w.T)
            ok_.append(oc.dequant_keys(ik, sg, nk, rk, ocodec))
            ov_.append(oc.dequant_values(iv, nv, ocodec))
    ok_ = np.stack(ok_).reshape(w.B, w.Hkv, w.T, w.d)
    ov_ = np.stack(ov_).reshape(w.B, w.Hkv, w.T, w.d)
    # the exact post-RoPE keys, in fp64 from the same tables
    Kr = K64.copy()
    if rope is not None:
        c, s = rope[0][:w.T].astype(np.float64), rope[1][:w.T].astype(np.float64)
        h2 = w.d // 2
        u, v = K64[..., :h2], K64[..., h2:]
        Kr = np.concatenate((u * c - v * s, v * c + u * s), axis=-1)
    # GPU: quantize the same inputs, dequantize through the C ABI
    dev = tl.to_device(K, w.dtype), tl.to_device(V, w.dtype)
    ncache = native.alloc_cache(ncodec, w.B, w.Hkv, rows_cap)
    rd = None if rope is None else (torch.from_numpy(rope[0]).cuda(), torch.from_numpy(rope[1]).cuda())
    native.quantize_kv(ncodec, dev[0], dev[1], ncache, rope=rd)
    got = []
    for which in (0, 1):
        out = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=torch.float32, device="cuda")
        native.dequantize(ncodec, ncache, which, 0, w.T, out)
        got.append(out.cpu().numpy().astype(np.float64))
    for xh_gpu, xh_or, x in ((got[0], ok_, Kr), (got[1], ov_, V64)):
        r_gpu, r_or = _rel(xh_gpu, x), _rel(xh_or, x)
        assert 0.0 < r_or < 1.0
        assert abs(r_gpu - r_or) <= 2e-3 * r_or, (r_gpu, r_or)


def test_quality_report_ranges():
    # Llama-shaped heads without the outlier channels: logits spread ~1, where
    # the oracle's own decode output keeps a cosine above 0.94 to exact
    # attention (with the 4 x20 outlier channels the spread is ~10 and even
    # the oracle's output cosine falls to ~0.8 on average at this length)
    r = bench.quality_extra("llama_decode", T=4096, overrides=dict(n_outliers=0, sigma_scale=None))
    assert set(r["variants"]) == {"prod", "mse"}
    for var, q in r["variants"].items():
        assert 0.0 < q["relMSE_K"] < 0.1 and 0.0 < q["relMSE_V"] < 0.05, (var, q)
        assert q["output_cosine_min"] is not None and q["output_cosine_min"] > 0.9, (var, q)
    # the same value codec in both variants: identical value error
    assert r["variants"]["prod"]["relMSE_V"] == pytest.approx(r["variants"]["mse"]["relMSE_V"], rel=1e-6)
    # 4 MSE bits reconstruct keys better than 3 MSE bits + the 1-bit sketch
    assert r["variants"]["mse"]["relMSE_K"] < r["variants"]["prod"]["relMSE_K"]
