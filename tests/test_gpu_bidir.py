"""Bidirectional attention over the compressed cache (ESM-2-shaped prefill
pass) through the C ABI, against the oracle on the same (oracle-encoded) cache.
Query i sits at position i and attends to every key; output within 2e-3
max-abs after dividing each value channel by its synthetic scale."""
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


def _run(w, T, Lq, heads=None, dtype=None):
    dtype = dtype or w.dtype
    ocodec, ncodec = tl.codecs(w)
    ww = w.scaled(T=T, Lq=Lq, dtype=dtype)
    K, V = synth.kv_inputs(ww)
    q = synth.query_inputs(ww)
    K64, V64 = synth.as_float64(K, dtype), synth.as_float64(V, dtype)
    rows_cap = (T + 31) // 32 * 32
    tmax = max(rows_cap, Lq)
    rope = synth.rope_for(w, tmax)
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    oc.quantize_into(ocache, K64, V64, ocodec, rope=rope)
    ncache = tl.upload_cache(ocache, ncodec, w.B, w.Hkv)
    scale = 1.0 / math.sqrt(w.d)
    ws = torch.empty(native.attention_bidir_workspace(ncodec, w.B, w.Hq, Lq), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((w.B, w.Hq, Lq, w.d), float("nan"), dtype=torch.float32, device="cuda")
    native.attention_bidir(ncodec, tl.to_device(q, dtype), ncache, T, scale, out, ws,
                           rope=tl.rope_device(rope))
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    ref = oatt.bidirectional(synth.as_float64(q, dtype), ocache, ocodec, T, scale, rope=rope,
                             heads=heads)
    vscale = tl.channel_scale_of_values(w)
    heads = heads or [(b, h) for b in range(w.B) for h in range(w.Hq)]
    worst = 0.0
    for b, h in heads:
        err = np.abs(got[b, h] - ref[b, h]) / vscale[h // (w.Hq // w.Hkv)][None, :]
        worst = max(worst, float(np.max(err)))
    assert worst <= 2e-3, worst
    return worst


@pytest.mark.parametrize("T,Lq", [(300, 300), (64, 200), (1000, 129)])
def test_bidir_small(T, Lq):
    w = synth.WORKLOADS["esm_prefill"].scaled(B=2, Hq=3, Hkv=3)
    _run(w, T, Lq)


def test_bidir_gqa_fp32_no_rope():
    w = synth.WORKLOADS["esm_prefill"].scaled(B=1, Hq=4, Hkv=2, rope_theta=None)
    _run(w, 257, 130, dtype="fp32")


def test_bidir_fullsize_sampled_heads():
    """ESM-2-650M shape: B=16, 20 heads, d=64, T=Lq=1024, all heads computed on
    the GPU; three (batch, head) pairs compared with the oracle."""
    w = synth.WORKLOADS["esm_prefill"]
    _run(w, w.T, w.Lq, heads=[(0, 0), (7, 13), (15, 19)])


def test_bidir_rejects_unsupported_head_dim():
    w = synth.WORKLOADS["tiny"]
    _, ncodec = tl.codecs(w)
    cache = native.alloc_cache(ncodec, 1, 1, 64)
    q = torch.zeros((1, 1, 8, 128), device="cuda")
    out = torch.empty((1, 1, 8, 128), device="cuda")
    ws = torch.empty(native.attention_bidir_workspace(ncodec, 1, 1, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(native.TqError) as e:
        native.attention_bidir(ncodec, q, cache, 64, 0.1, out, ws)
    assert e.value.code == native.TQ_ERR_UNSUPPORTED
