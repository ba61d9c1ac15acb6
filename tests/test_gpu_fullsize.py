"""Full-size parity in the launch configuration bench.py times.

Llama-3.1-8B-shaped decode layer (B=1, 32/8 heads, d=128, T=32768, 64 splits,
RoPE) and the long-context decode (B=4, 32/8 heads, T=131072, 128 splits):
* quantize: the whole context is encoded on the GPU exactly as the benchmark
  does (prefill of T-1 tokens, then the new token appended); a random sample
  of rows is re-encoded by the oracle one by one and compared under the
  boundary-window rule;
* decode: the oracle encodes every token of two sampled KV heads; those heads'
  planes replace the GPU's in the full cache, the full-size split-K decode
  runs, and the sampled query heads are compared with the oracle's decode.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import codec as oc
from oracle.rotation import apply_rope
from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


def _run(name, sample_rows, sample_heads):
    w = synth.WORKLOADS[name]
    ocodec, ncodec = tl.codecs(w)
    K, V = synth.kv_inputs(w)
    T = w.T
    rows_cap = (T + 31) // 32 * 32
    rope = synth.rope_for(w, rows_cap)
    rd = tl.rope_device(rope)
    kd, vd = tl.to_device(K, w.dtype), tl.to_device(V, w.dtype)
    cache = native.alloc_cache(ncodec, w.B, w.Hkv, rows_cap)
    native.quantize_kv(ncodec, kd[:, :, :T - 1], vd[:, :, :T - 1], cache, rope=rd)
    native.quantize_kv(ncodec, kd[:, :, T - 1:].contiguous(), vd[:, :, T - 1:].contiguous(),
                       cache, row0=T - 1, rope=rd, pos0=T - 1)
    torch.cuda.synchronize()
    del kd, vd
    gpu = tl.download_cache(cache)

    # ---- sampled-row quantize parity
    rng = np.random.default_rng(123)
    stats = tl.new_stats()
    for b in range(w.B):
        for h in range(w.Hkv):
            rows = np.sort(rng.choice(T, size=sample_rows, replace=False))
            rows[-1] = T - 1                      # always include the appended token
            rows = np.unique(rows)
            k = synth.as_float64(K[b, h, rows], w.dtype)
            if rope is not None:
                k = apply_rope(k, rope[0], rope[1], rows)
            ek = oc.quantize_keys(k, ocodec)
            ev = oc.quantize_values(synth.as_float64(V[b, h, rows], w.dtype), ocodec)
            tl.compare_rows(gpu, None, ocodec, b, h, rows, ek, ev, stats)
    tl.assert_mismatch_budget(stats)

    # ---- full-size decode on oracle-encoded heads
    q = synth.query_inputs(w, Lq=1)[:, :, 0]
    ocache = oc.empty_cache(ocodec, w.B, w.Hkv, rows_cap)
    for b, h in sample_heads:
        sub = oc.empty_cache(ocodec, 1, 1, rows_cap)
        oc.quantize_into(sub, synth.as_float64(K[b:b + 1, h:h + 1], w.dtype),
                         synth.as_float64(V[b:b + 1, h:h + 1], w.dtype), ocodec, rope=rope)
        for key in ("kcode", "kscale", "vcode", "vnorm"):
            ocache[key][b, h] = sub[key][0, 0]
            src = sub[key][0, 0].view(np.int32) if key == "vcode" else sub[key][0, 0]
            getattr(cache, key)[b, h].copy_(torch.from_numpy(np.ascontiguousarray(src)))
    ws = torch.empty(native.attention_workspace(ncodec, w.B, w.Hq, w.num_splits), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    scale = 1.0 / math.sqrt(w.d)
    native.attention_decode(ncodec, tl.to_device(q, w.dtype), cache, T, scale, out, ws, rope=rd,
                            num_splits=w.num_splits)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    heads = [(b, h * w.G + g) for b, h in sample_heads for g in range(w.G)]
    ref = oatt.decode(synth.as_float64(q, w.dtype), ocache, ocodec, [T] * w.B, scale, rope=rope,
                      heads=heads)
    vscale = tl.channel_scale_of_values(w)
    for b, hq in heads:
        err = np.abs(got[b, hq] - ref[b, hq]) / vscale[hq // w.G]
        assert np.max(err) <= 2e-3, (b, hq, float(np.max(err)))
    return stats


def test_fullsize_llama_decode():
    _run("llama_decode", sample_rows=512, sample_heads=[(0, 0), (0, 5)])


def test_fullsize_long_context_decode():
    _run("long_decode", sample_rows=128, sample_heads=[(1, 3), (3, 7)])
