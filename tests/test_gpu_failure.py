"""A bounded wait that gives up is reported, and the GPU stays usable.

Every wait inside the tensor-core decode, bidirectional and scan kernels polls
an mbarrier a bounded number of times.  TQ_WAIT_LIMIT (read at each launch)
sets that bound; 0 makes every wait give up at once, which is how these tests
make the failure happen without faulting or hanging anything: the kernel
drains its own copies and MMAs and reports the give-up (decode: the split-K
combine writes NaN for every output instead of merging incomplete partials;
bidirectional pass: the queries of a CTA that gave up are written as NaN;
scan: every result becomes index -1, score NaN; tile quantize and index
build: bit 31 of the call's status word).  The next call without the
override must be exact again."""
import math

import numpy as np
import pytest
import torch

from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


def test_decode_wait_give_up_is_reported_as_nan(monkeypatch):
    w = synth.WORKLOADS["llama_decode"].scaled(B=1, Hq=8, Hkv=2, T=2048)
    _, ncodec = tl.codecs(w)
    K, V = synth.kv_inputs_torch(w)
    r = synth.rope_for(w, w.T)
    rope = tl.rope_device(r)
    cache = native.alloc_cache(ncodec, w.B, w.Hkv, w.T)
    native.quantize_kv(ncodec, K, V, cache, rope=rope)
    q = synth.query_inputs_torch(w)[:, :, 0].contiguous()
    ws = torch.empty(native.attention_workspace(ncodec, w.B, w.Hq, 8), dtype=torch.uint8, device="cuda")
    scale = 1 / math.sqrt(w.d)
    good = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    native.attention_decode(ncodec, q, cache, w.T, scale, good, ws, rope=rope, num_splits=8)
    torch.cuda.synchronize()
    assert torch.isfinite(good).all()

    monkeypatch.setenv("TQ_WAIT_LIMIT", "0")
    bad = torch.zeros_like(good)
    native.attention_decode(ncodec, q, cache, w.T, scale, bad, ws, rope=rope, num_splits=8)
    torch.cuda.synchronize()
    assert torch.isnan(bad).all()

    monkeypatch.delenv("TQ_WAIT_LIMIT")
    again = torch.empty_like(good)
    native.attention_decode(ncodec, q, cache, w.T, scale, again, ws, rope=rope, num_splits=8)
    torch.cuda.synchronize()
    assert torch.equal(again, good)


def test_bidir_wait_give_up_is_reported_as_nan(monkeypatch):
    w = synth.WORKLOADS["esm_prefill"].scaled(B=1, Hq=2, Hkv=2, T=300, Lq=300)
    _, ncodec = tl.codecs(w)
    K, V = synth.kv_inputs_torch(w)
    r = synth.rope_for(w, 320)
    rope = tl.rope_device(r)
    cache = native.alloc_cache(ncodec, w.B, w.Hkv, 320)
    native.quantize_kv(ncodec, K, V, cache, rope=rope)
    q = synth.query_inputs_torch(w, Lq=w.Lq)
    ws = torch.empty(native.attention_bidir_workspace(ncodec, w.B, w.Hq, w.Lq), dtype=torch.uint8,
                     device="cuda")
    scale = 1 / math.sqrt(w.d)
    good = torch.empty((w.B, w.Hq, w.Lq, w.d), dtype=torch.float32, device="cuda")
    native.attention_bidir(ncodec, q, cache, w.T, scale, good, ws, rope=rope)
    torch.cuda.synchronize()
    assert torch.isfinite(good).all()

    monkeypatch.setenv("TQ_WAIT_LIMIT", "0")
    bad = torch.zeros_like(good)
    native.attention_bidir(ncodec, q, cache, w.T, scale, bad, ws, rope=rope)
    torch.cuda.synchronize()
    assert torch.isnan(bad).all()

    monkeypatch.delenv("TQ_WAIT_LIMIT")
    again = torch.empty_like(good)
    native.attention_bidir(ncodec, q, cache, w.T, scale, again, ws, rope=rope)
    torch.cuda.synchronize()
    assert torch.equal(again, good)


def test_scan_wait_give_up_is_reported(monkeypatch):
    D, n, nq, k = 1536, 3000, 40, 10
    w = synth.VECTOR_SEARCH
    ncodec = native.Codec(D, w.bits, True, 4, synth.rotation_signs(D, w.seed), synth.qjl_matrix_bf16(D, w.seed))
    x = torch.from_numpy(synth.unit_rows(n, D, 77, 0)).cuda()
    kcode = torch.empty((n, ncodec.planes_k, D // 8), dtype=torch.uint8, device="cuda")
    kscale = torch.empty((n, 2), dtype=torch.float16, device="cuda")
    iws = torch.empty(native.index_workspace(ncodec, n), dtype=torch.uint8, device="cuda")
    native.index_build(ncodec, x, kcode, kscale, iws)
    qd = torch.from_numpy(synth.unit_rows(nq, D, 77, 2)).cuda()
    ws = torch.empty(native.scan_workspace(ncodec, n, nq, k), dtype=torch.uint8, device="cuda")

    def scan():
        idx = torch.zeros((nq, k), dtype=torch.int32, device="cuda")
        score = torch.zeros((nq, k), dtype=torch.float32, device="cuda")
        native.scan_topk(ncodec, kcode, kscale, qd, k, idx, score, ws)
        torch.cuda.synchronize()
        return idx.cpu(), score.cpu()

    gi, gs = scan()
    assert (gi >= 0).all() and (gi < n).all() and torch.isfinite(gs).all()

    monkeypatch.setenv("TQ_WAIT_LIMIT", "0")
    bi, bs = scan()
    assert (bi == -1).all() and torch.isnan(bs).all()

    monkeypatch.delenv("TQ_WAIT_LIMIT")
    ai, as_ = scan()
    assert torch.equal(ai, gi) and torch.equal(as_, gs)


def test_tile_quantize_wait_give_up_sets_status_bit(monkeypatch):
    # a bf16 call of >= 256 token groups takes the tile kernel
    w = synth.WORKLOADS["esm_prefill"].scaled(B=2, Hq=4, Hkv=4, T=1024)
    _, ncodec = tl.codecs(w)
    K, V = synth.kv_inputs_torch(w)
    r = synth.rope_for(w, w.T)
    rope = tl.rope_device(r)

    def quantize():
        cache = native.alloc_cache(ncodec, w.B, w.Hkv, w.T)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        native.quantize_kv(ncodec, K, V, cache, rope=rope, status=status)
        torch.cuda.synchronize()
        return tl.download_cache(cache), int(status.item()) & 0xffffffff

    good, st = quantize()
    assert st == 0
    monkeypatch.setenv("TQ_WAIT_LIMIT", "0")
    _, st = quantize()
    assert st & (1 << 31)
    monkeypatch.delenv("TQ_WAIT_LIMIT")
    again, st = quantize()
    assert st == 0
    for key in ("kcode", "kscale", "vcode", "vnorm"):
        assert np.array_equal(again[key], good[key]), key


def test_index_build_wait_give_up_sets_status_bit(monkeypatch):
    D, n = 1536, 3000
    w = synth.VECTOR_SEARCH
    ncodec = native.Codec(D, w.bits, True, 4, synth.rotation_signs(D, w.seed), synth.qjl_matrix_bf16(D, w.seed))
    x = torch.from_numpy(synth.unit_rows(n, D, 78, 0)).cuda()

    def build():
        kcode = torch.empty((n, ncodec.planes_k, D // 8), dtype=torch.uint8, device="cuda")
        kscale = torch.empty((n, 2), dtype=torch.float16, device="cuda")
        ws = torch.empty(native.index_workspace(ncodec, n), dtype=torch.uint8, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        native.index_build(ncodec, x, kcode, kscale, ws, status=status)
        torch.cuda.synchronize()
        return kcode.cpu(), kscale.cpu(), int(status.item()) & 0xffffffff

    gk, gs, st = build()
    assert st == 0
    monkeypatch.setenv("TQ_WAIT_LIMIT", "0")
    _, _, st = build()
    assert st & (1 << 31)
    monkeypatch.delenv("TQ_WAIT_LIMIT")
    ak, as_, st = build()
    assert st == 0 and torch.equal(ak, gk) and torch.equal(as_, gs)
