"""A bounded wait that gives up is reported, and the GPU stays usable.

Every wait inside the tensor-core decode kernel polls an mbarrier a bounded
number of times.  TQ_WAIT_LIMIT (read at each launch) sets that bound; 0 makes
every wait of the main loop give up at once, which is how this test makes the
failure happen without faulting or hanging anything: the kernel drains its own
copies and MMAs, sets the call's status word, and the split-K combine writes
NaN for every output instead of merging incomplete partials.  The next call
without the override must be exact again."""
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
