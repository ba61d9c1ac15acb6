"""Decode for callers that cannot allocate device memory.

tq_attention_decode_noalloc takes no workspace: its scratch is a static array
inside the library, for callers (plugins in hosts that own every allocation,
serving processes with all HBM reserved) that cannot call cudaMalloc.  These
tests call it through the C ABI and check it against tq_attention_decode,
which uses a caller-allocated workspace, on two calls in a row with different
shapes (the second call must not be affected by what the first left in the
shared scratch).  The file is named to be collected last."""
import math

import pytest
import torch

from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

pytestmark = pytest.mark.gpu

TOL = 2e-3   # output tolerance of the decode parity tests (max-abs, per channel scale)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


def _setup(w, seed_salt):
    _, ncodec = tl.codecs(w)
    K, V = synth.kv_inputs_torch(w, seed_salt=seed_salt)
    rows_cap = (w.T + 31) // 32 * 32
    r = synth.rope_for(w, rows_cap)
    rope = tl.rope_device(r)
    cache = native.alloc_cache(ncodec, w.B, w.Hkv, rows_cap)
    native.quantize_kv(ncodec, K, V, cache, rope=rope)
    q = synth.query_inputs_torch(w, seed_salt=seed_salt)[:, :, 0].contiguous()
    return ncodec, cache, q, rope


def _reference(ncodec, cache, q, w, lens, rope, splits):
    ws = torch.empty(native.attention_workspace(ncodec, w.B, w.Hq, splits), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device="cuda")
    native.attention_decode(ncodec, q, cache, w.T, 1 / math.sqrt(w.d), out, ws, seq_lens=lens,
                            rope=rope, num_splits=splits)
    return out


def test_noalloc_matches_workspace_decode_two_calls():
    cases = [
        (synth.WORKLOADS["llama_decode"].scaled(B=2, T=3000), [3000, 1777], 24, 0),
        (synth.WORKLOADS["long_decode"].scaled(B=1, Hq=16, Hkv=4, T=5000), None, 64, 1),
    ]
    for w, lens, splits, salt in cases:
        ncodec, cache, q, rope = _setup(w, salt)
        sl = None if lens is None else torch.tensor(lens, dtype=torch.int32, device="cuda")
        ref = _reference(ncodec, cache, q, w, sl, rope, splits)
        out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
        native.attention_decode_noalloc(ncodec, q, cache, w.T, 1 / math.sqrt(w.d), out,
                                        seq_lens=sl, rope=rope, num_splits=splits)
        torch.cuda.synchronize()
        vscale = torch.as_tensor(tl.channel_scale_of_values(w), dtype=torch.float32,
                                 device="cuda").repeat_interleave(w.G, dim=0)
        err = ((out - ref).abs() / vscale[None]).max().item()
        assert err <= TOL, (w.name, err)
        assert torch.isfinite(out).all()


def test_noalloc_leftovers_of_a_larger_call_do_not_leak():
    """A call with many splits over many heads fills most of the shared
    scratch; the next call, with fewer splits and unequal lengths (so some of
    its chunks are empty), must not pick up any of those partials."""
    big = synth.WORKLOADS["long_decode"].scaled(B=4, Hq=32, Hkv=8, T=4096)
    ncodec, cache, q, rope = _setup(big, 2)
    out = torch.empty((big.B, big.Hq, big.d), dtype=torch.float32, device="cuda")
    native.attention_decode_noalloc(ncodec, q, cache, big.T, 1 / math.sqrt(big.d), out,
                                    rope=rope, num_splits=128)
    small = big.scaled(B=3)
    lens = torch.tensor([4096, 700, 1], dtype=torch.int32, device="cuda")
    q3 = q[:3].contiguous()
    cache3 = native.Cache(cache.kcode[:3], cache.kscale[:3], cache.vcode[:3], cache.vnorm[:3], 3,
                          cache.Hkv, cache.rows_cap)
    ref = _reference(ncodec, cache3, q3, small, lens, rope, 16)
    got = torch.full_like(ref, float("nan"))
    native.attention_decode_noalloc(ncodec, q3, cache3, small.T, 1 / math.sqrt(small.d), got,
                                    seq_lens=lens, rope=rope, num_splits=16)
    torch.cuda.synchronize()
    vscale = torch.as_tensor(tl.channel_scale_of_values(small), dtype=torch.float32,
                             device="cuda").repeat_interleave(small.G, dim=0)
    err = ((got - ref).abs() / vscale[None]).max().item()
    assert err <= TOL, err


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    w = synth.WORKLOADS["long_decode"]
    _, ncodec = tl.codecs(w)
    cache = native.alloc_cache(ncodec, 64, 8, 64)
    q = torch.zeros((64, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((64, 32, 128), dtype=torch.float32, device="cuda")
    need = native.attention_workspace(ncodec, 64, 32, 128)
    assert need > native.NOALLOC_SCRATCH_BYTES
    with pytest.raises(native.TqError) as e:
        native.attention_decode_noalloc(ncodec, q, cache, 64, 0.1, out, num_splits=128)
    assert e.value.code == native.TQ_ERR_WORKSPACE
