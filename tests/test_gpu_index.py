"""Vector-search index build and top-k scan (d = 1536, TurboQuant_prod at 4
bits) through the C ABI, against the oracle.

Encode parity: codes and signs bit-exact up to the boundary windows of the KV
tests (coordinates within 1e-5 of a threshold on the unit-variance scale, signs
with |S r|_i / rho < 1e-5), norms within one fp16 ulp.  Scan parity on an
oracle-encoded database, for both the tensor-core scan and the lookup-table
scan: every returned score within a tolerance of the oracle's score of that
row (relative to the RMS of the query's oracle scores; see LUT_SCORE_TOL and
MMA_SCORE_TOL), the returned list ordered by (score descending, index
ascending), the returned set equal to the oracle's top-k up to rows whose
oracle scores lie within twice that tolerance of the k-th best, and any two
returned rows further apart than that in the oracle's order.
"""
import numpy as np
import pytest
import torch

from oracle import codec as oc
from oracle import scan as oscan
from rotated_codebook_kv_tq_b200 import native, synth
import tq_testlib as tl

pytestmark = pytest.mark.gpu

D = 1536
# Score tolerances relative to the RMS of a query's oracle scores.  The LUT
# path scores in fp32 and takes the survey's 1e-3 reading as is.  The
# tensor-core path rounds both operands of every product to fp16 (rows
# [c[idx] | rho (2 sigma - 1)], queries scaled by a power of two) and sums
# 3072 of them: emulating that arithmetic on the oracle gives up to 1.1e-3 of
# the RMS on 3000 rows, so its bound is the derived 3e-3.
LUT_SCORE_TOL = 1e-3
MMA_SCORE_TOL = 3e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    tl.require_cuda()


@pytest.fixture(scope="module")
def codecs():
    w = synth.VECTOR_SEARCH
    Dv = synth.rotation_signs(D, w.seed)
    S = synth.qjl_matrix_bf16(D, w.seed)
    return (oc.make_codec(D, w.bits, True, 4, Dv, S), native.Codec(D, w.bits, True, 4, Dv, S))


def _encode_gpu(ncodec, x: torch.Tensor):
    n = x.shape[0]
    planes = ncodec.planes_k
    kcode = torch.empty((n, planes, D // 8), dtype=torch.uint8, device="cuda")
    kscale = torch.empty((n, 2), dtype=torch.float16, device="cuda")
    ws = torch.empty(native.index_workspace(ncodec, n), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    native.index_build(ncodec, x, kcode, kscale, ws, status=status)
    return kcode, kscale, status


def _check_codes(ocodec, gk: np.ndarray, gs: np.ndarray, enc: dict, stats: dict):
    ik, sg, nk, rk = oc.unpack_keys(gk, gs, ocodec)
    cm = ik != enc["idx"]
    win = tl.code_window(enc["u"], ocodec.cb_k.thresholds32, D)
    assert not np.any(cm & ~win), f"code mismatch outside window at {np.argwhere(cm & ~win)[:5]}"
    ok = ~np.any(cm, axis=1)
    sm = (sg != enc["sigma"]) & ok[:, None]
    rho = np.where(enc["rho"] > 0, enc["rho"], 1.0)
    swin = np.abs(enc["z"]) / rho[:, None] < tl.SIGN_WINDOW
    assert not np.any(sm & ~swin), f"sign mismatch outside window at {np.argwhere(sm & ~swin)[:5]}"
    assert np.all(tl.fp16_close(nk, enc["nu16"]))
    assert np.all(tl.fp16_close(rk[ok], enc["rho16"][ok]))
    stats["code_mism"] += int(cm.sum())
    stats["sign_mism"] += int(sm.sum())
    stats["coords"] += 2 * cm.size


def _check_topk(s: np.ndarray, gi: np.ndarray, gv: np.ndarray, k: int, rel: float):
    """s: oracle scores [nq, n]; gi/gv: GPU indices/scores [nq, k].

    With tol = rel * RMS of the query's oracle scores: every returned score is
    within tol of the oracle's score of that row; the list is ordered by
    (-score, index); every row whose oracle score beats the k-th best by more
    than 2 tol is returned and nothing returned falls below it by more than
    2 tol; and any two returned rows whose oracle scores differ by more than
    2 tol appear in the oracle's order."""
    for i in range(s.shape[0]):
        tol = rel * float(np.sqrt(np.mean(s[i] ** 2)))
        idx = gi[i].astype(np.int64)
        assert len(set(idx.tolist())) == k and idx.min() >= 0 and idx.max() < s.shape[1]
        assert np.all(np.abs(gv[i] - s[i, idx]) <= tol), (i, np.max(np.abs(gv[i] - s[i, idx])) / tol)
        for a in range(k - 1):   # ordered by (-score, index)
            assert gv[i, a] > gv[i, a + 1] or (gv[i, a] == gv[i, a + 1] and idx[a] < idx[a + 1])
        ref_idx, ref_val = oscan.topk(s[i:i + 1], k)
        kth = ref_val[0, -1]
        assert np.all(s[i, idx] >= kth - 2 * tol)
        must = ref_idx[0][ref_val[0] > kth + 2 * tol]
        assert set(must.tolist()) <= set(idx.tolist())
        os_ = s[i, idx]
        for a in range(k):
            for b in range(a + 1, k):
                assert os_[a] >= os_[b] - 2 * tol, (i, a, b)


def _special_rows(x: np.ndarray) -> np.ndarray:
    x = x.copy()
    x[3] = 0.0                  # zero row
    x[5, 17] = np.nan           # non-finite -> stored as a zero row
    x[9, 100] = np.inf
    x[11] *= 1e6                # norm above the fp16 range -> zero row
    return x


@pytest.mark.parametrize("n", [1000, 37])
def test_index_build_parity(codecs, n):
    """n = 1000 spans 8 GEMM row tiles with a ragged tail; 37 is a single partial tile."""
    ocodec, ncodec = codecs
    x = _special_rows(synth.unit_rows(n, D, 40 + n, 0)) if n > 20 else synth.unit_rows(n, D, 40 + n, 0)
    kcode, kscale, status = _encode_gpu(ncodec, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    enc = oc.quantize_keys(x.astype(np.float64), ocodec)
    stats = tl.new_stats()
    _check_codes(ocodec, kcode.cpu().numpy(), kscale.cpu().numpy(), enc, stats)
    tl.assert_mismatch_budget(stats)
    assert int(status.item()) == int(enc["bad"].sum())
    if n > 20:
        assert int(enc["bad"].sum()) == 3
        assert np.all(kscale.cpu().numpy()[[3, 5, 9, 11], 0] == 0)


@pytest.mark.parametrize("n,nq,k", [(1000, 130, 10), (37, 3, 16), (300, 1, 1), (20000, 64, 10)])
def test_scan_topk_parity(codecs, n, nq, k):
    """Scan over an oracle-encoded database (several query blocks, ragged row
    tiles, k at its limits, and a 20000-row case spread over many CTAs)."""
    ocodec, ncodec = codecs
    x = synth.unit_rows(n, D, 60 + n, 0).astype(np.float64)
    if n > 20:
        x[3] = 0.0
    q = synth.unit_rows(nq, D, 60 + n, 2)
    enc = oc.quantize_keys(x, ocodec)
    kc, ks = oc.pack_keys(enc, ocodec)
    s = oscan.scores(q.astype(np.float64), kc, ks, ocodec)
    kcode = torch.from_numpy(kc).cuda()
    kscale = torch.from_numpy(ks).cuda()
    qd = torch.from_numpy(q).cuda()
    idx = torch.empty((nq, k), dtype=torch.int32, device="cuda")
    score = torch.empty((nq, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(native.scan_workspace(ncodec, n, nq, k), dtype=torch.uint8, device="cuda")
    native.scan_topk(ncodec, kcode, kscale, qd, k, idx, score, ws)
    torch.cuda.synchronize()
    _check_topk(s, idx.cpu().numpy(), score.cpu().numpy().astype(np.float64), k, MMA_SCORE_TOL)
    # the lookup-table path on the same database and queries: fp32 scores
    idx2 = torch.empty_like(idx)
    score2 = torch.empty_like(score)
    native.scan_topk_lut(ncodec, kcode, kscale, qd, k, idx2, score2, ws)
    torch.cuda.synchronize()
    _check_topk(s, idx2.cpu().numpy(), score2.cpu().numpy().astype(np.float64), k, LUT_SCORE_TOL)


def test_scan_rejects_bad_arguments(codecs):
    _, ncodec = codecs
    kcode = torch.zeros((8, 4, D // 8), dtype=torch.uint8, device="cuda")
    kscale = torch.zeros((8, 2), dtype=torch.float16, device="cuda")
    q = torch.zeros((2, D), device="cuda")
    idx = torch.empty((2, 17), dtype=torch.int32, device="cuda")
    score = torch.empty((2, 17), device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    for k in (0, 9, 17):   # k > n and k > 16 are rejected before any launch
        with pytest.raises(native.TqError) as e:
            native.scan_topk(ncodec, kcode, kscale, q, k, idx, score, ws)
        assert e.value.code == native.TQ_ERR_INVALID_ARG
    small = native.Codec(128, 4, True, 4, synth.rotation_signs(128, 0), synth.qjl_matrix_bf16(128, 0))
    with pytest.raises(native.TqError) as e:
        native.scan_topk(small, kcode, kscale, q, 4, idx, score, ws)
    assert e.value.code == native.TQ_ERR_UNSUPPORTED
    with pytest.raises(native.TqError) as e:
        native.scan_topk(ncodec, kcode, kscale, q, 4, idx, score, ws[:64])
    assert e.value.code == native.TQ_ERR_WORKSPACE


def test_vector_search_fullsize_sampled(codecs):
    """10^6 x 1536 unit rows, 1024 unit queries, top-10, in the launch
    configuration the benchmark times.  Encode: 3000 sampled rows (both ends of
    every 65536-row batch included) against the oracle.  Scan: for 12 sampled
    queries, the oracle scores of the returned rows match, and no row among the
    300 with the largest exact inner product <q, x> has an oracle score above
    the returned k-th score (plus tolerance) without being returned."""
    ocodec, ncodec = codecs
    w = synth.VECTOR_SEARCH
    X, Q = synth.search_inputs(w)
    xd = torch.from_numpy(X).cuda()
    kcode, kscale, status = _encode_gpu(ncodec, xd)
    qd = torch.from_numpy(Q).cuda()
    idx = torch.empty((w.nq, w.k), dtype=torch.int32, device="cuda")
    score = torch.empty((w.nq, w.k), dtype=torch.float32, device="cuda")
    ws = torch.empty(native.scan_workspace(ncodec, w.n, w.nq, w.k), dtype=torch.uint8, device="cuda")
    native.scan_topk(ncodec, kcode, kscale, qd, w.k, idx, score, ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    del xd
    rng = np.random.default_rng(7)
    edges = np.concatenate([[b, b + 65535] for b in range(0, w.n, 65536)])
    rows = np.unique(np.concatenate([rng.choice(w.n, 3000 - len(edges), replace=False),
                                     np.clip(edges, 0, w.n - 1)]))
    gk, gs = kcode[torch.from_numpy(rows).cuda()].cpu().numpy(), kscale[torch.from_numpy(rows).cuda()].cpu().numpy()
    enc = oc.quantize_keys(X[rows].astype(np.float64), ocodec)
    stats = tl.new_stats()
    _check_codes(ocodec, gk, gs, enc, stats)
    tl.assert_mismatch_budget(stats)

    gi, gv = idx.cpu().numpy().astype(np.int64), score.cpu().numpy().astype(np.float64)
    for qi in rng.choice(w.nq, 12, replace=False):
        true_ip = X @ Q[qi]
        cand = np.argpartition(-true_ip, 300)[:300]
        pool = np.unique(np.concatenate([cand, gi[qi]]))
        e = oc.quantize_keys(X[pool].astype(np.float64), ocodec)
        kc, ks = oc.pack_keys(e, ocodec)
        sp = oscan.scores(Q[qi:qi + 1].astype(np.float64), kc, ks, ocodec)[0]
        where = {int(j): t for t, j in enumerate(pool)}
        # RMS of the exact inner products over all rows stands in for the
        # RMS of the query's oracle scores (slightly smaller: conservative)
        tol = MMA_SCORE_TOL * float(np.sqrt(np.mean(true_ip.astype(np.float64) ** 2)))
        mine = np.array([sp[where[int(j)]] for j in gi[qi]])
        assert np.all(np.abs(gv[qi] - mine) <= tol), (qi, gv[qi], mine)
        kth = gv[qi, -1]
        better = pool[sp > kth + 2 * tol]
        assert set(better.tolist()) <= set(gi[qi].tolist()), qi


@pytest.mark.parametrize("bits", [2, 3])   # key MSE bits 1 and 2 (+ QJL)
def test_index_and_scan_other_bit_widths(bits):
    """Index build and scan parity for the narrower key codecs the
    vector-search calls accept (the 4-bit default covers 3 MSE bits)."""
    w = synth.VECTOR_SEARCH
    Dv = synth.rotation_signs(D, w.seed)
    S = synth.qjl_matrix_bf16(D, w.seed)
    ocodec = oc.make_codec(D, bits, True, 4, Dv, S)
    ncodec = native.Codec(D, bits, True, 4, Dv, S)
    n, nq, k = 700, 70, 10
    x = synth.unit_rows(n, D, 80 + bits, 0)
    kcode, kscale, status = _encode_gpu(ncodec, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    enc = oc.quantize_keys(x.astype(np.float64), ocodec)
    stats = tl.new_stats()
    _check_codes(ocodec, kcode.cpu().numpy(), kscale.cpu().numpy(), enc, stats)
    tl.assert_mismatch_budget(stats)
    # scan over the oracle's own codes
    kc, ks = oc.pack_keys(enc, ocodec)
    q = synth.unit_rows(nq, D, 80 + bits, 2)
    s = oscan.scores(q.astype(np.float64), kc, ks, ocodec)
    idx = torch.empty((nq, k), dtype=torch.int32, device="cuda")
    score = torch.empty((nq, k), dtype=torch.float32, device="cuda")
    ws = torch.empty(native.scan_workspace(ncodec, n, nq, k), dtype=torch.uint8, device="cuda")
    kcd, ksd, qd = torch.from_numpy(kc).cuda(), torch.from_numpy(ks).cuda(), torch.from_numpy(q).cuda()
    native.scan_topk(ncodec, kcd, ksd, qd, k, idx, score, ws)
    torch.cuda.synchronize()
    _check_topk(s, idx.cpu().numpy(), score.cpu().numpy().astype(np.float64), k, MMA_SCORE_TOL)
    native.scan_topk_lut(ncodec, kcd, ksd, qd, k, idx, score, ws)
    torch.cuda.synchronize()
    _check_topk(s, idx.cpu().numpy(), score.cpu().numpy().astype(np.float64), k, LUT_SCORE_TOL)


def test_index_rejects_four_mse_bits():
    Dv = synth.rotation_signs(D, 4)
    ncodec = native.Codec(D, 5, True, 4, Dv, synth.qjl_matrix_bf16(D, 4))
    x = torch.zeros((8, D), device="cuda")
    with pytest.raises(native.TqError) as e:
        _encode_gpu(ncodec, x)
    assert e.value.code == native.TQ_ERR_UNSUPPORTED
