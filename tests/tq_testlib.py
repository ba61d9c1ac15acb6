"""Helpers shared by the GPU parity tests: build matching oracle / library
codecs from a workload, move seeded inputs to the device, upload an oracle
cache, and compare codes under the boundary-window rule.

Tolerances (the acceptance bars of the hot path, with the boundary window
measured on the unit-variance scale):
* codes and signs bit-exact, except coordinates whose rotated value lies
  within 1e-5 (unit-variance scale: sqrt(d) * |u - t|) of a decision
  threshold, or signs with |S r|_i / rho < 1e-5; mismatches must all be in the
  window and number at most 1e-4 of the coordinates.  Sign parity is checked
  on rows whose codes all match (a code flip changes the residual).
* dequantized rows and logits within 1e-3 relative; attention output within
  2e-3 max-abs (per-channel-scale normalised for scaled workloads).
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import codec as oc
from rotated_codebook_kv_tq_b200 import native, synth

CODE_WINDOW = 1e-5
SIGN_WINDOW = 1e-5
MISMATCH_CAP = 1e-4


def require_cuda():
    assert torch.cuda.is_available(), "GPU test needs CUDA"
    from rotated_codebook_kv_tq_b200.build import build
    build()


def codecs(w: synth.Workload, seed_offset: int = 0, haar: bool = False):
    """Matching oracle and library codecs.  haar: a dense Haar rotation from
    the workload's Gaussian matrix, factorised by each side on its own."""
    D = synth.rotation_signs(w.d, w.seed + seed_offset)
    S = synth.qjl_matrix_bf16(w.d, w.seed + seed_offset) if w.qjl_k else None
    if haar:
        from oracle.rotation import haar_rotation
        G = synth.haar_gaussian(w.d, w.seed + seed_offset)
        ocodec = oc.make_codec(w.d, w.bits_k, w.qjl_k, w.bits_v, D, S, Pi=haar_rotation(G))
        ncodec = native.Codec(w.d, w.bits_k, w.qjl_k, w.bits_v, None, S,
                              rotation=native.haar_rotation(G))
        return ocodec, ncodec
    ocodec = oc.make_codec(w.d, w.bits_k, w.qjl_k, w.bits_v, D, S)
    ncodec = native.Codec(w.d, w.bits_k, w.qjl_k, w.bits_v, D, S)
    return ocodec, ncodec


def to_device(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def rope_device(rope):
    if rope is None:
        return None
    return (torch.from_numpy(rope[0]).cuda(), torch.from_numpy(rope[1]).cuda())


def upload_cache(ocache: dict, ncodec, B: int, Hkv: int) -> native.Cache:
    c = native.alloc_cache(ncodec, B, Hkv, ocache["rows_cap"])
    c.kcode.copy_(torch.from_numpy(ocache["kcode"]))
    c.kscale.copy_(torch.from_numpy(ocache["kscale"]))
    c.vcode.copy_(torch.from_numpy(ocache["vcode"].view(np.int32)))
    c.vnorm.copy_(torch.from_numpy(ocache["vnorm"]))
    return c


def download_cache(c: native.Cache) -> dict:
    return dict(kcode=c.kcode.cpu().numpy(), kscale=c.kscale.cpu().numpy(),
                vcode=c.vcode.cpu().numpy().view(np.uint32), vnorm=c.vnorm.cpu().numpy(),
                rows_cap=c.rows_cap)


def code_window(u: np.ndarray, thresholds32: np.ndarray, d: int) -> np.ndarray:
    """True where sqrt(d) * |u - t_k| < CODE_WINDOW for some threshold."""
    dist = np.min(np.abs(u[..., None] - thresholds32.astype(np.float64)), axis=-1)
    return math.sqrt(d) * dist < CODE_WINDOW


def fp16_close(a: np.ndarray, b: np.ndarray, ulps: int = 1) -> np.ndarray:
    ia = a.astype(np.float16).view(np.int16).astype(np.int32)
    ib = b.astype(np.float16).view(np.int16).astype(np.int32)
    return np.abs(ia - ib) <= ulps


def compare_rows(gpu: dict, ref: dict, ocodec, b: int, h: int, rows: np.ndarray,
                 enc_k: dict, enc_v: dict, stats: dict) -> None:
    """Compare the GPU cache rows ``rows`` of (b, h) with the oracle encodings
    (``enc_k``/``enc_v`` indexed by position in ``rows``)."""
    d = ocodec.d
    ik, sg, nk, rk = oc.unpack_keys(gpu["kcode"][b, h, rows], gpu["kscale"][b, h, rows], ocodec)
    # keys: codes
    cm = ik != enc_k["idx"]
    win = code_window(enc_k["u"], ocodec.cb_k.thresholds32, d)
    assert not np.any(cm & ~win), f"key code mismatch outside window at {np.argwhere(cm & ~win)[:5]}"
    stats["code_mism"] += int(cm.sum())
    stats["code_window"] += int(win.sum())
    ok_rows = ~np.any(cm, axis=1)
    if ocodec.qjl_k:
        sm = (sg != enc_k["sigma"]) & ok_rows[:, None]
        rho = np.where(enc_k["rho"] > 0, enc_k["rho"], 1.0)
        swin = np.abs(enc_k["z"]) / rho[:, None] < SIGN_WINDOW
        assert not np.any(sm & ~swin), f"sign mismatch outside window at {np.argwhere(sm & ~swin)[:5]}"
        stats["sign_mism"] += int(sm.sum())
        stats["sign_window"] += int(swin.sum())
        assert np.all(fp16_close(rk[ok_rows], enc_k["rho16"][ok_rows]))
    assert np.all(fp16_close(nk, enc_k["nu16"]))
    # values (column groups)
    iv, nv = oc.unpack_values(gpu["vcode"][b, h], gpu["vnorm"][b, h], ocodec)
    vm = iv[rows] != enc_v["idx"]
    vwin = code_window(enc_v["u"], ocodec.cb_v.thresholds32, d)
    assert not np.any(vm & ~vwin), f"value code mismatch outside window at {np.argwhere(vm & ~vwin)[:5]}"
    stats["code_mism"] += int(vm.sum())
    stats["code_window"] += int(vwin.sum())
    assert np.all(fp16_close(nv[rows], enc_v["nu16"]))
    stats["coords"] += 2 * enc_k["idx"].size


def new_stats():
    return dict(code_mism=0, sign_mism=0, code_window=0, sign_window=0, coords=0)


# Boundary-window accounting of every parity check in this session: the
# mismatch count, the window population and the fraction of coordinates are
# printed in pytest's terminal summary (conftest.py) so they appear in the log.
MISMATCH_REPORT: list = []


def assert_mismatch_budget(stats: dict, label: str = "") -> None:
    import os
    frac = (stats["code_mism"] + stats["sign_mism"]) / max(1, stats["coords"])
    label = label or os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    MISMATCH_REPORT.append(dict(stats, test=label, fraction=frac))
    assert frac <= MISMATCH_CAP, stats


def channel_scale_of_values(w: synth.Workload) -> np.ndarray:
    """[Hkv, d] synthetic scale of each value channel (ones when unscaled)."""
    return synth.channel_scales(w)[1]
