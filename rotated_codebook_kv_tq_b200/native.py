"""ctypes binding of ``libtq_b200.so`` (the C ABI declared in ``include/tq.h``).

Argument marshalling only: every step of the codec runs in the library's CUDA
kernels.  Tensors are PyTorch tensors used for device memory and streams.  If
the shared library is missing the import of this module's functions raises:
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtq_b200.so")

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_ALIGNMENT, TQ_ERR_CUDA, TQ_ERR_WORKSPACE = range(6)
TQ_F32, TQ_BF16 = 0, 1

EXPORTS = [
    "tq_build_codebook", "tq_codec_create", "tq_codec_destroy", "tq_codec_codebooks",
    "tq_cache_bytes", "tq_quantize_kv", "tq_attention_workspace", "tq_attention_decode",
    "tq_attention_logits", "tq_decode_step", "tq_decode_step_host", "tq_attention_decode_noalloc", "tq_attention_bidir_workspace",
    "tq_attention_bidir", "tq_index_workspace", "tq_index_build", "tq_scan_workspace",
    "tq_scan_topk", "tq_scan_topk_lut", "tq_dequantize", "tq_split_channels",
    "tq_quantize_kv_split", "tq_attention_split_workspace", "tq_attention_decode_split",
    "tq_dequantize_split", "tq_haar_rotation", "tq_fq_build_codebook", "tq_fq_codec_create", "tq_fq_codec_destroy",
    "tq_fq_codec_codebooks", "tq_fq_cache_bytes", "tq_fq_quantize_kv", "tq_fq_attention_workspace",
    "tq_fq_attention_decode", "tq_fq_dequantize", "tq_set_timing_events", "tq_launch_count",
    "tq_last_error",
]


class TqError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"tq status {code}: {msg}")
        self.code = code


class CodecDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("bits_k", ctypes.c_int), ("qjl_k", ctypes.c_int),
                ("bits_v", ctypes.c_int), ("rotation_signs", ctypes.c_void_p),
                ("qjl_bf16", ctypes.c_void_p), ("rotation", ctypes.c_void_p)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("kcode", ctypes.c_void_p), ("kscale", ctypes.c_void_p),
                ("vcode", ctypes.c_void_p), ("vnorm", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Hkv", ctypes.c_int), ("rows_cap", ctypes.c_int64)]


class FqCodecDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("bits_k", ctypes.c_int), ("bits_v", ctypes.c_int),
                ("rotation_signs", ctypes.c_void_p)]


class SplitDesc(ctypes.Structure):
    _fields_ = [("hi", ctypes.c_void_p), ("lo", ctypes.c_void_p), ("channels", ctypes.c_void_p)]


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m rotated_codebook_kv_tq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
        sz = ctypes.c_size_t
        L.tq_build_codebook.argtypes = [i32, i32, vp, vp, vp]
        L.tq_codec_create.argtypes = [ctypes.POINTER(CodecDesc), ctypes.POINTER(vp)]
        L.tq_codec_destroy.argtypes = [vp]
        L.tq_codec_destroy.restype = None
        L.tq_codec_codebooks.argtypes = [vp, vp, vp, vp, vp]
        L.tq_cache_bytes.argtypes = [vp, i32, i32, i64, ctypes.POINTER(sz)]
        L.tq_quantize_kv.argtypes = [vp, vp, vp, i32, i32, i32, i32, i64, i64, i64, vp, vp, i64,
                                     ctypes.POINTER(CacheDesc), i64, vp, vp]
        L.tq_attention_workspace.argtypes = [vp, i32, i32, i32, ctypes.POINTER(sz)]
        L.tq_attention_decode.argtypes = [vp, vp, i32, i32, i32, i32, ctypes.POINTER(CacheDesc),
                                          vp, i32, f32, vp, vp, i32, vp, sz, vp, vp]
        L.tq_attention_logits.argtypes = L.tq_attention_decode.argtypes[:-1] + [vp, vp]
        L.tq_decode_step.argtypes = [vp, vp, vp, i32, vp, i32, i32, i32, i32,
                                     ctypes.POINTER(CacheDesc), i32, ctypes.c_float, vp, vp, i32,
                                     vp, sz, vp, vp]
        L.tq_decode_step_host.argtypes = [vp, vp, vp, sz, i32, i32, i32, i32, i32,
                                          ctypes.POINTER(CacheDesc), i32, ctypes.c_float, vp, vp, i32,
                                          vp, sz, vp, vp, vp]
        L.tq_attention_decode_noalloc.argtypes = [vp, vp, i32, i32, i32, i32,
                                                  ctypes.POINTER(CacheDesc), vp, i32, f32, vp,
                                                  vp, i32, vp, vp]
        L.tq_attention_bidir_workspace.argtypes = [vp, i32, i32, i32, ctypes.POINTER(sz)]
        L.tq_attention_bidir.argtypes = [vp, vp, i32, i32, i32, i32, i32, ctypes.POINTER(CacheDesc),
                                         i32, f32, vp, vp, vp, sz, vp, vp]
        L.tq_index_workspace.argtypes = [vp, i64, ctypes.POINTER(sz)]
        L.tq_index_build.argtypes = [vp, vp, i64, vp, vp, vp, vp, sz, vp]
        L.tq_scan_workspace.argtypes = [vp, i64, i32, i32, ctypes.POINTER(sz)]
        L.tq_scan_topk.argtypes = [vp, vp, vp, i64, vp, i32, i32, vp, vp, vp, sz, vp]
        L.tq_scan_topk_lut.argtypes = [vp, vp, vp, i64, vp, i32, i32, vp, vp, vp, sz, vp]
        L.tq_dequantize.argtypes = [vp, ctypes.POINTER(CacheDesc), i32, i64, i64, vp, vp]
        sp, cp = ctypes.POINTER(SplitDesc), ctypes.POINTER(CacheDesc)
        L.tq_split_channels.argtypes = [vp, i32, i32, vp]
        L.tq_quantize_kv_split.argtypes = [sp, vp, vp, i32, i32, i32, i32, i64, i64, i64, vp, vp,
                                           i64, cp, cp, i64, vp, vp]
        L.tq_attention_split_workspace.argtypes = [sp, i32, i32, i32, ctypes.POINTER(sz)]
        L.tq_attention_decode_split.argtypes = [sp, vp, i32, i32, i32, i32, cp, cp, vp, i32,
                                                ctypes.c_float, vp, vp, i32, vp, sz, vp, vp]
        L.tq_dequantize_split.argtypes = [sp, cp, cp, i32, i64, i64, vp, vp]
        L.tq_haar_rotation.argtypes = [i32, vp, vp]
        L.tq_fq_build_codebook.argtypes = [i32, i32, vp, vp]
        L.tq_fq_codec_create.argtypes = [ctypes.POINTER(FqCodecDesc), ctypes.POINTER(vp)]
        L.tq_fq_codec_destroy.argtypes = [vp]
        L.tq_fq_codec_destroy.restype = None
        L.tq_fq_codec_codebooks.argtypes = [vp, vp, vp]
        L.tq_fq_cache_bytes.argtypes = [vp, i32, i32, i64, ctypes.POINTER(sz)]
        L.tq_fq_quantize_kv.argtypes = L.tq_quantize_kv.argtypes
        L.tq_fq_attention_workspace.argtypes = [vp, i32, i32, i32, ctypes.POINTER(sz)]
        L.tq_fq_attention_decode.argtypes = L.tq_attention_decode.argtypes
        L.tq_fq_dequantize.argtypes = L.tq_dequantize.argtypes
        L.tq_set_timing_events.argtypes = [vp, vp]
        L.tq_launch_count.argtypes = []
        L.tq_launch_count.restype = ctypes.c_uint64
        L.tq_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def check(code: int) -> None:
    if code != TQ_OK:
        raise TqError(code, lib().tq_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


_RAW_STREAM = None


def _stream(stream) -> Optional[int]:
    """The cudaStream_t of ``stream`` (None: torch's current stream)."""
    global _RAW_STREAM
    if stream is None:
        if _RAW_STREAM is None:
            import torch
            # torch's direct query of the current raw stream (no Stream
            # object per call); the public route when it is missing
            raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
            dev = getattr(torch._C, "_cuda_getDevice", None)
            _RAW_STREAM = ((lambda: raw(dev())) if raw is not None and dev is not None
                           else (lambda: torch.cuda.current_stream().cuda_stream))
        return _RAW_STREAM()
    return stream if isinstance(stream, int) else stream.cuda_stream


# ---------------------------------------------------------------- codebook

def build_codebook(d: int, bits: int):
    """tq_build_codebook -> (centroids fp32, thresholds fp32, mse_per_coord)."""
    c = np.zeros(1 << bits, np.float32)
    t = np.zeros((1 << bits) - 1 if bits > 0 else 0, np.float32)
    mse = ctypes.c_double(0.0)
    check(lib().tq_build_codebook(d, bits, c.ctypes.data, t.ctypes.data, ctypes.addressof(mse)))
    return c, t, mse.value


# ---------------------------------------------------------------- codec

class Codec:
    """Owns a ``tq_codec`` (device copies of D, S and the codebooks)."""

    def __init__(self, d: int, bits_k: int, qjl_k: bool, bits_v: int,
                 rotation_signs: Optional[np.ndarray], qjl_bf16: Optional[np.ndarray],
                 rotation: Optional[np.ndarray] = None):
        self.d, self.bits_k, self.qjl_k, self.bits_v = d, bits_k, bool(qjl_k), bits_v
        self.mse_bits_k = bits_k - 1 if qjl_k else bits_k
        self.planes_k = self.mse_bits_k + (1 if qjl_k else 0)
        signs = None if rotation_signs is None else np.ascontiguousarray(rotation_signs, dtype=np.int8)
        s = None if qjl_bf16 is None else np.ascontiguousarray(qjl_bf16, dtype=np.uint16)
        rot = None if rotation is None else np.ascontiguousarray(rotation, dtype=np.float32)
        desc = CodecDesc(d, bits_k, 1 if qjl_k else 0, bits_v,
                         None if signs is None else signs.ctypes.data,
                         None if s is None else s.ctypes.data,
                         None if rot is None else rot.ctypes.data)
        h = ctypes.c_void_p()
        check(lib().tq_codec_create(ctypes.byref(desc), ctypes.byref(h)))
        self.handle = h

    def codebooks(self):
        nk, nv = 1 << self.mse_bits_k, 1 << self.bits_v
        ck, tk = np.zeros(nk, np.float32), np.zeros(nk - 1, np.float32)
        cv, tv = np.zeros(nv, np.float32), np.zeros(nv - 1, np.float32)
        check(lib().tq_codec_codebooks(self.handle, ck.ctypes.data, tk.ctypes.data,
                                       cv.ctypes.data, tv.ctypes.data))
        return ck, tk, cv, tv

    def close(self) -> None:
        if getattr(self, "handle", None):
            lib().tq_codec_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


@dataclass
class Cache:
    """Compressed cache planes (device tensors owned by the caller)."""
    kcode: "object"
    kscale: "object"
    vcode: "object"
    vnorm: "object"
    B: int
    Hkv: int
    rows_cap: int

    def desc(self) -> CacheDesc:
        key = (self.kcode.data_ptr(), self.kscale.data_ptr(), self.vcode.data_ptr(),
               self.vnorm.data_ptr(), self.B, self.Hkv, self.rows_cap)
        cached = self.__dict__.get("_desc")
        if cached is None or cached[0] != key:
            cached = (key, CacheDesc(*key))
            self.__dict__["_desc"] = cached
        return cached[1]


def cache_bytes(codec: Codec, B: int, Hkv: int, rows_cap: int):
    out = (ctypes.c_size_t * 4)()
    check(lib().tq_cache_bytes(codec.handle, B, Hkv, rows_cap, out))
    return list(out)


def alloc_cache(codec: Codec, B: int, Hkv: int, rows_cap: int, device="cuda") -> Cache:
    import torch
    d = codec.d
    return Cache(
        kcode=torch.zeros((B, Hkv, rows_cap, codec.planes_k, d // 8), dtype=torch.uint8, device=device),
        kscale=torch.zeros((B, Hkv, rows_cap, 2), dtype=torch.float16, device=device),
        vcode=torch.zeros((B, Hkv, rows_cap // 32, codec.bits_v, d), dtype=torch.int32, device=device),
        vnorm=torch.zeros((B, Hkv, rows_cap), dtype=torch.float16, device=device),
        B=B, Hkv=Hkv, rows_cap=rows_cap)


_DTYPES = None


def _dtype_code(t) -> int:
    return _code_of(t.dtype)


def _code_of(dtype) -> int:
    global _DTYPES
    if _DTYPES is None:
        import torch
        _DTYPES = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.int16: TQ_BF16,
                   torch.uint16: TQ_BF16}
    code = _DTYPES.get(dtype)
    if code is None:
        raise TypeError(f"unsupported dtype {dtype}")
    return code


# ---------------------------------------------------------------- calls

def quantize_kv(codec: Codec, k, v, cache: Cache, row0: int = 0, rope=None, pos0: int = 0,
                status=None, stream=None) -> None:
    """tq_quantize_kv on k, v [B, Hkv, T, d] (last dim contiguous, same strides)."""
    B, H, T, d = k.shape
    if tuple(v.shape) != tuple(k.shape) or v.stride() != k.stride() or k.stride(3) != 1:
        raise ValueError("k and v need the same shape and strides, last dim contiguous")
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    check(lib().tq_quantize_kv(codec.handle, k.data_ptr(), v.data_ptr(), _dtype_code(k), B, H, T,
                               k.stride(0), k.stride(1), k.stride(2), _ptr(rc), _ptr(rs), pos0,
                               ctypes.byref(desc), row0, _ptr(status), _stream(stream)))


def attention_workspace(codec: Codec, B: int, Hq: int, num_splits: int) -> int:
    n = ctypes.c_size_t(0)
    check(lib().tq_attention_workspace(codec.handle, B, Hq, num_splits, ctypes.byref(n)))
    return n.value


def attention_decode(codec: Codec, q, cache: Cache, max_seq_len: int, scale: float, out,
                     workspace, seq_lens=None, rope=None, num_splits: int = 0,
                     stream=None) -> None:
    """tq_attention_decode: q [B, Hq, d] -> out [B, Hq, d] fp32."""
    B, Hq, d = q.shape
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib().tq_attention_decode(codec.handle, q.data_ptr(), _dtype_code(q), B, Hq, cache.Hkv,
                                    ctypes.byref(desc), _ptr(seq_lens), max_seq_len,
                                    float(scale), _ptr(rc), _ptr(rs), num_splits,
                                    workspace.data_ptr(), ws_bytes, out.data_ptr(),
                                    _stream(stream)))


def decode_step(codec: Codec, k_new, v_new, q, cache: Cache, T: int, scale: float, out, workspace,
                rope=None, num_splits: int = 0, stream=None) -> None:
    """tq_decode_step: append k_new, v_new [B, Hkv, d] (or [B, Hkv, 1, d]) at
    row T - 1, then decode q [B, Hq, d] over rows 0 .. T - 1 into out."""
    B, Hq = q.shape[0], q.shape[1]
    if not (k_new.is_contiguous() and v_new.is_contiguous() and k_new.dtype == v_new.dtype):
        raise ValueError("k_new and v_new must be contiguous and of one dtype")
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    check(lib().tq_decode_step(codec.handle, k_new.data_ptr(), v_new.data_ptr(), _dtype_code(k_new),
                               q.data_ptr(), _dtype_code(q), B, Hq, cache.Hkv, ctypes.byref(desc), T,
                               float(scale), _ptr(rc), _ptr(rs), num_splits, workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), out.data_ptr(),
                               _stream(stream)))


def decode_step_host(codec: Codec, in_host, in_dev, kv_dtype, q_dtype, B: int, Hq: int, Hkv: int,
                     cache: Cache, T: int, scale: float, out_dev, out_host, workspace, rope=None,
                     num_splits: int = 0, stream=None) -> None:
    """tq_decode_step_host: in_host (pinned) holds k_new, v_new [B, Hkv, d] and
    q [B, Hq, d] back to back; it is copied to in_dev, the step runs, out_dev
    is copied to out_host and the call returns with the result on the host."""
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    check(lib().tq_decode_step_host(codec.handle, in_host.data_ptr(), in_dev.data_ptr(),
                                    in_host.numel() * in_host.element_size(), _code_of(kv_dtype),
                                    _code_of(q_dtype), B, Hq, Hkv, ctypes.byref(desc), T, float(scale),
                                    _ptr(rc), _ptr(rs), num_splits, workspace.data_ptr(),
                                    workspace.numel() * workspace.element_size(), out_dev.data_ptr(),
                                    out_host.data_ptr(), _stream(stream)))


def attention_logits(codec: Codec, q, cache: Cache, max_seq_len: int, scale: float, out,
                     logits, workspace, seq_lens=None, rope=None, num_splits: int = 0,
                     stream=None) -> None:
    """tq_attention_logits: decode plus the estimated logits [B, Hq, max_seq_len]."""
    B, Hq, d = q.shape
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib().tq_attention_logits(codec.handle, q.data_ptr(), _dtype_code(q), B, Hq, cache.Hkv,
                                    ctypes.byref(desc), _ptr(seq_lens), max_seq_len,
                                    float(scale), _ptr(rc), _ptr(rs), num_splits,
                                    workspace.data_ptr(), ws_bytes, out.data_ptr(),
                                    logits.data_ptr(), _stream(stream)))


def attention_bidir_workspace(codec: Codec, B: int, H: int, Lq: int) -> int:
    n = ctypes.c_size_t(0)
    check(lib().tq_attention_bidir_workspace(codec.handle, B, H, Lq, ctypes.byref(n)))
    return n.value


def attention_bidir(codec: Codec, q, cache: Cache, T: int, scale: float, out, workspace,
                    rope=None, stream=None) -> None:
    """tq_attention_bidir: q [B, H, Lq, d] (query i at position i) -> out fp32."""
    B, H, Lq, d = q.shape
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib().tq_attention_bidir(codec.handle, q.data_ptr(), _dtype_code(q), B, H, cache.Hkv,
                                   Lq, ctypes.byref(desc), T, float(scale), _ptr(rc), _ptr(rs),
                                   workspace.data_ptr(), ws_bytes, out.data_ptr(),
                                   _stream(stream)))


def index_workspace(codec: Codec, n: int) -> int:
    b = ctypes.c_size_t(0)
    check(lib().tq_index_workspace(codec.handle, ctypes.c_int64(n), ctypes.byref(b)))
    return b.value


def index_build(codec: Codec, x, kcode, kscale, workspace, status=None, stream=None) -> None:
    """tq_index_build: x fp32 [n, 1536] -> kcode u8 [n, planes, 192], kscale fp16 [n, 2]."""
    n = x.shape[0]
    check(lib().tq_index_build(codec.handle, x.data_ptr(), ctypes.c_int64(n), kcode.data_ptr(),
                               kscale.data_ptr(), _ptr(status), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream(stream)))


def scan_workspace(codec: Codec, n: int, nq: int, k: int) -> int:
    b = ctypes.c_size_t(0)
    check(lib().tq_scan_workspace(codec.handle, ctypes.c_int64(n), nq, k, ctypes.byref(b)))
    return b.value


def scan_topk(codec: Codec, kcode, kscale, q, k: int, idx, score, workspace,
              stream=None) -> None:
    """tq_scan_topk: q fp32 [nq, 1536] against n encoded rows -> idx int32 / score fp32 [nq, k]."""
    n = kcode.shape[0]
    nq = q.shape[0]
    check(lib().tq_scan_topk(codec.handle, kcode.data_ptr(), kscale.data_ptr(), ctypes.c_int64(n),
                             q.data_ptr(), nq, k, idx.data_ptr(), score.data_ptr(),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream(stream)))


def scan_topk_lut(codec: Codec, kcode, kscale, q, k: int, idx, score, workspace,
                  stream=None) -> None:
    """tq_scan_topk_lut: the lookup-table scan (fp32 scores), same arguments as scan_topk."""
    n = kcode.shape[0]
    nq = q.shape[0]
    check(lib().tq_scan_topk_lut(codec.handle, kcode.data_ptr(), kscale.data_ptr(), ctypes.c_int64(n),
                                 q.data_ptr(), nq, k, idx.data_ptr(), score.data_ptr(),
                                 workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                 _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def attention_decode_noalloc(codec: Codec, q, cache: Cache, max_seq_len: int, scale: float, out,
                             seq_lens=None, rope=None, num_splits: int = 0, stream=None) -> None:
    """tq_attention_decode_noalloc: decode with the library's static scratch
    (for callers that cannot allocate a workspace)."""
    B, Hq, d = q.shape
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    check(lib().tq_attention_decode_noalloc(codec.handle, q.data_ptr(), _dtype_code(q), B, Hq,
                                            cache.Hkv, ctypes.byref(desc), _ptr(seq_lens),
                                            max_seq_len, float(scale), _ptr(rc), _ptr(rs),
                                            num_splits, out.data_ptr(), _stream(stream)))


def dequantize(codec: Codec, cache: Cache, which: int, row0: int, rows: int, out,
               stream=None) -> None:
    """tq_dequantize: rows [row0, row0+rows) of every (b, h) -> out [B, Hkv, rows, d]."""
    desc = cache.desc()
    check(lib().tq_dequantize(codec.handle, ctypes.byref(desc), which, row0, rows,
                              _ptr(out), _stream(stream)))


# ---------------------------------------------------------------- outlier-channel split

def split_channels(score: np.ndarray) -> np.ndarray:
    """tq_split_channels: score [..., d] (host) -> int16 channel lists [..., d]."""
    sc = np.ascontiguousarray(score, dtype=np.float32)
    d = sc.shape[-1]
    out = np.zeros(sc.shape, dtype=np.int16)
    check(lib().tq_split_channels(sc.ctypes.data, sc.size // d, d, out.ctypes.data))
    return out


@dataclass
class Split:
    """A ``tq_split``: two codecs and the device channel lists [Hkv, 2, d]
    (int16) that assign each KV head's key and value channels to them."""
    hi: Codec
    lo: Codec
    channels: "object"

    def desc(self) -> SplitDesc:
        return SplitDesc(self.hi.handle, self.lo.handle, self.channels.data_ptr())


def quantize_kv_split(split: Split, k, v, cache_hi: Cache, cache_lo: Cache, row0: int = 0,
                      rope=None, pos0: int = 0, status=None, stream=None) -> None:
    """tq_quantize_kv_split on k, v [B, Hkv, T, d]."""
    B, H, T, d = k.shape
    if tuple(v.shape) != tuple(k.shape) or v.stride() != k.stride() or k.stride(3) != 1:
        raise ValueError("k and v need the same shape and strides, last dim contiguous")
    rc, rs = (None, None) if rope is None else rope
    sd, dh, dl = split.desc(), cache_hi.desc(), cache_lo.desc()
    check(lib().tq_quantize_kv_split(ctypes.byref(sd), k.data_ptr(), v.data_ptr(), _dtype_code(k),
                                     B, H, T, k.stride(0), k.stride(1), k.stride(2), _ptr(rc),
                                     _ptr(rs), pos0, ctypes.byref(dh), ctypes.byref(dl), row0,
                                     _ptr(status), _stream(stream)))


def attention_split_workspace(split: Split, B: int, Hq: int, num_splits: int) -> int:
    n = ctypes.c_size_t(0)
    sd = split.desc()
    check(lib().tq_attention_split_workspace(ctypes.byref(sd), B, Hq, num_splits, ctypes.byref(n)))
    return n.value


def attention_decode_split(split: Split, q, cache_hi: Cache, cache_lo: Cache, max_seq_len: int,
                           scale: float, out, workspace, seq_lens=None, rope=None,
                           num_splits: int = 0, stream=None) -> None:
    """tq_attention_decode_split: q [B, Hq, d] -> out [B, Hq, d] fp32."""
    B, Hq, d = q.shape
    rc, rs = (None, None) if rope is None else rope
    sd, dh, dl = split.desc(), cache_hi.desc(), cache_lo.desc()
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib().tq_attention_decode_split(ctypes.byref(sd), q.data_ptr(), _dtype_code(q), B, Hq,
                                          cache_hi.Hkv, ctypes.byref(dh), ctypes.byref(dl),
                                          _ptr(seq_lens), max_seq_len, float(scale), _ptr(rc),
                                          _ptr(rs), num_splits, workspace.data_ptr(), ws_bytes,
                                          out.data_ptr(), _stream(stream)))


def dequantize_split(split: Split, cache_hi: Cache, cache_lo: Cache, which: int, row0: int,
                     rows: int, out, stream=None) -> None:
    """tq_dequantize_split -> out [B, Hkv, rows, d] fp32."""
    sd, dh, dl = split.desc(), cache_hi.desc(), cache_lo.desc()
    check(lib().tq_dequantize_split(ctypes.byref(sd), ctypes.byref(dh), ctypes.byref(dl), which,
                                    row0, rows, _ptr(out), _stream(stream)))


def haar_rotation(gaussian: np.ndarray) -> np.ndarray:
    """tq_haar_rotation: d x d Gaussian (host) -> Haar rotation fp32 [d, d]."""
    g = np.ascontiguousarray(gaussian, dtype=np.float32)
    out = np.zeros(g.shape, np.float32)
    check(lib().tq_haar_rotation(g.shape[0], g.ctypes.data, out.ctypes.data))
    return out


# ---------------------------------------------------------------- FibQuant k = 2

def fq_build_codebook(d: int, bits: int):
    """tq_fq_build_codebook -> (codewords fp32 [2^bits, 2], quadrature MSE per block)."""
    c = np.zeros((1 << bits, 2), np.float32)
    mse = ctypes.c_double(0.0)
    check(lib().tq_fq_build_codebook(d, bits, c.ctypes.data, ctypes.addressof(mse)))
    return c, mse.value


class FqCodec:
    """Owns a ``tq_fq_codec`` (host only: its codebooks travel as kernel
    parameters)."""

    def __init__(self, d: int, bits_k: int, bits_v: int, rotation_signs: np.ndarray):
        self.d, self.bits_k, self.bits_v = d, bits_k, bits_v
        signs = np.ascontiguousarray(rotation_signs, dtype=np.int8)
        desc = FqCodecDesc(d, bits_k, bits_v, signs.ctypes.data)
        h = ctypes.c_void_p()
        check(lib().tq_fq_codec_create(ctypes.byref(desc), ctypes.byref(h)))
        self.handle = h

    def codebooks(self):
        ck = np.zeros((1 << self.bits_k, 2), np.float32)
        cv = np.zeros((1 << self.bits_v, 2), np.float32)
        check(lib().tq_fq_codec_codebooks(self.handle, ck.ctypes.data, cv.ctypes.data))
        return ck, cv

    def close(self) -> None:
        if getattr(self, "handle", None):
            lib().tq_fq_codec_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fq_alloc_cache(codec: FqCodec, B: int, Hkv: int, rows_cap: int, device="cuda") -> Cache:
    import torch
    d = codec.d
    return Cache(
        kcode=torch.zeros((B, Hkv, rows_cap, codec.bits_k, d // 16), dtype=torch.uint8, device=device),
        kscale=torch.zeros((B, Hkv, rows_cap, 2), dtype=torch.float16, device=device),
        vcode=torch.zeros((B, Hkv, rows_cap // 32, codec.bits_v, d // 2), dtype=torch.int32, device=device),
        vnorm=torch.zeros((B, Hkv, rows_cap), dtype=torch.float16, device=device),
        B=B, Hkv=Hkv, rows_cap=rows_cap)


def fq_cache_bytes(codec: FqCodec, B: int, Hkv: int, rows_cap: int):
    out = (ctypes.c_size_t * 4)()
    check(lib().tq_fq_cache_bytes(codec.handle, B, Hkv, rows_cap, out))
    return list(out)


def fq_quantize_kv(codec: FqCodec, k, v, cache: Cache, row0: int = 0, rope=None, pos0: int = 0,
                   status=None, stream=None) -> None:
    B, H, T, d = k.shape
    if tuple(v.shape) != tuple(k.shape) or v.stride() != k.stride() or k.stride(3) != 1:
        raise ValueError("k and v need the same shape and strides, last dim contiguous")
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    check(lib().tq_fq_quantize_kv(codec.handle, k.data_ptr(), v.data_ptr(), _dtype_code(k), B, H,
                                  T, k.stride(0), k.stride(1), k.stride(2), _ptr(rc), _ptr(rs),
                                  pos0, ctypes.byref(desc), row0, _ptr(status), _stream(stream)))


def fq_attention_workspace(codec: FqCodec, B: int, Hq: int, num_splits: int) -> int:
    n = ctypes.c_size_t(0)
    check(lib().tq_fq_attention_workspace(codec.handle, B, Hq, num_splits, ctypes.byref(n)))
    return n.value


def fq_attention_decode(codec: FqCodec, q, cache: Cache, max_seq_len: int, scale: float, out,
                        workspace, seq_lens=None, rope=None, num_splits: int = 0,
                        stream=None) -> None:
    B, Hq, d = q.shape
    rc, rs = (None, None) if rope is None else rope
    desc = cache.desc()
    ws_bytes = workspace.numel() * workspace.element_size()
    check(lib().tq_fq_attention_decode(codec.handle, q.data_ptr(), _dtype_code(q), B, Hq,
                                       cache.Hkv, ctypes.byref(desc), _ptr(seq_lens), max_seq_len,
                                       float(scale), _ptr(rc), _ptr(rs), num_splits,
                                       workspace.data_ptr(), ws_bytes, out.data_ptr(),
                                       _stream(stream)))


def fq_dequantize(codec: FqCodec, cache: Cache, which: int, row0: int, rows: int, out,
                  stream=None) -> None:
    desc = cache.desc()
    check(lib().tq_fq_dequantize(codec.handle, ctypes.byref(desc), which, row0, rows, _ptr(out),
                                 _stream(stream)))


def set_timing_events(start=None, stop=None) -> None:
    """tq_set_timing_events with torch.cuda.Event objects (or None, None)."""
    check(lib().tq_set_timing_events(None if start is None else start.cuda_event,
                                     None if stop is None else stop.cuda_event))


def launch_count() -> int:
    return int(lib().tq_launch_count())
