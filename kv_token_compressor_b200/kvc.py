"""Thin Python binding of the C ABI in include/kvc.h (ctypes).

Argument marshalling only: tensors are checked for device, dtype and contiguity, their
device pointers and the current CUDA stream are passed to libkvc.so, and a non-OK status
raises :class:`KvcError`.  Every step of the compressor runs in the library's kernels;
there is no fallback: if libkvc.so is missing this module raises on first use.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkvc.so")

# kvc_status
KVC_OK = 0
KVC_ERR_NULL = 1
KVC_ERR_SHAPE = 2
KVC_ERR_DTYPE = 3
KVC_ERR_ALIGN = 4
KVC_ERR_UNSUPPORTED = 5
KVC_ERR_CUDA = 6
KVC_ERR_TIMEOUT = 7
KVC_ERR_POINTER = 8
KVC_ERR_INDEX = 9
KVC_ERR_WORKSPACE = 10
KVC_ERR_TOO_LARGE = 11
# kvc_dtype
KVC_F32 = 0
KVC_BF16 = 1

# Every entry point the header declares, with its ctypes signature.
_i64, _i32, _p = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
_d, _f = ctypes.c_double, ctypes.c_float
SIGNATURES = {
    "kvc_num_entries": (_i64, [_i64, _i32]),
    "kvc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "csa_compress": (ctypes.c_int, [_p, _p, _p, _p, ctypes.c_int, _p, _p, _i64, _i64, _i64, _i32,
                                    _i32, _p, ctypes.c_int, _p]),
    "hca_compress": (ctypes.c_int, [_p, _p, ctypes.c_int, _p, _i64, _i64, _i64, _i32, _p,
                                    ctypes.c_int, _p]),
    "csa_compress_fused_proj": (ctypes.c_int, [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64,
                                               _i32, _i32, _p, ctypes.c_int, _p]),
    "hca_compress_fused_proj": (ctypes.c_int, [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _i32, _p,
                                               ctypes.c_int, _p]),
    "kvc_device_status": (ctypes.c_int, [_p]),
    "kvc_set_sync_check": (None, [_i32]),
    "kvc_sync_check": (_i32, []),
    "kvc_selftest_bounded_wait": (ctypes.c_int, [_p, _p]),
    "csa_compress_scalar_logits": (ctypes.c_int, [_p, _p, _p, _p, ctypes.c_int, _p, _p, _i64, _i64,
                                                  _i64, _i32, _i32, _p, ctypes.c_int, _p]),
    "hca_compress_scalar_logits": (ctypes.c_int, [_p, _p, ctypes.c_int, _p, _i64, _i64, _i64, _i32,
                                                  _p, ctypes.c_int, _p]),
    "csa_compress_entries": (ctypes.c_int, [_p, _p, _p, _p, ctypes.c_int, _p, _p, _i64, _i64, _i32,
                                            _i32, _p, _p, _p, _i64, _p, ctypes.c_int, _p]),
    "hca_compress_entries": (ctypes.c_int, [_p, _p, ctypes.c_int, _p, _i64, _i64, _i32, _p, _p, _p,
                                            _i64, _p, ctypes.c_int, _p]),
    "csa_compress_cache": (ctypes.c_int, [_p, _p, _p, _p, ctypes.c_int, _p, _p, _i64, _i64, _i64, _i32,
                                          _i32, _i32, _p, _d, _d, _f, _p, _p, _p]),
    "hca_compress_cache": (ctypes.c_int, [_p, _p, ctypes.c_int, _p, _i64, _i64, _i64, _i32, _i32, _p,
                                          _d, _d, _f, _p, _p, _p]),
    "csa_compress_entries_cache": (ctypes.c_int, [_p, _p, _p, _p, ctypes.c_int, _p, _p, _i64, _i64,
                                                  _i32, _i32, _p, _p, _p, _i64, _i32, _p, _d, _d, _f,
                                                  _p, _p, _p]),
    "hca_compress_entries_cache": (ctypes.c_int, [_p, _p, ctypes.c_int, _p, _i64, _i64, _i32, _p, _p,
                                                  _p, _i64, _i32, _p, _d, _d, _f, _p, _p, _p]),
    "lightning_indexer_scores": (ctypes.c_int, [_p, _p, _p, _p, _p, _i64, _i32, _i32, _i64, _i64, _p,
                                                _i64, _p]),
    "indexer_topk": (ctypes.c_int, [_p, _i64, _p, _i64, _i64, _i32, _p, _p, _p]),
    "kvc_topk_max_candidates": (_i64, []),
    "kvc_last_kernel": (ctypes.c_char_p, []),
    "hca_bias_workspace_bytes": (_i64, [_i64, _i32, ctypes.c_int]),
    "hca_prepare_bias": (ctypes.c_int, [_p, _i64, _i32, ctypes.c_int, _p, _i64, _p]),
    "hca_compress_prepared": (ctypes.c_int, [_p, _p, ctypes.c_int, _p, _i64, _i64, _i64, _i64, _i32,
                                             _p, ctypes.c_int, _p]),
    "csa_compress_fused_proj_scalar": (ctypes.c_int, [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64,
                                                      _i64, _i32, _i32, _p, ctypes.c_int, _p]),
    "hca_compress_fused_proj_scalar": (ctypes.c_int, [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _i32,
                                                      _p, ctypes.c_int, _p]),
    "hca_compress_noalloc": (ctypes.c_int, [_p, _p, ctypes.c_int, _p, _i64, _i64, _i64, _i32, _p,
                                            ctypes.c_int, _p]),
    "csa_compress_fused_proj_cache": (ctypes.c_int, [_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64,
                                                     _i64, _i32, _i32, _i32, _p, _d, _d, _f, _p,
                                                     _p, _p]),
    "hca_compress_fused_proj_cache": (ctypes.c_int, [_p, _p, _p, _p, _i64, _i64, _i64, _i64, _i32,
                                                     _i32, _p, _d, _d, _f, _p, _p, _p]),
}

_lib = None


class KvcError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded libkvc.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m kv_token_compressor_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().kvc_status_string(status).decode()


def num_entries(n: int, m: int) -> int:
    return int(lib().kvc_num_entries(n, m))


def last_kernel() -> str:
    """Name of the kernel this host thread's last successful launch ran ("" before any)."""
    return lib().kvc_last_kernel().decode()


def _check(status: int, where: str):
    if status != KVC_OK:
        raise KvcError(status, where)


def _torch():
    import torch

    return torch


def _dtype_code(dt) -> int:
    torch = _torch()
    if dt == torch.float32:
        return KVC_F32
    if dt == torch.bfloat16:
        return KVC_BF16
    raise TypeError(f"unsupported dtype {dt}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _out(out, shape, dtype, like):
    torch = _torch()
    if out is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    if tuple(out.shape) != tuple(shape) or out.dtype != dtype:
        raise ValueError(f"out must be {tuple(shape)} {dtype}")
    return out


def _need(name, t, numel, dtype):
    """The library will read `numel` elements of `dtype` from `t`, and it sees only the
    pointer: refuse a tensor of another type or one too small to hold them.  None is passed
    on (the library reports a missing pointer it needs)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the call reads {numel}")


def _streams(lead, others, overlap_only, overlap):
    """The other streams of a call: the lead stream's dtype and at least its size."""
    for name, t in others:
        if overlap or name not in overlap_only:
            _need(name, t, lead.numel(), lead.dtype)


def _biases(m, width, overlap, **bs):
    """Position biases: fp32, m x width values each (Bb / bb only with overlap)."""
    torch = _torch()
    for name, t in bs.items():
        if overlap or name not in ("Bb", "bb"):
            _need(name, t, m * width, torch.float32)


def _rope_freqs(inv_freq, r, c):
    """inv_freq: fp32, r / 2 values, when r is one the library accepts (else it reports r)."""
    if 0 < r <= c and r % 8 == 0:
        _need("inv_freq", inv_freq, r // 2, _torch().float32)


def csa_compress(Ca, Cb, Za, Zb, Ba, Bb, m: int = 4, overlap: bool = True, out=None,
                 out_dtype=None, stream=None):
    """CSA compressor over precomputed streams [batch, n, c] (bf16 or fp32) with fp32
    biases [m, c].  Returns [batch, n // m, c] in ``out_dtype`` (default: input dtype)."""
    batch, n, c = Ca.shape
    _streams(Ca, (("Cb", Cb), ("Za", Za), ("Zb", Zb)), ("Cb", "Zb"), overlap)
    _biases(m, c, overlap, Ba=Ba, Bb=Bb)
    out_dtype = Ca.dtype if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, Ca)
    st = lib().csa_compress(_ptr(Ca), _ptr(Cb) if overlap else None, _ptr(Za),
                            _ptr(Zb) if overlap else None, _dtype_code(Ca.dtype), _ptr(Ba),
                            _ptr(Bb) if overlap else None, batch, n, c, m, int(bool(overlap)),
                            _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "csa_compress")
    return out


def hca_compress(C, Z, B, m: int = 128, out=None, out_dtype=None, stream=None):
    """HCA compressor over precomputed streams C, Z [batch, n, c] with bias B [m, c]."""
    batch, n, c = C.shape
    _streams(C, (("Z", Z),), (), True)
    _biases(m, c, True, B=B)
    out_dtype = C.dtype if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, C)
    st = lib().hca_compress(_ptr(C), _ptr(Z), _dtype_code(C.dtype), _ptr(B), batch, n, c, m,
                            _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "hca_compress")
    return out


def hca_bias_workspace_bytes(c: int, m: int, in_dtype) -> int:
    """Bytes of the prepared-bias workspace for c channels, window m, streams of in_dtype."""
    return int(lib().hca_bias_workspace_bytes(c, m, _dtype_code(in_dtype)))


def hca_prepare_bias(B, in_dtype, workspace=None, stream=None):
    """Prepare the HCA bias B [m, c] (fp32, device) for hca_compress_prepared with streams of
    in_dtype; returns the workspace (a uint8 device tensor)."""
    torch = _torch()
    m, c = B.shape
    _need("B", B, m * c, torch.float32)
    nbytes = hca_bias_workspace_bytes(c, m, in_dtype)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 0), dtype=torch.uint8, device=B.device)
    st = lib().hca_prepare_bias(_ptr(B), c, m, _dtype_code(in_dtype), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "hca_prepare_bias")
    return workspace


def hca_compress_prepared(C, Z, workspace, m: int = 128, out=None, out_dtype=None, stream=None):
    """hca_compress with the bias taken from a workspace of hca_prepare_bias."""
    batch, n, c = C.shape
    _streams(C, (("Z", Z),), (), True)
    out_dtype = C.dtype if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, C)
    st = lib().hca_compress_prepared(_ptr(C), _ptr(Z), _dtype_code(C.dtype), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), batch, n, c, m,
                                     _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "hca_compress_prepared")
    return out


def hca_compress_noalloc(C, Z, B, m: int = 128, out=None, out_dtype=None, stream=None):
    """hca_compress for callers that cannot allocate device memory while they run: the
    library keeps the prepared bias in a fixed 1 MiB scratch of its own (shared by all
    calls on a device; calls that overlap on the GPU race on it).  Pass `out` to avoid the
    allocation this wrapper would otherwise make for the result."""
    batch, n, c = C.shape
    _streams(C, (("Z", Z),), (), True)
    _biases(m, c, True, B=B)
    out_dtype = C.dtype if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, C)
    st = lib().hca_compress_noalloc(_ptr(C), _ptr(Z), _dtype_code(C.dtype), _ptr(B), batch, n, c, m,
                                    _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "hca_compress_noalloc")
    return out


def csa_compress_scalar_logits(Ca, Cb, za, zb, ba, bb, m: int = 4, overlap: bool = True, out=None,
                               out_dtype=None, stream=None):
    """Scalar-logit CSA: streams Ca, Cb [batch, n, c], logits za, zb [batch, n] (same dtype),
    fp32 biases ba, bb [m].  Returns [batch, n // m, c]."""
    batch, n, c = Ca.shape
    if tuple(za.shape) != (batch, n) or za.dtype != Ca.dtype:
        raise ValueError("za must be [batch, n] with the streams' dtype")
    _streams(Ca, (("Cb", Cb),), ("Cb",), overlap)
    _streams(za, (("zb", zb),), ("zb",), overlap)
    _biases(m, 1, overlap, ba=ba, bb=bb)
    out_dtype = Ca.dtype if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, Ca)
    st = lib().csa_compress_scalar_logits(
        _ptr(Ca), _ptr(Cb) if overlap else None, _ptr(za), _ptr(zb) if overlap else None,
        _dtype_code(Ca.dtype), _ptr(ba), _ptr(bb) if overlap else None, batch, n, c, m,
        int(bool(overlap)), _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "csa_compress_scalar_logits")
    return out


def hca_compress_scalar_logits(C, z, b, m: int = 128, out=None, out_dtype=None, stream=None):
    """Scalar-logit HCA: C [batch, n, c], logits z [batch, n], fp32 bias b [m]."""
    batch, n, c = C.shape
    if tuple(z.shape) != (batch, n) or z.dtype != C.dtype:
        raise ValueError("z must be [batch, n] with C's dtype")
    _biases(m, 1, True, b=b)
    out_dtype = C.dtype if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, C)
    st = lib().hca_compress_scalar_logits(_ptr(C), _ptr(z), _dtype_code(C.dtype), _ptr(b), batch, n,
                                          c, m, _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "hca_compress_scalar_logits")
    return out


def _index(t, num):
    torch = _torch()
    if t.dtype != torch.int64 or tuple(t.shape) != (num,):
        raise ValueError("index arrays must be int64 [num]")
    return _ptr(t)


def csa_compress_entries(Ca, Cb, Za, Zb, Ba, Bb, seq_start, seq_len, entry, m: int = 4,
                         overlap: bool = True, out=None, out_dtype=None, stream=None):
    """CSA entries listed by device int64 arrays (seq_start, seq_len, entry) over packed
    streams [total_rows, c].  Returns [num, c]; row k is entry entry[k] of its sequence."""
    total_rows, c = Ca.shape
    num = entry.shape[0]
    _streams(Ca, (("Cb", Cb), ("Za", Za), ("Zb", Zb)), ("Cb", "Zb"), overlap)
    _biases(m, c, overlap, Ba=Ba, Bb=Bb)
    out_dtype = Ca.dtype if out_dtype is None else out_dtype
    out = _out(out, (num, c), out_dtype, Ca)
    st = lib().csa_compress_entries(
        _ptr(Ca), _ptr(Cb) if overlap else None, _ptr(Za), _ptr(Zb) if overlap else None,
        _dtype_code(Ca.dtype), _ptr(Ba), _ptr(Bb) if overlap else None, total_rows, c, m,
        int(bool(overlap)), _index(seq_start, num), _index(seq_len, num), _index(entry, num), num,
        _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "csa_compress_entries")
    return out


def hca_compress_entries(C, Z, B, seq_start, seq_len, entry, m: int = 128, out=None,
                         out_dtype=None, stream=None):
    """HCA entries listed by device int64 arrays over packed streams [total_rows, c]."""
    total_rows, c = C.shape
    num = entry.shape[0]
    _streams(C, (("Z", Z),), (), True)
    _biases(m, c, True, B=B)
    out_dtype = C.dtype if out_dtype is None else out_dtype
    out = _out(out, (num, c), out_dtype, C)
    st = lib().hca_compress_entries(_ptr(C), _ptr(Z), _dtype_code(C.dtype), _ptr(B), total_rows, c,
                                    m, _index(seq_start, num), _index(seq_len, num),
                                    _index(entry, num), num, _ptr(out), _dtype_code(out_dtype),
                                    _stream(stream))
    _check(st, "hca_compress_entries")
    return out


def _cache_outs(rows, c, r, like, out_nope, out_rope):
    # sizes are clamped so that an invalid r reaches the library, which reports it
    torch = _torch()
    cn, rr = max(c - r, 0), max(min(r, c), 0)
    if out_nope is None:
        out_nope = torch.empty((rows, cn), dtype=torch.uint8, device=like.device)
    if out_rope is None:
        out_rope = torch.empty((rows, rr), dtype=torch.bfloat16, device=like.device)
    if out_nope.dtype not in (torch.uint8, torch.float8_e4m3fn) or out_nope.numel() != rows * cn:
        raise ValueError("out_nope must hold rows x (c - r) E4M3 bytes")
    if out_rope.dtype != torch.bfloat16 or out_rope.numel() != rows * rr:
        raise ValueError("out_rope must be rows x r bf16")
    return out_nope, out_rope


def _cache_args(r, inv_freq, pos_stride, pos_offset, fp8_scale, out_nope, out_rope, c):
    return (r, _ptr(inv_freq) if r > 0 else None, float(pos_stride), float(pos_offset),
            float(fp8_scale), _ptr(out_nope) if c - r > 0 else None, _ptr(out_rope) if r > 0 else None)


def csa_compress_cache(Ca, Cb, Za, Zb, Ba, Bb, r, inv_freq, pos_stride=4.0, pos_offset=1.5,
                       fp8_scale=1.0, m: int = 4, overlap: bool = True, out_nope=None,
                       out_rope=None, stream=None):
    """CSA entries in the cache layout: E4M3 bytes [batch, N_e, c - r] and RoPE'd bf16
    [batch, N_e, r].  The default position is the centre of the entry's own m-block."""
    batch, n, c = Ca.shape
    _streams(Ca, (("Cb", Cb), ("Za", Za), ("Zb", Zb)), ("Cb", "Zb"), overlap)
    _biases(m, c, overlap, Ba=Ba, Bb=Bb)
    _rope_freqs(inv_freq, r, c)
    ne = n // m
    nope, rope = _cache_outs(batch * ne, c, r, Ca, out_nope, out_rope)
    st = lib().csa_compress_cache(
        _ptr(Ca), _ptr(Cb) if overlap else None, _ptr(Za), _ptr(Zb) if overlap else None,
        _dtype_code(Ca.dtype), _ptr(Ba), _ptr(Bb) if overlap else None, batch, n, c, m,
        int(bool(overlap)), *_cache_args(r, inv_freq, pos_stride, pos_offset, fp8_scale, nope, rope, c),
        _stream(stream))
    _check(st, "csa_compress_cache")
    return nope.view(batch, ne, max(c - r, 0)), rope.view(batch, ne, max(min(r, c), 0))


def hca_compress_cache(C, Z, B, r, inv_freq, pos_stride=128.0, pos_offset=63.5, fp8_scale=1.0,
                       m: int = 128, out_nope=None, out_rope=None, stream=None):
    """HCA entries in the cache layout (default position: the segment centre)."""
    batch, n, c = C.shape
    _streams(C, (("Z", Z),), (), True)
    _biases(m, c, True, B=B)
    _rope_freqs(inv_freq, r, c)
    ne = n // m
    nope, rope = _cache_outs(batch * ne, c, r, C, out_nope, out_rope)
    st = lib().hca_compress_cache(_ptr(C), _ptr(Z), _dtype_code(C.dtype), _ptr(B), batch, n, c, m,
                                  *_cache_args(r, inv_freq, pos_stride, pos_offset, fp8_scale, nope,
                                               rope, c), _stream(stream))
    _check(st, "hca_compress_cache")
    return nope.view(batch, ne, max(c - r, 0)), rope.view(batch, ne, max(min(r, c), 0))


def csa_compress_entries_cache(Ca, Cb, Za, Zb, Ba, Bb, seq_start, seq_len, entry, r, inv_freq,
                               pos_stride=4.0, pos_offset=1.5, fp8_scale=1.0, m: int = 4,
                               overlap: bool = True, out_nope=None, out_rope=None, stream=None):
    """Listed CSA entries (decode-time cache insertion) in the cache layout."""
    total_rows, c = Ca.shape
    num = entry.shape[0]
    _streams(Ca, (("Cb", Cb), ("Za", Za), ("Zb", Zb)), ("Cb", "Zb"), overlap)
    _biases(m, c, overlap, Ba=Ba, Bb=Bb)
    _rope_freqs(inv_freq, r, c)
    nope, rope = _cache_outs(num, c, r, Ca, out_nope, out_rope)
    st = lib().csa_compress_entries_cache(
        _ptr(Ca), _ptr(Cb) if overlap else None, _ptr(Za), _ptr(Zb) if overlap else None,
        _dtype_code(Ca.dtype), _ptr(Ba), _ptr(Bb) if overlap else None, total_rows, c, m,
        int(bool(overlap)), _index(seq_start, num), _index(seq_len, num), _index(entry, num), num,
        *_cache_args(r, inv_freq, pos_stride, pos_offset, fp8_scale, nope, rope, c), _stream(stream))
    _check(st, "csa_compress_entries_cache")
    return nope.view(num, max(c - r, 0)), rope.view(num, max(min(r, c), 0))


def hca_compress_entries_cache(C, Z, B, seq_start, seq_len, entry, r, inv_freq, pos_stride=128.0,
                               pos_offset=63.5, fp8_scale=1.0, m: int = 128, out_nope=None,
                               out_rope=None, stream=None):
    """Listed HCA entries in the cache layout."""
    total_rows, c = C.shape
    num = entry.shape[0]
    _streams(C, (("Z", Z),), (), True)
    _biases(m, c, True, B=B)
    _rope_freqs(inv_freq, r, c)
    nope, rope = _cache_outs(num, c, r, C, out_nope, out_rope)
    st = lib().hca_compress_entries_cache(
        _ptr(C), _ptr(Z), _dtype_code(C.dtype), _ptr(B), total_rows, c, m, _index(seq_start, num),
        _index(seq_len, num), _index(entry, num), num,
        *_cache_args(r, inv_freq, pos_stride, pos_offset, fp8_scale, nope, rope, c), _stream(stream))
    _check(st, "hca_compress_entries_cache")
    return nope.view(num, max(c - r, 0)), rope.view(num, max(min(r, c), 0))


def csa_compress_fused_proj(H, W_kva, W_kvb, W_za, W_zb, Ba, Bb, batch: int, n: int, m: int = 4,
                            overlap: bool = True, out=None, out_dtype=None, stream=None):
    """CSA compressor fed by hidden states H [batch*n, d] bf16 and W's [d, c] bf16."""
    torch = _torch()
    d = H.shape[1]
    c = W_kva.shape[1]
    _need("H", H, batch * n * d, torch.bfloat16)
    for name, w in (("W_kva", W_kva), ("W_kvb", W_kvb), ("W_za", W_za), ("W_zb", W_zb)):
        if overlap or name not in ("W_kvb", "W_zb"):
            _need(name, w, d * c, torch.bfloat16)
    _biases(m, c, overlap, Ba=Ba, Bb=Bb)
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, H)
    st = lib().csa_compress_fused_proj(
        _ptr(H), _ptr(W_kva), _ptr(W_kvb) if overlap else None, _ptr(W_za),
        _ptr(W_zb) if overlap else None, _ptr(Ba), _ptr(Bb) if overlap else None,
        batch, n, d, c, m, int(bool(overlap)), _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "csa_compress_fused_proj")
    return out


def hca_compress_fused_proj(H, W_kv, W_z, B, batch: int, n: int, m: int = 128, out=None,
                            out_dtype=None, stream=None):
    """HCA compressor fed by hidden states H [batch*n, d] bf16 and W's [d, c] bf16."""
    torch = _torch()
    d = H.shape[1]
    c = W_kv.shape[1]
    _need("H", H, batch * n * d, torch.bfloat16)
    _need("W_kv", W_kv, d * c, torch.bfloat16)
    _need("W_z", W_z, d * c, torch.bfloat16)
    _biases(m, c, True, B=B)
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, H)
    st = lib().hca_compress_fused_proj(_ptr(H), _ptr(W_kv), _ptr(W_z), _ptr(B), batch, n, d, c, m,
                                       _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "hca_compress_fused_proj")
    return out


def csa_compress_fused_proj_cache(H, W_kva, W_kvb, W_za, W_zb, Ba, Bb, batch: int, n: int, r: int,
                                  inv_freq, pos_stride=4.0, pos_offset=1.5, fp8_scale=1.0,
                                  m: int = 4, out_nope=None, out_rope=None, stream=None):
    """Fused CSA (H [batch*n, d] bf16, W's [d, c] bf16) writing the cache layout: E4M3 bytes
    [batch, N_e, c - r] and RoPE'd bf16 [batch, N_e, r]."""
    torch = _torch()
    d = H.shape[1]
    c = W_kva.shape[1]
    _need("H", H, batch * n * d, torch.bfloat16)
    for name, w in (("W_kva", W_kva), ("W_kvb", W_kvb), ("W_za", W_za), ("W_zb", W_zb)):
        _need(name, w, d * c, torch.bfloat16)
    _biases(m, c, True, Ba=Ba, Bb=Bb)
    _rope_freqs(inv_freq, r, c)
    ne = n // m
    nope, rope = _cache_outs(batch * ne, c, r, H, out_nope, out_rope)
    st = lib().csa_compress_fused_proj_cache(
        _ptr(H), _ptr(W_kva), _ptr(W_kvb), _ptr(W_za), _ptr(W_zb), _ptr(Ba), _ptr(Bb), batch, n, d,
        c, m, 1, *_cache_args(r, inv_freq, pos_stride, pos_offset, fp8_scale, nope, rope, c),
        _stream(stream))
    _check(st, "csa_compress_fused_proj_cache")
    return nope.view(batch, ne, max(c - r, 0)), rope.view(batch, ne, max(min(r, c), 0))


def hca_compress_fused_proj_cache(H, W_kv, W_z, B, batch: int, n: int, r: int, inv_freq,
                                  pos_stride=128.0, pos_offset=63.5, fp8_scale=1.0, m: int = 128,
                                  out_nope=None, out_rope=None, stream=None):
    """Fused HCA writing the cache layout (default position: the segment centre)."""
    torch = _torch()
    d = H.shape[1]
    c = W_kv.shape[1]
    _need("H", H, batch * n * d, torch.bfloat16)
    _need("W_kv", W_kv, d * c, torch.bfloat16)
    _need("W_z", W_z, d * c, torch.bfloat16)
    _biases(m, c, True, B=B)
    _rope_freqs(inv_freq, r, c)
    ne = n // m
    nope, rope = _cache_outs(batch * ne, c, r, H, out_nope, out_rope)
    st = lib().hca_compress_fused_proj_cache(
        _ptr(H), _ptr(W_kv), _ptr(W_z), _ptr(B), batch, n, d, c, m,
        *_cache_args(r, inv_freq, pos_stride, pos_offset, fp8_scale, nope, rope, c),
        _stream(stream))
    _check(st, "hca_compress_fused_proj_cache")
    return nope.view(batch, ne, max(c - r, 0)), rope.view(batch, ne, max(min(r, c), 0))


def csa_compress_fused_proj_scalar(H, W_kva, W_kvb, w_za, w_zb, ba, bb, batch: int, n: int,
                                   m: int = 4, out=None, out_dtype=None, stream=None):
    """Fused scalar-logit CSA: H [batch*n, d] bf16, W_kva/W_kvb [d, c] bf16, score vectors
    w_za/w_zb [d] bf16, biases ba/bb [m] fp32.  Returns [batch, n // m, c]."""
    torch = _torch()
    d = H.shape[1]
    c = W_kva.shape[1]
    _need("H", H, batch * n * d, torch.bfloat16)
    for name, w in (("W_kva", W_kva), ("W_kvb", W_kvb)):
        _need(name, w, d * c, torch.bfloat16)
    for name, w in (("w_za", w_za), ("w_zb", w_zb)):
        _need(name, w, d, torch.bfloat16)
    _biases(m, 1, True, ba=ba, bb=bb)
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, H)
    st = lib().csa_compress_fused_proj_scalar(
        _ptr(H), _ptr(W_kva), _ptr(W_kvb), _ptr(w_za), _ptr(w_zb), _ptr(ba), _ptr(bb), batch, n,
        d, c, m, 1, _ptr(out), _dtype_code(out_dtype), _stream(stream))
    _check(st, "csa_compress_fused_proj_scalar")
    return out


def hca_compress_fused_proj_scalar(H, W_kv, w_z, b, batch: int, n: int, m: int = 128, out=None,
                                   out_dtype=None, stream=None):
    """Fused scalar-logit HCA: H [batch*n, d] bf16, W_kv [d, c] bf16, w_z [d] bf16, b [m]."""
    torch = _torch()
    d = H.shape[1]
    c = W_kv.shape[1]
    _need("H", H, batch * n * d, torch.bfloat16)
    _need("W_kv", W_kv, d * c, torch.bfloat16)
    _need("w_z", w_z, d, torch.bfloat16)
    _biases(m, 1, True, b=b)
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    out = _out(out, (batch, n // m, c), out_dtype, H)
    st = lib().hca_compress_fused_proj_scalar(_ptr(H), _ptr(W_kv), _ptr(w_z), _ptr(b), batch, n, d,
                                              c, m, _ptr(out), _dtype_code(out_dtype),
                                              _stream(stream))
    _check(st, "hca_compress_fused_proj_scalar")
    return out


def lightning_indexer_scores(q, w, K, key_start, n_visible, max_visible: int, scores=None,
                             stream=None):
    """Lightning-indexer scores: q [T, H, 128] bf16, w [T, H] fp32, K [rows, 128] bf16,
    key_start / n_visible device int64 [T]; max_visible bounds n_visible.  Returns (or
    fills) scores [T, ld] fp32 with scores[t, s] = sum_h w[t, h] relu(q[t, h] . K[key_start[t]
    + s]) for s < n_visible[t] (the rest of each row untouched)."""
    torch = _torch()
    T, H, D = q.shape
    _need("q", q, T * H * D, torch.bfloat16)
    _need("w", w, T * H, torch.float32)
    if K.dim() != 2 or K.shape[1] != D:
        raise ValueError(f"K must be [rows, {D}]")
    _need("K", K, K.shape[0] * D, torch.bfloat16)
    if scores is None:
        ld = max(4, -(-int(max_visible) // 4) * 4)
        scores = torch.zeros((T, ld), dtype=torch.float32, device=q.device)
    if scores.dim() != 2 or scores.shape[0] != T or scores.dtype != torch.float32:
        raise ValueError("scores must be fp32 [T, ld]")
    st = lib().lightning_indexer_scores(_ptr(q), _ptr(w), _ptr(K), _index(key_start, T),
                                        _index(n_visible, T), T, H, D, K.shape[0], int(max_visible),
                                        _ptr(scores), scores.shape[1], _stream(stream))
    _check(st, "lightning_indexer_scores")
    return scores


def indexer_topk(scores, n_visible, k: int, max_visible: int, out_idx=None, out_score=None,
                 want_scores: bool = True, stream=None):
    """Top-k of every score row over its first n_visible[t] entries: (idx int32 [T, k],
    scores fp32 [T, k] or None), descending, equal scores by ascending index, -1 / -inf
    past n_visible[t]."""
    torch = _torch()
    T, ld = scores.shape
    _need("scores", scores, T * ld, torch.float32)
    out_idx = _out(out_idx, (T, k), torch.int32, scores)
    if want_scores:
        out_score = _out(out_score, (T, k), torch.float32, scores)
    st = lib().indexer_topk(_ptr(scores), ld, _index(n_visible, T), T, int(max_visible), k,
                            _ptr(out_idx), _ptr(out_score) if want_scores else None,
                            _stream(stream))
    _check(st, "indexer_topk")
    return out_idx, (out_score if want_scores else None)


def topk_max_candidates() -> int:
    return int(lib().kvc_topk_max_candidates())


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the kernels' device error status."""
    return int(lib().kvc_device_status(_stream(stream)))


def set_sync_check(on: bool) -> None:
    """Turn the library's sync check on or off: with it on, every call synchronises its
    stream and raises KvcError for what the kernels reported (a bounded wait that gave up,
    a listed entry out of range, ...) instead of leaving it to device_status()."""
    lib().kvc_set_sync_check(1 if on else 0)


def sync_check() -> bool:
    return bool(lib().kvc_sync_check())


def selftest_bounded_wait(stream=None):
    """Run the bounded-wait self-test kernel (about 2 s); returns the device int32[2] flags
    (first wait gave up, second waiter left on the abort flag)."""
    torch = _torch()
    out = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    _check(lib().kvc_selftest_bounded_wait(_ptr(out), _stream(stream)), "kvc_selftest_bounded_wait")
    return out
