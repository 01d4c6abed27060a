"""B200 (sm_100a) packed variable-length attention: Python binding of ``libpackattn.so``.

The functions named ``pa_*`` mirror the C ABI in ``include/packattn.h`` one to
one and only marshal arguments (torch tensors -> device pointers, the current
CUDA stream -> ``cudaStream_t``).  Every step of the computation runs in the
library's CUDA kernels; there is no CPU or PyTorch fallback: if the library is
missing or cannot be loaded, every call raises.

``varlen_attn_fwd`` is the convenience form: it allocates ``out`` and ``lse``,
calls ``pa_varlen_attn_fwd`` and raises on a host-side error status.
"""
import ctypes
import math
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpackattn.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "packattn.h")

PA_OK = 0
PA_ERR_NULL = -1
PA_ERR_ALIGN = -2
PA_ERR_HEAD_DIM = -3
PA_ERR_SHAPE = -4
PA_ERR_CU_SEQLENS = -5
PA_ERR_MAX_SEQLEN = -6
PA_ERR_TIMEOUT = -7
PA_ERR_CUDA = -8
PA_ERR_SCALE = -9
PA_ERR_NOT_DEVICE = -10
PA_ERR_NOALLOC_LIMIT = -11
NOALLOC_MAX_BATCH = 1024

_lib = None


class PackAttnError(RuntimeError):
    def __init__(self, code, where=""):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (status {code})" if where else status_string(code))


def load_library(path=None):
    """Loads the in-tree C-ABI library (built by ``_build.py`` / ``__graft_entry__.build()``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m dit_resolution_packed_b200._build` "
                           "(there is no fallback implementation)")
    lib = ctypes.CDLL(p)
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    lib.pa_varlen_attn_fwd.restype = ctypes.c_int
    lib.pa_varlen_attn_fwd.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, ctypes.c_float, vp, vp, vp]
    lib.pa_varlen_attn_fwd_noalloc.restype = ctypes.c_int
    lib.pa_varlen_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, ctypes.c_float, vp, vp,
                                               vp, vp]
    lib.pa_varlen_attn_bwd.restype = ctypes.c_int
    lib.pa_varlen_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, ctypes.c_float,
                                       vp, vp, vp, vp]
    lib.pa_qkv_rope_fwd.restype = ctypes.c_int
    lib.pa_qkv_rope_fwd.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, ctypes.c_float, vp, vp, vp, vp]
    lib.pa_linear_fwd.restype = ctypes.c_int
    lib.pa_linear_fwd.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    lib.pa_fp8_vt_keys.restype = ctypes.c_int64
    lib.pa_fp8_vt_keys.argtypes = [i32, i32]
    lib.pa_fp8_quantize_qkv.restype = ctypes.c_int
    lib.pa_fp8_quantize_qkv.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp]
    lib.pa_fp8_quantize_qkv_delayed.restype = ctypes.c_int
    lib.pa_fp8_quantize_qkv_delayed.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.pa_varlen_attn_fwd_fp8.restype = ctypes.c_int
    lib.pa_varlen_attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, ctypes.c_float, vp, vp, vp]
    lib.pa_get_error.restype = ctypes.c_int
    lib.pa_get_error.argtypes = [vp]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_status_string.argtypes = [ctypes.c_int]
    lib.pa_version.restype = ctypes.c_int
    lib.pa_version.argtypes = []
    lib.pa_release_workspace.restype = None
    lib.pa_release_workspace.argtypes = []
    lib.pa_set_short_packing.restype = None
    lib.pa_set_short_packing.argtypes = [ctypes.c_int]
    lib.pa_schedule_stats.restype = ctypes.c_int
    lib.pa_schedule_stats.argtypes = [vp, ctypes.POINTER(ctypes.c_int64)]
    lib.pa_set_wait_limit_ms.restype = None
    lib.pa_set_wait_limit_ms.argtypes = [ctypes.c_int]
    lib.pa_selftest_wait_timeout.restype = ctypes.c_int
    lib.pa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
    lib.pa_profile_enable.restype = None
    lib.pa_profile_enable.argtypes = [ctypes.c_int]
    lib.pa_profile_read.restype = ctypes.c_int
    lib.pa_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int32)]
    if path is None:
        _lib = lib
    return lib


def header_functions(path=HEADER_PATH):
    """Names of the functions ``include/packattn.h`` declares."""
    with open(path) as f:
        text = f.read()
    return re.findall(r"PA_API\s+[\w\s\*]+?\b(pa_\w+)\s*\(", text)


def _stream_handle(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def pa_varlen_attn_fwd(q, k, v, cu_seqlens, max_seqlen, scale, out, lse, stream=None):
    """C ``pa_varlen_attn_fwd`` on torch tensors: q, k, v, out bf16 [T, H, d]; cu_seqlens int32 [B+1];
    lse fp32 [T, H].  Returns the status code (enqueued on ``stream``, default: the current stream)."""
    import torch
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16), ("v", v, torch.bfloat16),
                        ("out", out, torch.bfloat16), ("cu_seqlens", cu_seqlens, torch.int32),
                        ("lse", lse, torch.float32)):
        if t.dtype != dt:
            raise TypeError(f"{name} must be {dt}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    T, H, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or out.shape != q.shape or tuple(lse.shape) != (T, H):
        raise ValueError("shape mismatch: q, k, v, out [T, H, d]; lse [T, H]")
    B = cu_seqlens.numel() - 1
    return load_library().pa_varlen_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), B, T, H, d,
                                             int(max_seqlen), float(scale), _ptr(out), _ptr(lse),
                                             _stream_handle(stream))


def pa_varlen_attn_fwd_noalloc(q, k, v, cu_seqlens, max_seqlen, scale, out, lse, status=None, stream=None):
    """C ``pa_varlen_attn_fwd_noalloc``: the forward without any device allocation by the library.

    For callers whose device memory is owned by someone else (a framework's
    caching allocator or arena, a plug-in host, a serving loop that must not
    allocate): every buffer is the caller's -- q, k, v, out bf16 [T, H, d],
    cu_seqlens int32 [B+1], lse fp32 [T, H], and optionally ``status``, an int32
    device tensor of at least one element that receives this call's device-side
    error code.  The library's own scratch is a fixed array in its device image
    (at most ``NOALLOC_MAX_BATCH`` segments); calls that overlap on one GPU race
    on it.  Returns the host-side status code."""
    import torch
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16), ("v", v, torch.bfloat16),
                        ("out", out, torch.bfloat16), ("cu_seqlens", cu_seqlens, torch.int32),
                        ("lse", lse, torch.float32)) + ((("status", status, torch.int32),) if status is not None
                                                        else ()):
        if t.dtype != dt:
            raise TypeError(f"{name} must be {dt}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    T, H, d = q.shape
    if k.shape != q.shape or v.shape != q.shape or out.shape != q.shape or tuple(lse.shape) != (T, H):
        raise ValueError("shape mismatch: q, k, v, out [T, H, d]; lse [T, H]")
    B = cu_seqlens.numel() - 1
    return load_library().pa_varlen_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), B, T, H, d,
                                                     int(max_seqlen), float(scale), _ptr(out), _ptr(lse),
                                                     _ptr(status), _stream_handle(stream))


def varlen_attn_fwd(q, k, v, cu_seqlens, max_seqlen, scale=None, out=None, lse=None, stream=None):
    """Packed varlen bidirectional attention forward; returns (out bf16 [T, H, d], lse fp32 [T, H])."""
    import torch
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[0], q.shape[1], dtype=torch.float32, device=q.device)
    rc = pa_varlen_attn_fwd(q, k, v, cu_seqlens, max_seqlen, scale, out, lse, stream)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_varlen_attn_fwd")
    return out, lse


def pa_varlen_attn_bwd(q, k, v, out, lse, dout, cu_seqlens, max_seqlen, scale, dq, dk, dv, stream=None):
    """C ``pa_varlen_attn_bwd`` on torch tensors: q, k, v, out, dout, dq, dk, dv bf16 [T, H, d];
    lse fp32 [T, H]; cu_seqlens int32 [B+1].  Returns the status code."""
    import torch
    for name, t, dt in (("q", q, torch.bfloat16), ("k", k, torch.bfloat16), ("v", v, torch.bfloat16),
                        ("out", out, torch.bfloat16), ("dout", dout, torch.bfloat16), ("dq", dq, torch.bfloat16),
                        ("dk", dk, torch.bfloat16), ("dv", dv, torch.bfloat16), ("lse", lse, torch.float32),
                        ("cu_seqlens", cu_seqlens, torch.int32)):
        if t.dtype != dt:
            raise TypeError(f"{name} must be {dt}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    T, H, d = q.shape
    for t in (k, v, out, dout, dq, dk, dv):
        if t.shape != q.shape:
            raise ValueError("shape mismatch: q, k, v, out, dout, dq, dk, dv [T, H, d]")
    if tuple(lse.shape) != (T, H):
        raise ValueError("lse must be [T, H]")
    B = cu_seqlens.numel() - 1
    return load_library().pa_varlen_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout),
                                             _ptr(cu_seqlens), B, T, H, d, int(max_seqlen), float(scale),
                                             _ptr(dq), _ptr(dk), _ptr(dv), _stream_handle(stream))


def varlen_attn_bwd(q, k, v, out, lse, dout, cu_seqlens, max_seqlen, scale=None, stream=None):
    """Gradients of ``varlen_attn_fwd``; returns (dq, dk, dv), bf16 [T, H, d]."""
    import torch
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rc = pa_varlen_attn_bwd(q, k, v, out, lse, dout, cu_seqlens, max_seqlen, scale, dq, dk, dv, stream)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_varlen_attn_bwd")
    return dq, dk, dv


def _check_bf16(**tensors):
    import torch
    for name, t in tensors.items():
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def pa_qkv_rope_fwd(x, w_qkv, cu_seqlens, max_seqlen, rope_theta, q, k, v, stream=None):
    """C ``pa_qkv_rope_fwd``: x [T, C], w_qkv [3*H*d, C], q, k, v [T, H, d] (bf16); cu_seqlens int32 [B+1]."""
    _check_bf16(x=x, w_qkv=w_qkv, q=q, k=k, v=v)
    T, C = x.shape
    _, H, d = q.shape
    if w_qkv.shape != (3 * H * d, C) or k.shape != q.shape or v.shape != q.shape or q.shape[0] != T:
        raise ValueError("shape mismatch: x [T, C], w_qkv [3*H*d, C], q, k, v [T, H, d]")
    B = cu_seqlens.numel() - 1
    return load_library().pa_qkv_rope_fwd(_ptr(x), _ptr(w_qkv), _ptr(cu_seqlens), B, T, C, H, d, int(max_seqlen),
                                          float(rope_theta), _ptr(q), _ptr(k), _ptr(v), _stream_handle(stream))


def qkv_rope_fwd(x, w_qkv, cu_seqlens, max_seqlen, heads, head_dim, rope_theta=10000.0, stream=None):
    """Fused QKV projection + RoPE; returns q, k, v bf16 [T, H, d]."""
    import torch
    T = x.shape[0]
    q, k, v = (torch.empty(T, heads, head_dim, dtype=torch.bfloat16, device=x.device) for _ in range(3))
    rc = pa_qkv_rope_fwd(x, w_qkv, cu_seqlens, max_seqlen, rope_theta, q, k, v, stream)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_qkv_rope_fwd")
    return q, k, v


def pa_linear_fwd(x, w, y, stream=None):
    """C ``pa_linear_fwd``: y [rows, out] = x [rows, in] w[out, in]^T (bf16)."""
    _check_bf16(x=x, w=w, y=y)
    rows, fin = x.shape
    fout = w.shape[0]
    if w.shape != (fout, fin) or y.shape != (rows, fout):
        raise ValueError("shape mismatch: x [rows, in], w [out, in], y [rows, out]")
    return load_library().pa_linear_fwd(_ptr(x), _ptr(w), rows, fin, fout, _ptr(y), _stream_handle(stream))


def linear_fwd(x, w, stream=None):
    """y = x w^T (bf16) through ``pa_linear_fwd``."""
    import torch
    y = torch.empty(x.shape[0], w.shape[0], dtype=torch.bfloat16, device=x.device)
    rc = pa_linear_fwd(x, w, y, stream)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_linear_fwd")
    return y


def _check_bytes(**tensors):
    import torch
    for name, t in tensors.items():
        if t.dtype not in (torch.uint8, torch.float8_e4m3fn):
            raise TypeError(f"{name} must be uint8 or float8_e4m3fn, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def pa_fp8_vt_keys(batch, total_tokens):
    """C ``pa_fp8_vt_keys``: keys per row of the transposed FP8 V buffer."""
    return int(load_library().pa_fp8_vt_keys(int(batch), int(total_tokens)))


def pa_fp8_quantize_qkv(q, k, v, cu_seqlens, q8, k8, v8t, scales, stream=None):
    """C ``pa_fp8_quantize_qkv``: q, k, v bf16 [T, H, 128] -> q8, k8 [T, H, 128], v8t [H*128, keys]
    (bytes), scales fp32 [4 + H*128].  Returns the status code."""
    import torch
    _check_bf16(q=q, k=k, v=v)
    _check_bytes(q8=q8, k8=k8, v8t=v8t)
    if scales.dtype != torch.float32 or not scales.is_contiguous():
        raise TypeError("scales must be a contiguous float32 tensor")
    T, H, d = q.shape
    B = cu_seqlens.numel() - 1
    if (k.shape != q.shape or v.shape != q.shape or q8.shape != q.shape or k8.shape != q.shape
            or tuple(v8t.shape) != (H * d, pa_fp8_vt_keys(B, T)) or scales.numel() != 4 + H * d):
        raise ValueError("shape mismatch: q, k, v, q8, k8 [T, H, d]; v8t [H*d, keys]; scales [4 + H*d]")
    return load_library().pa_fp8_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), B, T, H, d, _ptr(q8),
                                              _ptr(k8), _ptr(v8t), _ptr(scales), _stream_handle(stream))


def fp8_quantize_qkv(q, k, v, cu_seqlens, stream=None):
    """Quantise q, k, v for the FP8 forward; returns a dict q8, k8, v8t (uint8) and scales (fp32)."""
    import torch
    T, H, d = q.shape
    B = cu_seqlens.numel() - 1
    dev = q.device
    qz = dict(q8=torch.empty(T, H, d, dtype=torch.uint8, device=dev),
              k8=torch.empty(T, H, d, dtype=torch.uint8, device=dev),
              v8t=torch.empty(H * d, max(pa_fp8_vt_keys(B, T), 0), dtype=torch.uint8, device=dev),
              scales=torch.empty(4 + H * d, dtype=torch.float32, device=dev))
    rc = pa_fp8_quantize_qkv(q, k, v, cu_seqlens, qz["q8"], qz["k8"], qz["v8t"], qz["scales"], stream)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_fp8_quantize_qkv")
    return qz


def pa_fp8_quantize_qkv_delayed(q, k, v, cu_seqlens, amax_in, amax_out, q8, k8, v8t, scales, stream=None):
    """C ``pa_fp8_quantize_qkv_delayed``: as ``pa_fp8_quantize_qkv`` with the scales from amax_in (fp32
    [4 + H*128]); this call's maxima go to amax_out (same layout).  Returns the status code."""
    import torch
    _check_bf16(q=q, k=k, v=v)
    _check_bytes(q8=q8, k8=k8, v8t=v8t)
    for name, t in (("scales", scales), ("amax_in", amax_in), ("amax_out", amax_out)):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous float32 tensor")
    T, H, d = q.shape
    B = cu_seqlens.numel() - 1
    if (k.shape != q.shape or v.shape != q.shape or q8.shape != q.shape or k8.shape != q.shape
            or tuple(v8t.shape) != (H * d, pa_fp8_vt_keys(B, T)) or scales.numel() != 4 + H * d
            or amax_in.numel() != 4 + H * d or amax_out.numel() != 4 + H * d):
        raise ValueError("shape mismatch: q, k, v, q8, k8 [T, H, d]; v8t [H*d, keys]; scales, amax [4 + H*d]")
    return load_library().pa_fp8_quantize_qkv_delayed(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), B, T, H, d, _ptr(amax_in), _ptr(amax_out), _ptr(q8), _ptr(k8),
        _ptr(v8t), _ptr(scales), _stream_handle(stream))


def fp8_quantize_qkv_delayed(q, k, v, cu_seqlens, amax_in, stream=None):
    """Delayed-scaling quantiser: scales from amax_in; returns the dict of ``fp8_quantize_qkv`` plus
    ``amax`` (this call's maxima, fp32 [4 + H*128], for the next call)."""
    import torch
    T, H, d = q.shape
    B = cu_seqlens.numel() - 1
    dev = q.device
    qz = dict(q8=torch.empty(T, H, d, dtype=torch.uint8, device=dev),
              k8=torch.empty(T, H, d, dtype=torch.uint8, device=dev),
              v8t=torch.empty(H * d, max(pa_fp8_vt_keys(B, T), 0), dtype=torch.uint8, device=dev),
              scales=torch.empty(4 + H * d, dtype=torch.float32, device=dev),
              amax=torch.empty(4 + H * d, dtype=torch.float32, device=dev))
    rc = pa_fp8_quantize_qkv_delayed(q, k, v, cu_seqlens, amax_in, qz["amax"], qz["q8"], qz["k8"], qz["v8t"],
                                     qz["scales"], stream)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_fp8_quantize_qkv_delayed")
    return qz


def pa_varlen_attn_fwd_fp8(q8, k8, v8t, scales, cu_seqlens, max_seqlen, scale, out, lse, stream=None):
    """C ``pa_varlen_attn_fwd_fp8`` on the quantiser's tensors; out bf16 [T, H, 128], lse fp32 [T, H]."""
    import torch
    _check_bytes(q8=q8, k8=k8, v8t=v8t)
    _check_bf16(out=out)
    if lse.dtype != torch.float32 or scales.dtype != torch.float32:
        raise TypeError("lse and scales must be float32")
    T, H, d = q8.shape
    B = cu_seqlens.numel() - 1
    if (k8.shape != q8.shape or out.shape != q8.shape or tuple(lse.shape) != (T, H)
            or tuple(v8t.shape) != (H * d, pa_fp8_vt_keys(B, T)) or scales.numel() != 4 + H * d):
        raise ValueError("shape mismatch: q8, k8, out [T, H, d]; v8t [H*d, keys]; lse [T, H]; scales [4 + H*d]")
    return load_library().pa_varlen_attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8t), _ptr(scales), _ptr(cu_seqlens),
                                                 B, T, H, d, int(max_seqlen), float(scale), _ptr(out), _ptr(lse),
                                                 _stream_handle(stream))


def varlen_attn_fwd_fp8(qz, cu_seqlens, max_seqlen, scale=None, out=None, lse=None, stream=None):
    """FP8 forward on a ``fp8_quantize_qkv`` result; returns (out bf16 [T, H, 128], lse fp32 [T, H])."""
    import torch
    q8 = qz["q8"]
    if scale is None:
        scale = 1.0 / math.sqrt(q8.shape[-1])
    if out is None:
        out = torch.empty(q8.shape, dtype=torch.bfloat16, device=q8.device)
    if lse is None:
        lse = torch.empty(q8.shape[0], q8.shape[1], dtype=torch.float32, device=q8.device)
    rc = pa_varlen_attn_fwd_fp8(q8, qz["k8"], qz["v8t"], qz["scales"], cu_seqlens, max_seqlen, scale, out, lse,
                                stream)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_varlen_attn_fwd_fp8")
    return out, lse


def pa_get_error(stream=None):
    return load_library().pa_get_error(_stream_handle(stream))


def pa_status_string(code):
    return load_library().pa_status_string(int(code)).decode()


status_string = pa_status_string


def pa_version():
    return load_library().pa_version()


def pa_release_workspace():
    load_library().pa_release_workspace()


def pa_set_short_packing(on):
    """C ``pa_set_short_packing``: consecutive short segments share 128-row tiles (default on)."""
    load_library().pa_set_short_packing(1 if on else 0)


def pa_schedule_stats(stream=None):
    """C ``pa_schedule_stats``: the tile ledger of the last forward call on ``stream`` as a dict
    (items, units, score_tiles, useful_pairs, groups, grouped_segments, tile_utilisation)."""
    out = (ctypes.c_int64 * 6)()
    rc = load_library().pa_schedule_stats(_stream_handle(stream), out)
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_schedule_stats")
    keys = ("items", "units", "score_tiles", "useful_pairs", "groups", "grouped_segments")
    rec = dict(zip(keys, (int(x) for x in out)))
    rec["tile_utilisation"] = rec["useful_pairs"] / (rec["score_tiles"] * 16384.0) if rec["score_tiles"] else 0.0
    return rec


def pa_set_wait_limit_ms(ms):
    load_library().pa_set_wait_limit_ms(int(ms))


def pa_selftest_wait_timeout(limit_us, stream=None):
    return load_library().pa_selftest_wait_timeout(int(limit_us), _stream_handle(stream))


def pa_profile_enable(on):
    load_library().pa_profile_enable(1 if on else 0)


def pa_profile_read():
    """(summed attention-kernel milliseconds, launches) since the last read."""
    ms, n = ctypes.c_double(0.0), ctypes.c_int32(0)
    rc = load_library().pa_profile_read(ctypes.byref(ms), ctypes.byref(n))
    if rc != PA_OK:
        raise PackAttnError(rc, "pa_profile_read")
    return ms.value, n.value
