"""fp64 CPU oracle for packed variable-length bidirectional attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline / reference legs of ``bench.py``; never by the
product package.  It shares no code with the CUDA path.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, two passes per query
row) and, for the gradients, ``attn_bwd_oracle.c`` (the chain rule through the
same definition, P recomputed in fp64).  Definitions followed:
  * "AIGC fundamentals: SparseAttn", section 3.1 (scaled dot-product scores,
    softmax rows, restricted softmax over the kept keys);
  * Mage-Flow page, "Packing + Flash Attention varlen" (cu_seqlens segments,
    non-causal, each image attends only to itself);
  * GigaPath-Flash page, section 2.2 (standard attention, scores materialised).

The forward is pinned by ``tests/test_oracle_pins.py``, the gradients by
``tests/test_oracle_bwd_pins.py``.
"""
import ctypes
import os

import numpy as np

from . import build as _build

IN_F64 = 0
IN_BF16 = 1
_ERRORS = {-1: "invalid arguments", -2: "invalid cu_seqlens", -3: "invalid sampled rows", -4: "out of memory"}
_lib = None


def bind(path):
    """Load an oracle library from ``path`` and declare its C signatures."""
    lib = ctypes.CDLL(path)
    lib.oracle_varlen_attn.restype = ctypes.c_int
    lib.oracle_varlen_attn.argtypes = [
        ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.oracle_default_threads.restype = ctypes.c_int
    if hasattr(lib, "oracle_varlen_attn_bwd"):
        vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_varlen_attn_bwd.restype = ctypes.c_int
        lib.oracle_varlen_attn_bwd.argtypes = [ctypes.c_int, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, f64,
                                               vp, vp, vp, ctypes.c_int]
        lib.oracle_varlen_attn_bwd_dq_rows.restype = ctypes.c_int
        lib.oracle_varlen_attn_bwd_dq_rows.argtypes = [ctypes.c_int, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32,
                                                       f64, i64, vp, vp, vp, ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(_build.build())
    return _lib


def default_threads():
    return int(_load().oracle_default_threads())


def _as_input(x):
    """numpy fp64 array, or a torch bf16 tensor / numpy uint16 array of bf16 bits."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        return IN_BF16, np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))
    if hasattr(x, "numpy") and not isinstance(x, np.ndarray):
        x = x.numpy()
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return IN_BF16, np.ascontiguousarray(x)
    return IN_F64, np.ascontiguousarray(x, dtype=np.float64)


def varlen_attention(q, k, v, cu_seqlens, scale, rows=None, n_threads=0, lib=None):
    """Block-diagonal attention in fp64.

    q, k: [T, H, d]; v: [T, H, dv] (all fp64, or all bf16).  ``cu_seqlens``: [B+1].
    rows: None for every row (returns out [T, H, dv], lse [T, H]) or a pair
    (token int64 [n], head int32 [n]) (returns out [n, dv], lse [n]).
    lse is the natural-log log-sum-exp of the scaled scores of the row.
    """
    kq, qa = _as_input(q)
    kk, ka = _as_input(k)
    kv, va = _as_input(v)
    if not (kq == kk == kv):
        raise TypeError("q, k, v must share one input kind")
    if qa.ndim != 3 or ka.shape != qa.shape or va.ndim != 3 or va.shape[:2] != qa.shape[:2]:
        raise ValueError("expected q, k [T, H, d] and v [T, H, dv]")
    T, H, d = qa.shape
    dv = va.shape[2]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64).astype(np.int32))
    B = cu.shape[0] - 1
    if B < 0:
        raise ValueError("cu_seqlens must have at least one entry")
    if rows is None:
        out = np.empty((T, H, dv), dtype=np.float64)
        lse = np.empty((T, H), dtype=np.float64)
        n, rt, rh = 0, None, None
    else:
        rt = np.ascontiguousarray(np.asarray(rows[0], dtype=np.int64))
        rh = np.ascontiguousarray(np.asarray(rows[1], dtype=np.int32))
        n = rt.shape[0]
        out = np.empty((n, dv), dtype=np.float64)
        lse = np.empty((n,), dtype=np.float64)
    ptr = lambda a: None if a is None else a.ctypes.data
    rc = (lib or _load()).oracle_varlen_attn(kq, ptr(qa), ptr(ka), ptr(va), ptr(cu), B, T, H, d, dv,
                                    float(scale), n, ptr(rt), ptr(rh), ptr(out), ptr(lse), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle: {_ERRORS.get(rc, rc)}")
    return out, lse


def varlen_attention_bwd(q, k, v, dout, cu_seqlens, scale, rows=None, n_threads=0, lib=None):
    """Gradients of block-diagonal attention in fp64 (dout = dL/dout).

    q, k: [T, H, d]; v, dout: [T, H, dv] (all fp64, or all bf16).  rows: None for
    every row (returns dq [T, H, d], dk [T, H, d], dv [T, H, dv]) or a pair
    (token int64 [n], head int32 [n]) (returns dq [n, d] of those rows only).
    """
    kinds_arrays = [_as_input(x) for x in (q, k, v, dout)]
    if len({kd for kd, _ in kinds_arrays}) != 1:
        raise TypeError("q, k, v, dout must share one input kind")
    kind = kinds_arrays[0][0]
    qa, ka, va, ga = (a for _, a in kinds_arrays)
    if qa.ndim != 3 or ka.shape != qa.shape or va.ndim != 3 or va.shape[:2] != qa.shape[:2] or ga.shape != va.shape:
        raise ValueError("expected q, k [T, H, d] and v, dout [T, H, dv]")
    T, H, d = qa.shape
    dv = va.shape[2]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64).astype(np.int32))
    B = cu.shape[0] - 1
    if B < 0:
        raise ValueError("cu_seqlens must have at least one entry")
    L = lib or _load()
    ptr = lambda a: None if a is None else a.ctypes.data
    if rows is None:
        dq = np.zeros((T, H, d)); dk = np.zeros((T, H, d)); dvo = np.zeros((T, H, dv))
        rc = L.oracle_varlen_attn_bwd(kind, ptr(qa), ptr(ka), ptr(va), ptr(ga), ptr(cu), B, T, H, d, dv,
                                      float(scale), ptr(dq), ptr(dk), ptr(dvo), int(n_threads))
        if rc != 0:
            raise ValueError(f"oracle: {_ERRORS.get(rc, rc)}")
        return dq, dk, dvo
    rt = np.ascontiguousarray(np.asarray(rows[0], dtype=np.int64))
    rh = np.ascontiguousarray(np.asarray(rows[1], dtype=np.int32))
    dq = np.zeros((rt.shape[0], d))
    rc = L.oracle_varlen_attn_bwd_dq_rows(kind, ptr(qa), ptr(ka), ptr(va), ptr(ga), ptr(cu), B, T, H, d, dv,
                                          float(scale), rt.shape[0], ptr(rt), ptr(rh), ptr(dq), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle: {_ERRORS.get(rc, rc)}")
    return dq
