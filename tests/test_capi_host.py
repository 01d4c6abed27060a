"""The C-ABI library on a machine without a GPU: it builds, loads, exports every
declared symbol, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import math
import subprocess

import pytest

import dit_resolution_packed_b200 as pa
from dit_resolution_packed_b200 import _build


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return pa.load_library()


def test_header_declares_the_abi():
    names = pa.header_functions()
    assert "pa_varlen_attn_fwd" in names and "pa_get_error" in names
    assert len(names) == len(set(names)) == 19


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True, text=True, check=True)
    exported = {line.split()[-1] for line in out.stdout.splitlines() if " T " in line}
    missing = set(pa.header_functions()) - exported
    assert not missing, missing
    # nothing of the statically linked CUDA runtime leaks out of the library
    assert not any(n.startswith("cuda") for n in exported)
    for name in pa.header_functions():
        assert hasattr(lib, name)


def test_version_and_status_strings(lib):
    assert pa.pa_version() == 100
    codes = [0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -10, -11]
    texts = [pa.status_string(c) for c in codes]
    assert len(set(texts)) == len(codes) and "unknown" not in " ".join(texts)
    assert pa.status_string(-99) == "unknown status"


def _raw(lib, q=16, k=16, v=16, cu=16, batch=1, total=4, heads=1, head_dim=64, max_seqlen=4, scale=0.125,
         out=16, lse=16):
    return lib.pa_varlen_attn_fwd(q, k, v, cu, batch, total, heads, head_dim, max_seqlen, ctypes.c_float(scale),
                                  out, lse, None)


def test_host_validation_before_any_cuda_call(lib):
    assert _raw(lib, head_dim=96) == pa.PA_ERR_HEAD_DIM
    assert _raw(lib, head_dim=256) == pa.PA_ERR_HEAD_DIM
    assert _raw(lib, heads=0) == pa.PA_ERR_SHAPE
    assert _raw(lib, batch=-1) == pa.PA_ERR_SHAPE
    assert _raw(lib, total=-5) == pa.PA_ERR_SHAPE
    assert _raw(lib, batch=0, total=3) == pa.PA_ERR_SHAPE
    assert _raw(lib, scale=math.nan) == pa.PA_ERR_SCALE
    assert _raw(lib, scale=math.inf) == pa.PA_ERR_SCALE
    assert _raw(lib, batch=0, total=0) == pa.PA_OK
    assert _raw(lib, batch=3, total=0) == pa.PA_OK
    assert _raw(lib, max_seqlen=0) == pa.PA_ERR_MAX_SEQLEN
    assert _raw(lib, q=None) == pa.PA_ERR_NULL
    assert _raw(lib, lse=None) == pa.PA_ERR_NULL
    assert _raw(lib, k=24) == pa.PA_ERR_ALIGN
    assert _raw(lib, out=8) == pa.PA_ERR_ALIGN
    assert _raw(lib, lse=18) == pa.PA_ERR_ALIGN
    assert _raw(lib, heads=1 << 20, head_dim=64, total=1 << 30) == pa.PA_ERR_SHAPE


def test_noalloc_rejects_batch_above_its_limit_before_any_cuda_call(lib):
    f = lib.pa_varlen_attn_fwd_noalloc
    args = lambda batch, head_dim=64: (16, 16, 16, 16, batch, 4096, 1, head_dim, 4, ctypes.c_float(0.125), 16, 16,
                                       None, None)
    assert f(*args(pa.NOALLOC_MAX_BATCH + 1)) == pa.PA_ERR_NOALLOC_LIMIT
    assert f(*args(1 << 30)) == pa.PA_ERR_NOALLOC_LIMIT
    assert f(*args(pa.NOALLOC_MAX_BATCH, head_dim=96)) == pa.PA_ERR_HEAD_DIM
    assert f(16, 16, 16, 16, 3, 0, 1, 64, 4, ctypes.c_float(0.125), 16, 16, None, None) == pa.PA_OK


def test_bwd_host_validation_before_any_cuda_call(lib):
    def raw(q=16, out=16, lse=16, dout=16, batch=1, total=4, heads=1, head_dim=64, max_seqlen=4, scale=0.125,
            dq=16):
        return lib.pa_varlen_attn_bwd(q, 16, 16, out, lse, dout, 16, batch, total, heads, head_dim, max_seqlen,
                                      ctypes.c_float(scale), dq, 16, 16, None)
    assert raw(head_dim=80) == pa.PA_ERR_HEAD_DIM
    assert raw(heads=0) == pa.PA_ERR_SHAPE
    assert raw(batch=0, total=3) == pa.PA_ERR_SHAPE
    assert raw(batch=0, total=0) == pa.PA_OK
    assert raw(scale=math.inf) == pa.PA_ERR_SCALE
    assert raw(max_seqlen=0) == pa.PA_ERR_MAX_SEQLEN
    assert raw(dout=None) == pa.PA_ERR_NULL
    assert raw(lse=None) == pa.PA_ERR_NULL
    assert raw(dq=24) == pa.PA_ERR_ALIGN
    assert raw(out=8) == pa.PA_ERR_ALIGN
    assert raw(lse=18) == pa.PA_ERR_ALIGN


def test_projection_host_validation_before_any_cuda_call(lib):
    f = lib.pa_linear_fwd
    assert f(16, 16, 4, 12, 64, 16, None) == pa.PA_ERR_SHAPE       # in_features not a multiple of 8
    assert f(16, 16, 4, 16, 48, 16, None) == pa.PA_ERR_SHAPE       # out_features not a multiple of 32
    assert f(16, 16, 0, 16, 64, 16, None) == pa.PA_OK
    assert f(None, 16, 4, 16, 64, 16, None) == pa.PA_ERR_NULL
    assert f(16, 24, 4, 16, 64, 16, None) == pa.PA_ERR_ALIGN
    g = lib.pa_qkv_rope_fwd
    args = lambda **kw: (kw.get("x", 16), 16, kw.get("cu", 16), kw.get("batch", 1), kw.get("total", 4),
                         kw.get("hidden", 64), 1, kw.get("d", 64), kw.get("max_seqlen", 4),
                         ctypes.c_float(kw.get("theta", 10000.0)), 16, 16, 16, None)
    assert g(*args(d=96)) == pa.PA_ERR_HEAD_DIM
    assert g(*args(hidden=60)) == pa.PA_ERR_SHAPE
    assert g(*args(theta=math.nan)) == pa.PA_ERR_SCALE
    assert g(*args(max_seqlen=0)) == pa.PA_ERR_MAX_SEQLEN
    assert g(*args(cu=None)) == pa.PA_ERR_NULL
    assert g(*args(batch=0, total=0)) == pa.PA_OK


def test_fp8_host_validation_before_any_cuda_call(lib):
    # keys per transposed-V row: 16*ceil(T/16) + 16*B
    assert pa.pa_fp8_vt_keys(3, 100) == 112 + 48
    assert pa.pa_fp8_vt_keys(1, 16) == 32 and pa.pa_fp8_vt_keys(0, 0) == 0
    assert pa.pa_fp8_vt_keys(-1, 4) == -1
    q = lib.pa_fp8_quantize_qkv
    qargs = lambda **kw: (kw.get("q", 16), 16, 16, kw.get("cu", 16), kw.get("batch", 1), kw.get("total", 4),
                          kw.get("heads", 1), kw.get("d", 128), 16, 16, kw.get("v8t", 16), kw.get("scales", 16), None)
    assert q(*qargs(d=64)) == pa.PA_ERR_HEAD_DIM
    assert q(*qargs(batch=0, total=3)) == pa.PA_ERR_SHAPE
    assert q(*qargs(batch=0, total=0)) == pa.PA_OK
    assert q(*qargs(q=None)) == pa.PA_ERR_NULL
    assert q(*qargs(v8t=24)) == pa.PA_ERR_ALIGN
    assert q(*qargs(scales=8)) == pa.PA_ERR_ALIGN
    assert q(*qargs(heads=65536)) == pa.PA_ERR_SHAPE
    qd = lib.pa_fp8_quantize_qkv_delayed
    dargs = lambda **kw: (16, 16, 16, 16, kw.get("batch", 1), kw.get("total", 4), 1, kw.get("d", 128),
                          kw.get("ain", 4096), kw.get("aout", 8192), 16, 16, 16, 16, None)
    assert qd(*dargs(d=64)) == pa.PA_ERR_HEAD_DIM
    assert qd(*dargs(ain=None)) == pa.PA_ERR_NULL
    assert qd(*dargs(aout=None)) == pa.PA_ERR_NULL
    assert qd(*dargs(ain=4098)) == pa.PA_ERR_ALIGN
    assert qd(*dargs(aout=4096 + 8)) == pa.PA_ERR_SHAPE  # overlaps amax_in (4 * (4 + 128) bytes)
    assert qd(*dargs(batch=0, total=3)) == pa.PA_ERR_SHAPE
    f = lib.pa_varlen_attn_fwd_fp8
    fargs = lambda **kw: (16, 16, kw.get("v8t", 16), kw.get("scales", 16), 16, kw.get("batch", 1), kw.get("total", 4),
                          1, kw.get("d", 128), kw.get("max_seqlen", 4), ctypes.c_float(kw.get("scale", 0.1)),
                          kw.get("out", 16), 16, None)
    assert f(*fargs(d=64)) == pa.PA_ERR_HEAD_DIM
    assert f(*fargs(scale=math.nan)) == pa.PA_ERR_SCALE
    assert f(*fargs(max_seqlen=0)) == pa.PA_ERR_MAX_SEQLEN
    assert f(*fargs(scales=None)) == pa.PA_ERR_NULL
    assert f(*fargs(scales=20)) == pa.PA_ERR_ALIGN
    assert f(*fargs(out=8)) == pa.PA_ERR_ALIGN
    assert f(*fargs(batch=3, total=0)) == pa.PA_OK


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        pa.load_library(str(tmp_path / "libpackattn.so"))


def test_schedule_stats_without_a_call(lib):
    """The ledger query refuses a NULL output and a (device, stream) pair that has no call yet,
    without touching a GPU."""
    out = (ctypes.c_int64 * 6)()
    assert lib.pa_schedule_stats(None, None) == pa.PA_ERR_NULL
    rc = lib.pa_schedule_stats(None, out)
    assert rc in (pa.PA_ERR_NOT_DEVICE, pa.PA_ERR_CUDA)
    pa.pa_set_short_packing(False)
    pa.pa_set_short_packing(True)
