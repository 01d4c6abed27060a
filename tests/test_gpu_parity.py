"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200)."""
import math

import numpy as np
import pytest
import torch

import dit_resolution_packed_b200 as pa
import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


def _to_dev(p, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in p.items()}


def _run(p, dev, scale=None):
    g = _to_dev(p, dev)
    out, lse = pa.varlen_attn_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], g["max_seqlen"],
                                  p["scale"] if scale is None else scale)
    rc = pa.pa_get_error()
    assert rc == pa.PA_OK, pa.status_string(rc)
    return out, lse


def _full_check(p, dev, scale=None):
    sc = p["scale"] if scale is None else scale
    out, lse = _run(p, dev, sc)
    ref_o, ref_l = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], sc)
    errs = parity.errors(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l)
    parity.check(errs)
    return errs


def test_tiny_config_all_rows(cuda_device):
    p = workloads.make_inputs(workloads.load_config("tiny"))
    _full_check(p, cuda_device)


@pytest.mark.parametrize("d", [64, 128])
def test_ragged_edge_lengths_all_rows(cuda_device, d):
    lens = [1, 2, 127, 128, 129, 255, 256, 257, 383, 384, 385, 511, 513, 1000]
    p = workloads.random_pack(lens, heads=3, head_dim=d, seed=11)
    _full_check(p, cuda_device)


def test_many_short_segments_all_rows(cuda_device):
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 301, size=300).tolist()
    p = workloads.random_pack(lens, heads=2, head_dim=64, seed=12)
    _full_check(p, cuda_device)


def test_batch_beyond_the_staged_schedule_path(cuda_device):
    """5000 segments: more cu_seqlens entries than the scheduler stages in shared memory
    (4097), so it reads them from global memory; short segments, all rows checked."""
    rng = np.random.default_rng(8)
    lens = rng.integers(0, 41, size=5000).tolist()
    p = workloads.random_pack(lens, heads=2, head_dim=64, seed=22)
    _full_check(p, cuda_device)


def test_zero_length_segments(cuda_device):
    p = workloads.random_pack([0, 5, 0, 130, 0, 0, 257, 0], heads=2, head_dim=128, seed=13)
    _full_check(p, cuda_device)


@pytest.mark.parametrize("scale", [-0.1, 0.0, 0.5])
def test_other_scales(cuda_device, scale):
    p = workloads.random_pack([77, 300, 129], heads=2, head_dim=64, seed=14)
    _full_check(p, cuda_device, scale=scale)


def test_single_segment_longer_than_l2_tile(cuda_device):
    p = workloads.random_pack([3000], heads=2, head_dim=128, seed=15)
    _full_check(p, cuda_device)


def _report(name, errs):
    """One line per full-size check (pytest -s shows it): the worst errors against the bounds."""
    print(f"\nparity {name}: bound_ratio {errs['bound_ratio']:.4f} max_abs {errs['max_abs']:.3e} "
          f"rel_fro {errs['rel_fro']:.3e} lse_abs {errs['lse_abs']:.3e}")


@pytest.mark.parametrize("name", ["mixed", "training", "interactive"])
def test_full_size_config_all_rows(cuda_device, name):
    """Full-size workloads in the benchmark's launch configuration, every (token, head) row
    compared with the fp64 oracle (the interactive pack includes its outlier keys)."""
    p = workloads.make_inputs(workloads.load_config(name))
    errs = _full_check(p, cuda_device)
    _report(name, errs)


def test_full_size_long_sampled_rows(cuda_device):
    """The 65 536-token single segment: 512 seeded query rows per head against the full fp64
    softmax over all keys; every row of the output is finite."""
    cfg = workloads.load_config("long")
    p = workloads.make_inputs(cfg)
    out, lse = _run(p, cuda_device)
    tok, head = workloads.sampled_rows(cfg, per_head=512)
    ref_o, ref_l = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"], rows=(tok, head))
    go, gl = parity.gather_rows(out, lse, tok, head)
    errs = parity.errors(go, gl, ref_o, ref_l)
    parity.check(errs)
    _report("long (512 rows per head)", errs)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_deterministic(cuda_device):
    p = workloads.make_inputs(workloads.load_config("mixed"))
    o1, l1 = _run(p, cuda_device)
    o2, l2 = _run(p, cuda_device)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_no_writes_outside_outputs(cuda_device):
    """Guard bands around out and lse stay untouched (stands in for a memory checker)."""
    p = workloads.random_pack([129, 1, 255, 64], heads=3, head_dim=128, seed=16)
    g = _to_dev(p, cuda_device)
    T, H, d = g["q"].shape
    pad = 4096
    out_buf = torch.full((pad * 2 + T * H * d,), 7.0, dtype=torch.bfloat16, device=cuda_device)
    lse_buf = torch.full((pad * 2 + T * H,), 7.0, dtype=torch.float32, device=cuda_device)
    out = out_buf[pad:pad + T * H * d].view(T, H, d)
    lse = lse_buf[pad:pad + T * H].view(T, H)
    rc = pa.pa_varlen_attn_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], g["max_seqlen"], p["scale"], out, lse)
    assert rc == pa.PA_OK and pa.pa_get_error() == pa.PA_OK
    assert torch.all(out_buf[:pad] == 7.0) and torch.all(out_buf[-pad:] == 7.0)
    assert torch.all(lse_buf[:pad] == 7.0) and torch.all(lse_buf[-pad:] == 7.0)
    ref_o, ref_l = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"])
    parity.check(parity.errors(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l))


def test_non_default_stream(cuda_device):
    p = workloads.random_pack([200, 333], heads=2, head_dim=64, seed=17)
    s = torch.cuda.Stream()
    g = _to_dev(p, cuda_device)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        out, lse = pa.varlen_attn_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], g["max_seqlen"], p["scale"])
        assert pa.pa_get_error(s) == pa.PA_OK
    ref_o, ref_l = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"])
    parity.check(parity.errors(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l))


def _call_raw(g, cu, max_seqlen, scale=0.125):
    T, H, d = g["q"].shape
    out = torch.empty_like(g["q"])
    lse = torch.empty(T, H, dtype=torch.float32, device=g["q"].device)
    return pa.pa_varlen_attn_fwd(g["q"], g["k"], g["v"], cu, max_seqlen, scale, out, lse)


def test_device_rejects_bad_cu_seqlens_then_recovers(cuda_device):
    p = workloads.random_pack([100, 50], heads=2, head_dim=64, seed=18)
    g = _to_dev(p, cuda_device)
    for bad in ([0, 120, 100], [3, 100, 150], [0, 100, 149]):
        cu = torch.tensor(bad, dtype=torch.int32, device=cuda_device)
        assert _call_raw(g, cu, 200) == pa.PA_OK  # enqueued; the device finds the problem
        assert pa.pa_get_error() == pa.PA_ERR_CU_SEQLENS
    _full_check(p, cuda_device)


def test_device_rejects_segment_longer_than_max_seqlen(cuda_device):
    p = workloads.random_pack([100, 50], heads=2, head_dim=64, seed=19)
    g = _to_dev(p, cuda_device)
    assert _call_raw(g, g["cu_seqlens"], 99) == pa.PA_OK
    assert pa.pa_get_error() == pa.PA_ERR_MAX_SEQLEN
    _full_check(p, cuda_device)


def test_bounded_wait_records_timeout_and_context_survives(cuda_device):
    assert pa.pa_selftest_wait_timeout(2000) == pa.PA_OK
    assert pa.pa_get_error() == pa.PA_ERR_TIMEOUT
    assert pa.pa_get_error() == pa.PA_OK
    _full_check(workloads.random_pack([300], heads=1, head_dim=128, seed=20), cuda_device)


def test_host_side_errors(cuda_device):
    p = workloads.random_pack([10], heads=1, head_dim=64, seed=21)
    g = _to_dev(p, cuda_device)
    cu = g["cu_seqlens"]
    assert _call_raw(g, cu, 10, scale=math.inf) == pa.PA_ERR_SCALE
    assert _call_raw(g, cu, 0) == pa.PA_ERR_MAX_SEQLEN
    host = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in g.items()}
    assert _call_raw(host, host["cu_seqlens"], 10) == pa.PA_ERR_NOT_DEVICE
    q96 = torch.zeros(10, 1, 96, dtype=torch.bfloat16, device=cuda_device)
    out = torch.empty_like(q96)
    lse = torch.empty(10, 1, dtype=torch.float32, device=cuda_device)
    assert pa.pa_varlen_attn_fwd(q96, q96, q96, cu, 10, 0.1, out, lse) == pa.PA_ERR_HEAD_DIM
    empty = torch.zeros(0, 2, 64, dtype=torch.bfloat16, device=cuda_device)
    e_out = torch.empty_like(empty)
    e_lse = torch.empty(0, 2, dtype=torch.float32, device=cuda_device)
    cu0 = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    assert pa.pa_varlen_attn_fwd(empty, empty, empty, cu0, 0, 0.1, e_out, e_lse) == pa.PA_OK
