"""Projections on the GPU (pa_qkv_rope_fwd, pa_linear_fwd) vs the fp64 projection oracle."""
import numpy as np
import pytest
import torch

import dit_resolution_packed_b200 as pa
import workloads
from oracle import proj
from tests import parity

pytestmark = pytest.mark.gpu


def _randn(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("rows,fin,fout", [(300, 256, 512), (1, 64, 32), (129, 136, 96), (257, 512, 320),
                                           (4097, 1024, 256)])
def test_linear_matches_fp64(cuda_device, rows, fin, fout):
    x, w = _randn((rows, fin), 1), _randn((fout, fin), 2, scale=fin ** -0.5)
    y = pa.linear_fwd(x.to(cuda_device), w.to(cuda_device))
    assert pa.pa_get_error() == pa.PA_OK
    parity.proj_check(y.double().cpu().numpy(), proj.linear(x, w), "y")


@pytest.mark.parametrize("heads,d,theta", [(4, 64, 10000.0), (2, 128, 10000.0), (3, 128, 0.0), (5, 64, 500.0)])
def test_qkv_rope_matches_fp64(cuda_device, heads, d, theta):
    lens = [1, 130, 257, 0, 64]
    T, C = sum(lens), 192
    x, w = _randn((T, C), 3), _randn((3 * heads * d, C), 4, scale=C ** -0.5)
    cu = workloads.cu_seqlens_from_lengths(lens)
    q, k, v = pa.qkv_rope_fwd(x.to(cuda_device), w.to(cuda_device), cu.to(cuda_device), max(lens), heads, d,
                              rope_theta=theta)
    assert pa.pa_get_error() == pa.PA_OK
    rq, rk, rv = proj.qkv_rope(x, w, cu.numpy(), heads, d, theta)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        parity.proj_check(got.double().cpu().numpy(), ref, name)


def test_qkv_rope_full_size_sampled_rows(cuda_device):
    """The mixed pack's shape (6416 tokens, hidden 3072, 24 heads of 128): sampled rows."""
    segs = [1024, 4096, 1296]
    T, C, H, d = sum(segs), 3072, 24, 128
    x, w = _randn((T, C), 5), _randn((3 * H * d, C), 6, scale=C ** -0.5)
    cu = workloads.cu_seqlens_from_lengths(segs)
    q, k, v = pa.qkv_rope_fwd(x.to(cuda_device), w.to(cuda_device), cu.to(cuda_device), max(segs), H, d)
    assert pa.pa_get_error() == pa.PA_OK
    rows = np.random.default_rng(7).choice(T, size=48, replace=False)
    rows.sort()
    pos = proj.positions(cu.numpy(), T)[rows]
    qkv = x[rows].double().numpy() @ w.double().numpy().T
    rq, rk, rv = (qkv[:, i * H * d:(i + 1) * H * d].reshape(len(rows), H, d) for i in range(3))
    rq, rk = proj.rope(rq, pos, 10000.0), proj.rope(rk, pos, 10000.0)
    idx = torch.from_numpy(rows).to(cuda_device)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        parity.proj_check(got[idx].double().cpu().numpy(), ref, name)


def test_projection_then_attention_pipeline(cuda_device):
    """x -> QKV + RoPE -> packed attention -> output projection, against the fp64 chain of oracles
    fed with the GPU's own q, k, v and attention output (each stage checked on its own inputs)."""
    import oracle
    lens = [200, 57, 300]
    T, C, H, d = sum(lens), 256, 2, 128
    x, w, wo = _randn((T, C), 8), _randn((3 * H * d, C), 9, scale=C ** -0.5), _randn((C, H * d), 10, scale=0.1)
    cu = workloads.cu_seqlens_from_lengths(lens)
    dev = cuda_device
    q, k, v = pa.qkv_rope_fwd(x.to(dev), w.to(dev), cu.to(dev), max(lens), H, d)
    out, lse = pa.varlen_attn_fwd(q, k, v, cu.to(dev), max(lens), d ** -0.5)
    y = pa.linear_fwd(out.view(T, H * d), wo.to(dev))
    assert pa.pa_get_error() == pa.PA_OK
    ref_o, _ = oracle.varlen_attention(q.cpu(), k.cpu(), v.cpu(), cu, d ** -0.5)
    parity.check(parity.errors(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o,
                               oracle.varlen_attention(q.cpu(), k.cpu(), v.cpu(), cu, d ** -0.5)[1]))
    parity.proj_check(y.double().cpu().numpy(), proj.linear(out.view(T, H * d).cpu(), wo), "y")


def test_qkv_rope_device_errors(cuda_device):
    lens = [10, 20]
    x, w = _randn((30, 64), 11), _randn((3 * 64, 64), 12)
    bad = torch.tensor([0, 25, 20], dtype=torch.int32, device=cuda_device)
    q, k, v = (torch.empty(30, 1, 64, dtype=torch.bfloat16, device=cuda_device) for _ in range(3))
    rc = pa.pa_qkv_rope_fwd(x.to(cuda_device), w.to(cuda_device), bad, 20, 10000.0, q, k, v)
    assert rc == pa.PA_OK and pa.pa_get_error() == pa.PA_ERR_CU_SEQLENS
    cu = workloads.cu_seqlens_from_lengths(lens).to(cuda_device)
    rc = pa.pa_qkv_rope_fwd(x.to(cuda_device), w.to(cuda_device), cu, 15, 10000.0, q, k, v)
    assert rc == pa.PA_OK and pa.pa_get_error() == pa.PA_ERR_MAX_SEQLEN
