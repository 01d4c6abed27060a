"""Gradients on the GPU (pa_varlen_attn_bwd) vs the fp64 gradient oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import dit_resolution_packed_b200 as pa
import oracle
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


def _forward_backward(p, dev, dout_seed, scale=None):
    sc = p["scale"] if scale is None else scale
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in p.items()}
    out, lse = pa.varlen_attn_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], g["max_seqlen"], sc)
    dout_cpu = workloads.random_dout(p["q"].shape, dout_seed)
    dq, dk, dv = pa.varlen_attn_bwd(g["q"], g["k"], g["v"], out, lse, dout_cpu.to(dev), g["cu_seqlens"],
                                    g["max_seqlen"], sc)
    rc = pa.pa_get_error()
    assert rc == pa.PA_OK, pa.status_string(rc)
    return dq, dk, dv, dout_cpu, sc


def _full_check(p, dev, dout_seed=100, scale=None):
    dq, dk, dv, dout, sc = _forward_backward(p, dev, dout_seed, scale)
    ref = oracle.varlen_attention_bwd(p["q"], p["k"], p["v"], dout, p["cu_seqlens"], sc)
    errs = {}
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        errs[name] = parity.bwd_errors(got.double().cpu().numpy(), r)
        parity.bwd_check(errs[name], name)
    return errs


def test_bwd_tiny_config(cuda_device):
    _full_check(workloads.make_inputs(workloads.load_config("tiny")), cuda_device)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_ragged_edge_lengths(cuda_device, d):
    lens = [1, 2, 127, 128, 129, 255, 256, 257, 511, 513, 1000]
    _full_check(workloads.random_pack(lens, heads=2, head_dim=d, seed=41), cuda_device)


def test_bwd_zero_length_segments(cuda_device):
    _full_check(workloads.random_pack([0, 5, 0, 130, 0, 0, 257, 0], heads=2, head_dim=128, seed=42), cuda_device)


def test_bwd_many_short_segments(cuda_device):
    lens = np.random.default_rng(43).integers(1, 301, size=300).tolist()
    _full_check(workloads.random_pack(lens, heads=2, head_dim=64, seed=44), cuda_device)


@pytest.mark.parametrize("scale", [-0.1, 0.0, 0.3])
def test_bwd_other_scales(cuda_device, scale):
    _full_check(workloads.random_pack([200, 333, 64], heads=2, head_dim=128, seed=45), cuda_device, scale=scale)


def test_bwd_medium_pack_many_heads(cuda_device):
    _full_check(workloads.random_pack([1024, 300, 700], heads=3, head_dim=128, seed=46), cuda_device)


def test_bwd_mixed_config_all_elements(cuda_device):
    """Full-size mixed pack (24 heads, d = 128): every element of dq, dk and dv against the fp64
    gradient oracle."""
    errs = _full_check(workloads.make_inputs(workloads.load_config("mixed")), cuda_device, dout_seed=47)
    for name, e in errs.items():
        print(f"\nbwd parity mixed {name}: max_abs {e['max_abs']:.3e} (of max|ref| {e['ref_max']:.3e}) "
              f"rel_fro {e['rel_fro']:.3e}")


def test_bwd_dk_dv_deterministic(cuda_device):
    p = workloads.random_pack([300, 129, 700], heads=2, head_dim=128, seed=48)
    a = _forward_backward(p, cuda_device, 49)
    b = _forward_backward(p, cuda_device, 49)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 1e-2 * a[0].float().abs().max().item()


def test_bwd_device_rejects_bad_cu_seqlens(cuda_device):
    p = workloads.random_pack([100, 50], heads=2, head_dim=64, seed=50)
    g = {k: (v.to(cuda_device) if torch.is_tensor(v) else v) for k, v in p.items()}
    out, lse = pa.varlen_attn_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], g["max_seqlen"], p["scale"])
    assert pa.pa_get_error() == pa.PA_OK
    bad = torch.tensor([0, 120, 100], dtype=torch.int32, device=cuda_device)
    dq, dk, dv = (torch.empty_like(g["q"]) for _ in range(3))
    rc = pa.pa_varlen_attn_bwd(g["q"], g["k"], g["v"], out, lse, torch.ones_like(g["q"]), bad, 200, p["scale"],
                               dq, dk, dv)
    assert rc == pa.PA_OK
    assert pa.pa_get_error() == pa.PA_ERR_CU_SEQLENS
    _full_check(p, cuda_device)


@pytest.mark.parametrize("name,per_head", [("long", 6), ("interactive", 3)])
def test_bwd_full_size_sampled_dq_rows_and_closed_forms(cuda_device, name, per_head):
    """Full-size packs (65 536 tokens at d = 64; 16 384 tokens with outlier keys at d = 128):
    dq of sampled query rows against the oracle, and per head the closed forms of the exact
    gradient, sum_j dv_j = sum_r dout_r and sum_j dk_j = 0, within the accumulated bf16 rounding."""
    cfg = workloads.load_config(name)
    p = workloads.make_inputs(cfg)
    dq, dk, dv, dout, sc = _forward_backward(p, cuda_device, 51)
    tok, head = workloads.sampled_rows(cfg, per_head=per_head)
    ref = oracle.varlen_attention_bwd(p["q"], p["k"], p["v"], dout, p["cu_seqlens"], sc,
                                      rows=(tok.numpy(), head.numpy()))
    got = dq[tok.to(cuda_device), head.to(cuda_device).long()].double().cpu().numpy()
    parity.bwd_check(parity.bwd_errors(got, ref), "dq")
    g = dout.to(cuda_device).double()
    for h in range(cfg["heads"]):  # one segment per pack
        sv = dv[:, h].double().sum(0) - g[:, h].sum(0)
        assert sv.abs().max().item() <= parity.BWD_REL_FRO * g[:, h].abs().sum(0).max().item()
        sk = dk[:, h].double().sum(0)
        assert sk.abs().max().item() <= parity.BWD_REL_FRO * dk[:, h].double().abs().sum(0).max().item()
