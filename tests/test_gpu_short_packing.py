"""Short-segment packing on the GPU: several short images share one 128-row tile with an in-tile
block-diagonal mask.  Every row is compared with the fp64 oracle, with packing on and off, and
the device's tile ledger is compared with the scheduler's rules restated on the host."""
import numpy as np
import pytest
import torch

import dit_resolution_packed_b200 as pa
import oracle
import workloads
from tests import parity
from tests import schedule_model as sm

pytestmark = pytest.mark.gpu


@pytest.fixture
def packing(cuda_device):
    """Restores the library default (packing on) after a test that switches it."""
    yield pa.pa_set_short_packing
    pa.pa_set_short_packing(True)


def _check(p, dev, short_packing=True):
    pa.pa_set_short_packing(short_packing)
    g = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in p.items()}
    out, lse = pa.varlen_attn_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], g["max_seqlen"], p["scale"])
    rc = pa.pa_get_error()
    assert rc == pa.PA_OK, pa.status_string(rc)
    led = pa.pa_schedule_stats()
    ref_o, ref_l = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"])
    errs = parity.errors(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l)
    parity.check(errs)
    want = sm.ledger(p["segments"], p["heads"], short_packing)
    assert {k: led[k] for k in want} == want, (led, want)
    return out, lse, led


def _lengths(seed, n, lo, hi):
    return np.random.default_rng(seed).integers(lo, hi + 1, size=n).tolist()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("short_packing", [True, False])
def test_segments_of_1_to_127_tokens(cuda_device, packing, d, short_packing):
    lens = _lengths(60 + d, 300, 1, 127)
    _check(workloads.random_pack(lens, heads=3, head_dim=d, seed=61), cuda_device, short_packing)


@pytest.mark.parametrize("d", [64, 128])
def test_empty_and_one_token_segments(cuda_device, packing, d):
    lens = [0, 1, 0, 0, 1, 1, 5, 0, 127, 1, 0, 128, 0, 1, 64, 64, 1, 0] + [1] * 300 + [0, 0]
    _check(workloads.random_pack(lens, heads=2, head_dim=d, seed=62), cuda_device)


def test_short_runs_between_long_segments(cuda_device, packing):
    lens = [30, 90, 700, 1, 2, 3, 129, 128, 128, 0, 300, 17, 111, 64, 65, 1000, 5]
    _check(workloads.random_pack(lens, heads=2, head_dim=128, seed=63), cuda_device)


def test_runs_cut_at_token_blocks(cuda_device, packing):
    # 40 segments of 100 tokens: every 1024-token block starts a new walk
    _check(workloads.random_pack([100] * 40, heads=2, head_dim=64, seed=64), cuda_device)


def test_only_empty_segments_and_one_token(cuda_device, packing):
    _check(workloads.random_pack([0, 0, 1, 0], heads=1, head_dim=128, seed=65), cuda_device)


def test_many_one_token_segments_unstaged_schedule(cuda_device, packing):
    """5000 segments (more than the scheduler stages in shared memory) of 0-3 tokens:
    hundreds of segments per tile, walks of many ballots."""
    lens = _lengths(66, 5000, 0, 3)
    _check(workloads.random_pack(lens, heads=2, head_dim=64, seed=67), cuda_device)


@pytest.mark.parametrize("scale", [-0.2, 0.0])
def test_other_scales_in_groups(cuda_device, packing, scale):
    p = workloads.random_pack(_lengths(68, 50, 1, 60), heads=2, head_dim=128, seed=69, scale=scale)
    _check(p, cuda_device)


def test_guard_bands_with_groups(cuda_device, packing):
    """No write outside out / lse when rows of several segments share a tile."""
    p = workloads.random_pack([3, 50, 1, 74, 0, 100, 28, 2], heads=3, head_dim=64, seed=70)
    g = {k: (v.to(cuda_device) if torch.is_tensor(v) else v) for k, v in p.items()}
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


@pytest.mark.parametrize("name", workloads.SHORT_PACK_NAMES)
def test_short_segment_packs_all_rows(cuda_device, packing, name):
    """The benchmark's short-segment packs (300 small images; 2048 thumbnails), every row."""
    p = workloads.make_inputs(workloads.load_config(name))
    _, _, led = _check(p, cuda_device)
    print(f"\nledger {name}: {led}")


def test_ledger_of_the_configurations(cuda_device, packing):
    """The device's ledger of every workload configuration equals the host restatement."""
    for name in workloads.CONFIG_NAMES:
        cfg = workloads.load_config(name)
        segs = cfg["segments"]
        T, H, d = sum(segs), cfg["heads"], cfg["head_dim"]
        q = torch.zeros(T, H, d, dtype=torch.bfloat16, device=cuda_device)
        cu = workloads.cu_seqlens_from_lengths(segs).to(cuda_device)
        pa.varlen_attn_fwd(q, q, q, cu, max(segs))
        assert pa.pa_get_error() == pa.PA_OK
        led = pa.pa_schedule_stats()
        want = sm.ledger(segs, H)
        assert {k: led[k] for k in want} == want, (name, led, want)
