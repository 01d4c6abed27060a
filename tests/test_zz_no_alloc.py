"""pa_varlen_attn_fwd_noalloc through the C ABI (needs a B200).

That entry point is for callers that cannot let the library allocate device
memory: a framework whose caching allocator or arena owns the GPU's memory, a
plug-in host that forbids allocation where it calls us, or a serving loop that
stops allocating after warm-up.  It runs the same kernels as pa_varlen_attn_fwd
but keeps its workspace in a fixed array of the library's device image, shared
by every call on a GPU.  These tests check that two calls in a row through that
shared array give what the allocating entry point gives, and that its status
word and size limit behave as declared.  The file name makes pytest collect it
last; it also passes alone in a fresh process, where its first call is the one
that sets up the array.
"""
import pytest
import torch

import dit_resolution_packed_b200 as pa
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


def _to_dev(p, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in p.items()}


def _caller_buffers(g):
    """The caller's own out, lse and status buffers (allocated by the caller, not by the library)."""
    T, H, _ = g["q"].shape
    out = torch.full_like(g["q"], 3.0)
    lse = torch.full((T, H), 3.0, dtype=torch.float32, device=g["q"].device)
    status = torch.full((1,), -99, dtype=torch.int32, device=g["q"].device)
    return out, lse, status


def _noalloc(g, p, out, lse, status, cu=None, max_seqlen=None):
    return pa.pa_varlen_attn_fwd_noalloc(g["q"], g["k"], g["v"], g["cu_seqlens"] if cu is None else cu,
                                         g["max_seqlen"] if max_seqlen is None else max_seqlen, p["scale"],
                                         out, lse, status)


def _allocating(g, p):
    out, lse = pa.varlen_attn_fwd(g["q"], g["k"], g["v"], g["cu_seqlens"], g["max_seqlen"], p["scale"])
    rc = pa.pa_get_error()
    assert rc == pa.PA_OK, pa.status_string(rc)
    return out, lse


def test_two_calls_in_a_row_match_the_allocating_entry_point(cuda_device):
    # the first call has more segments than the second, so the second runs on a
    # scratch array that still holds the first call's longer schedule and maps
    packs = [workloads.random_pack([1, 127, 128, 129, 257, 513, 1000, 3], heads=3, head_dim=128, seed=31),
             workloads.random_pack([5, 300, 64, 700], heads=2, head_dim=64, seed=32)]
    devs = [_to_dev(p, cuda_device) for p in packs]
    bufs = [_caller_buffers(g) for g in devs]
    torch.cuda.synchronize()
    for g, p, (out, lse, status) in zip(devs, packs, bufs):
        assert _noalloc(g, p, out, lse, status) == pa.PA_OK
    torch.cuda.synchronize()
    for g, p, (out, lse, status) in zip(devs, packs, bufs):
        assert int(status.item()) == pa.PA_OK
        ref_o, ref_l = _allocating(g, p)
        errs = parity.errors(out.double().cpu().numpy(), lse.double().cpu().numpy(),
                             ref_o.double().cpu().numpy(), ref_l.double().cpu().numpy())
        parity.check(errs)
        # the same kernels run on the same schedule: the results agree bit for bit
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l), errs


def test_status_word_reports_device_errors_and_is_cleared_by_the_next_call(cuda_device):
    p = workloads.random_pack([100, 50], heads=2, head_dim=64, seed=33)
    g = _to_dev(p, cuda_device)
    out, lse, status = _caller_buffers(g)
    bad = torch.tensor([0, 120, 100], dtype=torch.int32, device=cuda_device)
    assert _noalloc(g, p, out, lse, status, cu=bad) == pa.PA_OK  # enqueued; the device finds the problem
    torch.cuda.synchronize()
    assert int(status.item()) == pa.PA_ERR_CU_SEQLENS
    assert _noalloc(g, p, out, lse, status, max_seqlen=99) == pa.PA_OK
    torch.cuda.synchronize()
    assert int(status.item()) == pa.PA_ERR_MAX_SEQLEN
    assert _noalloc(g, p, out, lse, status) == pa.PA_OK
    torch.cuda.synchronize()
    assert int(status.item()) == pa.PA_OK
    ref_o, ref_l = _allocating(g, p)
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    # without a status buffer the call still runs (errors then go unreported)
    out2, lse2, _ = _caller_buffers(g)
    assert _noalloc(g, p, out2, lse2, None) == pa.PA_OK
    torch.cuda.synchronize()
    assert torch.equal(out2, ref_o) and torch.equal(lse2, ref_l)


def test_rejects_more_segments_than_its_scratch_holds(cuda_device):
    lens = [1] * (pa.NOALLOC_MAX_BATCH + 1)
    p = workloads.random_pack(lens, heads=1, head_dim=64, seed=34)
    g = _to_dev(p, cuda_device)
    out, lse, status = _caller_buffers(g)
    assert _noalloc(g, p, out, lse, status) == pa.PA_ERR_NOALLOC_LIMIT
    torch.cuda.synchronize()
    assert int(status.item()) == -99  # nothing was enqueued
    # exactly at the limit it runs and matches the allocating entry point
    p = workloads.random_pack([1 + (i % 7) for i in range(pa.NOALLOC_MAX_BATCH)], heads=1, head_dim=64, seed=35)
    g = _to_dev(p, cuda_device)
    out, lse, status = _caller_buffers(g)
    assert _noalloc(g, p, out, lse, status) == pa.PA_OK
    torch.cuda.synchronize()
    assert int(status.item()) == pa.PA_OK
    ref_o, ref_l = _allocating(g, p)
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
