"""The fp64 oracle against what the pages and the mathematics fix (CPU only)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests import oracle_pins as pins


@pytest.mark.parametrize("check", pins.ALL_CHECKS + [pins.check_token_counts], ids=lambda c: c.__name__)
def test_pin(check):
    check()


def test_sampled_rows_equal_full_rows():
    lens, H, d = [40, 3, 77], 3, 8
    rng = np.random.default_rng(1)
    q, k, v = (rng.normal(size=(sum(lens), H, d)) for _ in range(3))
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, lse = oracle.varlen_attention(q, k, v, cu, 0.35)
    tok = np.array([0, 39, 40, 42, 43, 119, 7], dtype=np.int64)
    hd = np.array([0, 2, 1, 1, 0, 2, 2], dtype=np.int32)
    o2, l2 = oracle.varlen_attention(q, k, v, cu, 0.35, rows=(tok, hd))
    assert np.array_equal(o2, out[tok, hd]) and np.array_equal(l2, lse[tok, hd])


def test_bf16_inputs_widen_exactly():
    p = workloads.random_pack([19, 5], heads=2, head_dim=16, seed=9)
    o_bf, l_bf = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"])
    f = lambda t: t.to(torch.float64).numpy()
    o64, l64 = oracle.varlen_attention(f(p["q"]), f(p["k"]), f(p["v"]), p["cu_seqlens"], p["scale"])
    assert np.array_equal(o_bf, o64) and np.array_equal(l_bf, l64)


def test_thread_count_does_not_change_results():
    p = workloads.random_pack([300, 45], heads=2, head_dim=32, seed=2)
    a = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"], n_threads=1)
    b = oracle.varlen_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["scale"], n_threads=0)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("cu", [[1, 4, 6], [0, 4, 3, 6], [0, 2, 5]])
def test_invalid_cu_seqlens_rejected(cu):
    q = np.zeros((6, 1, 2))
    with pytest.raises(ValueError):
        oracle.varlen_attention(q, q, q, cu, 1.0)


def test_empty_pack():
    q = np.zeros((0, 2, 4))
    out, lse = oracle.varlen_attention(q, q, q, [0], 1.0)
    assert out.shape == (0, 2, 4) and lse.shape == (0, 2)


def test_frozen_configs():
    """Frozen packs match the pages' resolutions and the documented training-pack draw."""
    from workloads import freeze_configs
    got = {c["name"]: c for c in workloads.all_configs()}
    assert got["tiny"]["segments"] == [256, 108]
    assert got["mixed"]["segments"] == [1024, 4096, 1296] and got["mixed"]["total_tokens"] == 6416
    assert got["interactive"]["segments"] == [16384]
    assert got["long"]["segments"] == [65536]
    seed, imgs = freeze_configs.search_training_pack()
    assert seed == got["training"]["pack_seed"] and imgs == got["training"]["images"]
    assert sum(got["training"]["segments"]) == got["training"]["total_tokens"] == 40808
    for c in got.values():
        assert c["scale"] == 1.0 / math.sqrt(c["head_dim"])


def test_interactive_outliers_are_exact_powers_of_two():
    cfg = dict(workloads.load_config("interactive"))
    cfg["segments"] = [1000]  # same recipe on a smaller pack
    p = workloads.make_inputs(cfg)
    idx = p["outlier_rows"]
    assert idx.numel() == 10 and len(set(idx.tolist())) == 10
    _, k0, _, _ = workloads.random_qkv(1000, cfg["heads"], cfg["head_dim"], cfg["seed"])
    assert torch.equal(p["k"][idx].float(), k0[idx].float() * 8)
    rest = torch.ones(1000, dtype=torch.bool); rest[idx] = False
    assert torch.equal(p["k"][rest], k0[rest])


def test_sampled_rows_are_distinct_per_head():
    cfg = workloads.load_config("long")
    tok, hd = workloads.sampled_rows(cfg)
    assert tok.numel() == 512 * 8
    for h in range(8):
        t = tok[hd == h]
        assert t.unique().numel() == 512 and int(t.max()) < 65536
