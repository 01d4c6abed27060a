"""The comparison helpers used by the GPU parity tests (CPU only)."""
import numpy as np
import torch

from tests import parity


def _bf16_step(x):
    """Distance from the bf16 grid point 2^floor(log2|x|) to the next bf16 value (bit pattern + 1)."""
    g = torch.tensor([2.0 ** np.floor(np.log2(abs(x)))], dtype=torch.bfloat16)
    bits = g.view(torch.int16) + 1
    return float(bits.view(torch.bfloat16).float() - g.float())


def test_bf16_ulp_matches_the_bf16_grid():
    xs = np.array([0.3, 1.0, 1.7, 2.0, 3.99, 4.0, 4.37, 100.0, -6.5])
    assert np.array_equal(parity.bf16_ulp(xs), [_bf16_step(x) for x in xs])


def test_bound_is_stated_value_below_two_and_one_ulp_above():
    ref = np.array([0.5, 1.9, 4.5])
    ok = ref + np.array([0.0149, -0.0149, 0.031])
    bad = ref + np.array([0.0151, 0.0, 0.0])
    lse = np.zeros(3)
    assert parity.errors(ok, lse, ref, lse)["bound_ratio"] <= 1.0
    assert parity.errors(bad, lse, ref, lse)["bound_ratio"] > 1.0


def test_packing_layouts():
    import workloads
    lays = workloads.packing_layouts([100, 400, 250, 0, 50, 300], bucket_size=2)
    assert lays["packed"]["segments"] == [100, 400, 250, 50, 300]
    assert lays["padded"]["segments"] == [400] * 5
    assert lays["bucketed"]["segments"] == [100, 100, 300, 300, 400]  # sorted 50,100 | 250,300 | 400
    assert abs(lays["padded"]["token_utilisation"] - 1100 / 2000) < 1e-12
    assert abs(lays["bucketed"]["token_utilisation"] - 1100 / 1200) < 1e-12
    assert lays["packed"]["token_utilisation"] == 1.0
