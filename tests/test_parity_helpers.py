"""The comparison helpers used by the GPU parity tests (CPU only)."""
import numpy as np
import torch

from tests import parity


def test_bf16_ulp_matches_the_bf16_grid():
    xs = np.array([0.3, 1.0, 1.7, 2.0, 3.99, 4.0, 4.37, 100.0, -6.5])
    for x, u in zip(xs, parity.bf16_ulp(xs)):
        b = torch.tensor(abs(x), dtype=torch.float32).to(torch.bfloat16)
        nxt = torch.nextafter(b.float(), torch.tensor(float("inf"))).to(torch.bfloat16)
        # the next representable bf16 above a grid point is one ulp away
        grid = torch.tensor(2.0 ** np.floor(np.log2(abs(x))), dtype=torch.bfloat16)
        step = (torch.nextafter(grid.float(), torch.tensor(float("inf"))).to(torch.bfloat16).float() - grid.float())
        assert abs(float(step) - u) == 0.0, (x, float(step), u)
        del b, nxt


def test_bound_is_stated_value_below_two_and_one_ulp_above():
    ref = np.array([0.5, 1.9, 4.5])
    ok = ref + np.array([0.0149, -0.0149, 0.031])
    bad = ref + np.array([0.0151, 0.0, 0.0])
    lse = np.zeros(3)
    assert parity.errors(ok, lse, ref, lse)["bound_ratio"] <= 1.0
    assert parity.errors(bad, lse, ref, lse)["bound_ratio"] > 1.0
