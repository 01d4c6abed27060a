"""The projection oracle (fused QKV + RoPE, output projection) against facts outside itself."""
import numpy as np
import torch

from oracle import proj


def _rng(seed):
    return np.random.default_rng(seed)


def test_linear_is_the_matrix_product_and_split_order():
    rng = _rng(0)
    x, w = rng.standard_normal((7, 12)), rng.standard_normal((30, 12))
    np.testing.assert_allclose(proj.linear(x, w), np.einsum("tc,oc->to", x, w), rtol=0, atol=1e-12)
    # the q / k / v slices are consecutive blocks of W_qkv's rows, head-major inside each
    H, d = 2, 5
    w = rng.standard_normal((3 * H * d, 12))
    q, k, v = proj.qkv_rope(x, w, [0, 7], H, d, theta=0.0)
    np.testing.assert_allclose(q[3, 1], x[3] @ w[1 * d:2 * d].T, atol=1e-12)
    np.testing.assert_allclose(k[2, 0], x[2] @ w[H * d:H * d + d].T, atol=1e-12)
    np.testing.assert_allclose(v[6, 1], x[6] @ w[2 * H * d + d:2 * H * d + 2 * d].T, atol=1e-12)


def test_rope_matches_complex_rotation():
    """Each pair (x_i, x_{i+d/2}) is the complex number x_i + i x_{i+d/2} times e^{i p theta_i}."""
    rng = _rng(1)
    T, H, d, theta = 9, 3, 8, 10000.0
    x = rng.standard_normal((T, H, d))
    pos = rng.integers(0, 5000, size=T)
    got = proj.rope(x, pos, theta)
    z = (x[..., :d // 2] + 1j * x[..., d // 2:]) * np.exp(
        1j * pos[:, None, None] * theta ** (-2.0 * np.arange(d // 2) / d)[None, None, :])
    np.testing.assert_allclose(got[..., :d // 2], z.real, atol=1e-12)
    np.testing.assert_allclose(got[..., d // 2:], z.imag, atol=1e-12)


def test_rope_invariants():
    rng = _rng(2)
    T, d, theta = 6, 16, 500.0
    q, k = rng.standard_normal((T, 1, d)), rng.standard_normal((T, 1, d))
    # position 0 is the identity; rotations keep the norm
    np.testing.assert_allclose(proj.rope(q, np.zeros(T, int), theta), q, atol=0)
    pos = np.arange(T) * 37
    np.testing.assert_allclose(np.linalg.norm(proj.rope(q, pos, theta), axis=-1), np.linalg.norm(q, axis=-1),
                               rtol=1e-13)
    # relative positions: <R(m) q, R(n) k> depends on m - n only
    m, n, s = 11, 4, 23
    def dot(pm, pn):
        return float(np.sum(proj.rope(q[:1], [pm], theta) * proj.rope(k[:1], [pn], theta)))
    assert abs(dot(m, n) - dot(m + s, n + s)) < 1e-12


def test_positions_restart_at_every_segment():
    np.testing.assert_array_equal(proj.positions([0, 3, 3, 5], 5), [0, 1, 2, 0, 1])


def test_qkv_rope_rotates_q_and_k_not_v_and_accepts_bf16():
    rng = _rng(3)
    T, C, H, d = 10, 16, 2, 8
    x = torch.from_numpy(rng.standard_normal((T, C))).to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((3 * H * d, C))).to(torch.bfloat16)
    cu = [0, 4, 10]
    q0, k0, v0 = proj.qkv_rope(x, w, cu, H, d, theta=0.0)
    q1, k1, v1 = proj.qkv_rope(x, w, cu, H, d, theta=1000.0)
    np.testing.assert_array_equal(v0, v1)
    pos = proj.positions(cu, T)
    np.testing.assert_allclose(q1, proj.rope(q0, pos, 1000.0), atol=1e-12)
    np.testing.assert_allclose(k1, proj.rope(k0, pos, 1000.0), atol=1e-12)
    np.testing.assert_allclose(q1[0], q0[0], atol=0)   # position 0 of the first image
    np.testing.assert_allclose(q1[4], q0[4], atol=0)   # position 0 of the second image
