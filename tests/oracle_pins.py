"""Checks that pin the fp64 oracle to facts outside itself.

Each ``check_*`` function takes an oracle library handle (``None`` = the
committed oracle) and raises ``AssertionError`` when the oracle disagrees with
what the pages or the mathematics fix.  ``test_oracle_pins.py`` runs them on
the committed oracle; ``test_oracle_mutants.py`` runs them on copies of the
oracle with planted mistakes and requires every mistake to be caught.
"""
import json
import math
import os

import numpy as np
import torch

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def brute_force(q, k, v, cu, scale):
    """Materialised masked softmax: the whole [T, T] score matrix per head, -inf
    outside the block diagonal, then a row softmax and a matmul (GigaPath-Flash
    page 4.1 naive attention; SparseAttn page section 04 masked attention)."""
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    T, H, _ = q.shape
    seg = np.zeros(T, dtype=np.int64)
    for i in range(len(cu) - 1):
        seg[cu[i]:cu[i + 1]] = i
    mask = seg[:, None] == seg[None, :]
    out = np.empty((T, H, v.shape[2])); lse = np.empty((T, H))
    for h in range(H):
        s = scale * (q[:, h, :] @ k[:, h, :].T)
        s = np.where(mask, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        out[:, h, :] = (e / z) @ v[:, h, :]
        lse[:, h] = (m + np.log(z))[:, 0]
    return out, lse


def _rand(T, H, d, dv, seed):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(T, H, d)), rng.normal(size=(T, H, d)), rng.normal(size=(T, H, dv))


def check_token_counts(lib=None):
    """Mage-Flow page, packing section: 512^2 -> 1024, 1024^2 -> 4096, 768x432 -> 1296 tokens."""
    assert workloads.tokens_for_image(512, 512) == 1024
    assert workloads.tokens_for_image(1024, 1024) == 4096
    assert workloads.tokens_for_image(768, 432) == 1296
    assert workloads.cu_seqlens_from_lengths([1024, 4096, 1296]).tolist() == [0, 1024, 5120, 6416]


def check_counterexample(lib=None):
    """SparseAttn page 3.2 / 09: weights 0.99 / 0.01 over values 0 / 100 give output 1; dropping key 2 gives 0."""
    g = _golden("counterexample.json")
    k0 = math.log(99.0)
    # One segment of two tokens; row 0 is the page's query.  Row 1 is an extra query (q = 0).
    q = np.array([[[1.0]], [[0.0]]]); k = np.array([[[k0]], [[0.0]]]); v = np.array([[[0.0]], [[100.0]]])
    out, lse = oracle.varlen_attention(q, k, v, [0, 2], 1.0, lib=lib)
    assert abs(out[0, 0, 0] - g["dense_output"]) <= 1e-12
    assert abs(lse[0, 0] - math.log(100.0)) <= 1e-12
    # q = 0 row: equal weights, mean of the values, lse = ln 2
    assert abs(out[1, 0, 0] - 50.0) <= 1e-12 and abs(lse[1, 0] - math.log(2.0)) <= 1e-12
    # restricted to the first key: two segments of one token each
    out, lse = oracle.varlen_attention(q, k, v, [0, 1, 2], 1.0, lib=lib)
    assert out[0, 0, 0] == g["pruned_output"]
    assert abs(lse[0, 0] - math.log(99.0)) <= 1e-12


def _example_heads_layout(ex):
    q = ex["q"].transpose(1, 0, 2).copy()
    k = ex["k"].transpose(1, 0, 2).copy()
    v = np.stack([ex["v"], ex["v"]], axis=1)
    return q, k, v


def _close10(got, printed):
    """Agreement with a number printed as text, to half a unit in its last printed place
    (plus a little slack for the page's own floating-point rounding)."""
    mant = printed.lower().split("e")
    exp = int(mant[1]) if len(mant) > 1 else 0
    decimals = len(mant[0].split(".")[1]) if "." in mant[0] else 0
    unit = 10.0 ** (exp - decimals)
    return abs(got - float(printed)) <= 0.51 * unit


def check_worked_example(lib=None):
    """SparseAttn page section 04 table: same-frame and (permuted) same-position masks vs full attention."""
    g = _golden("sparseattn_worked_example.json")
    ex = workloads.sparseattn_worked_example()
    q, k, v = _example_heads_layout(ex)
    scale = 1.0 / math.sqrt(20.0)
    full, lse_full = oracle.varlen_attention(q, k, v, [0, 64], scale, lib=lib)
    sf = g["same_frame"]
    y, lse = oracle.varlen_attention(q, k, v, sf["cu_seqlens"], scale, lib=lib)
    vmax = np.linalg.norm(ex["v"], axis=-1).max()
    for h in (0, 1):
        want = sf[f"head{h}"]
        retained = np.exp(lse[:, h] - lse_full[:, h])  # kept probability mass z_i (section 3.1)
        assert _close10(retained.mean(), want["retained_mass_mean"]), (h, retained.mean())
        mse = np.mean((y[:, h] - full[:, h]) ** 2)
        assert _close10(mse, want["mse_vs_full"]), (h, mse)
        if "max_row_error" in want:
            err = np.linalg.norm(y[:, h] - full[:, h], axis=-1)
            bound = 2.0 * np.maximum(0.0, 1.0 - retained) * vmax
            assert _close10(err.max(), want["max_row_error"])
            assert _close10(bound.max(), want["max_bound"])
            assert np.all(err <= bound + 1e-12)  # section 3.2 row bound
    sp = g["same_position_permuted"]
    perm = np.argsort(ex["position"], kind="stable")
    yp, lp = oracle.varlen_attention(q[perm], k[perm], v[perm], sp["cu_seqlens"], scale, lib=lib)
    y = np.empty_like(yp); y[perm] = yp
    lse = np.empty_like(lp); lse[perm] = lp
    for h in (0, 1):
        want = sp[f"head{h}"]
        retained = np.exp(lse[:, h] - lse_full[:, h])
        assert _close10(retained.mean(), want["retained_mass_mean"]), (h, retained.mean())
        assert _close10(np.mean((y[:, h] - full[:, h]) ** 2), want["mse_vs_full"])


def check_brute_force(lib=None):
    """Oracle equals the materialised masked softmax (naive attention) on small ragged packs."""
    cases = [([5, 1, 17, 9], 3, 7, 5, 0.37), ([33, 2, 64], 2, 16, 16, 0.125), ([1], 1, 3, 2, -0.8),
             ([0, 12, 0, 4], 2, 8, 3, 0.5)]
    for i, (lens, H, d, dv, scale) in enumerate(cases):
        T = sum(lens)
        q, k, v = _rand(T, H, d, dv, 100 + i)
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        out, lse = oracle.varlen_attention(q, k, v, cu, scale, lib=lib)
        bo, bl = brute_force(q, k, v, cu, scale)
        assert np.max(np.abs(out - bo)) <= 1e-12, i
        assert np.max(np.abs(lse - bl)) <= 1e-12, i


def check_sdpa(lib=None):
    """Oracle equals torch's fp64 scaled_dot_product_attention run per segment (a library special case)."""
    lens, H, d = [7, 40, 13], 3, 16
    q, k, v = _rand(sum(lens), H, d, d, 7)
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, _ = oracle.varlen_attention(q, k, v, cu, 0.25, lib=lib)
    for i in range(len(lens)):
        a, b = cu[i], cu[i + 1]
        t = lambda x: torch.from_numpy(x[a:b]).transpose(0, 1)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=0.25)[0].transpose(0, 1)
        assert np.max(np.abs(out[a:b] - ref.numpy())) <= 1e-12


def check_permutation(lib=None):
    """Reordering whole segments permutes the outputs and nothing else (SparseAttn page 3.4); bit-exact."""
    lens, H, d = [9, 30, 1, 17], 2, 8
    q, k, v = _rand(sum(lens), H, d, d, 11)
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, lse = oracle.varlen_attention(q, k, v, cu, 0.3, lib=lib)
    order = [2, 0, 3, 1]
    idx = np.concatenate([np.arange(cu[i], cu[i + 1]) for i in order])
    cu2 = np.concatenate([[0], np.cumsum([lens[i] for i in order])])
    out2, lse2 = oracle.varlen_attention(q[idx], k[idx], v[idx], cu2, 0.3, lib=lib)
    assert np.array_equal(out2, out[idx]) and np.array_equal(lse2, lse[idx])


def check_equal_scores(lib=None):
    """q = 0 gives equal weights: the output is the segment's mean value row and lse = ln L."""
    lens, H, d = [3, 10, 1], 2, 4
    _, k, v = _rand(sum(lens), H, d, d, 3)
    q = np.zeros_like(k)
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, lse = oracle.varlen_attention(q, k, v, cu, 0.7, lib=lib)
    for i, n in enumerate(lens):
        a, b = cu[i], cu[i + 1]
        assert np.max(np.abs(out[a:b] - v[a:b].mean(axis=0, keepdims=True))) <= 1e-13
        assert np.max(np.abs(lse[a:b] - math.log(n))) <= 1e-13


def check_identical_values(lib=None):
    """Weights sum to one, so identical value rows give exactly that row (SparseAttn page 3.1)."""
    lens, H, d = [6, 21], 2, 5
    q, k, _ = _rand(sum(lens), H, d, d, 4)
    v = np.empty((sum(lens), H, 3))
    v[:6] = [1.5, -2.0, 0.25]
    v[6:] = [-7.0, 3.0, 0.5]
    out, _ = oracle.varlen_attention(q, k, v, [0, 6, 27], 0.9, lib=lib)
    assert np.max(np.abs(out[:6] - v[:6])) <= 1e-14 and np.max(np.abs(out[6:] - v[6:])) <= 1e-13


def check_single_token(lib=None):
    """A one-token segment returns its own value row and lse = scale * q . k."""
    q, k, v = _rand(3, 2, 6, 4, 5)
    out, lse = oracle.varlen_attention(q, k, v, [0, 1, 2, 3], 0.6, lib=lib)
    assert np.array_equal(out, v)
    assert np.max(np.abs(lse - 0.6 * np.einsum("thc,thc->th", q, k))) <= 1e-14


ALL_CHECKS = [check_counterexample, check_worked_example, check_brute_force, check_sdpa,
              check_permutation, check_equal_scores, check_identical_values, check_single_token]
