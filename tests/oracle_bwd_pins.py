"""Checks that pin the fp64 gradient oracle to facts outside itself.

Each ``check_*`` takes a library handle holding ``oracle_varlen_attn_bwd``
(``None`` = the committed oracle) and raises ``AssertionError`` on a mismatch.
``test_oracle_bwd_pins.py`` runs them on the committed oracle,
``test_oracle_bwd_mutants.py`` on copies with planted mistakes.

What pins the gradients:
  * central finite differences of the forward oracle (itself pinned by
    ``oracle_pins.py``): the gradient of sum(out * G) with respect to every
    element of q, k and v;
  * torch autograd in fp64 through the materialised masked attention (the
    whole [T, T] score matrix, -inf outside the block diagonal): a library
    special case of the same definition;
  * closed forms: the softmax Jacobian annihilates constants, so over each
    segment and head sum_j dk_j = 0 and sum_j dv_j = sum_r dout_r; a
    one-token segment has dq = dk = 0 and dv = dout; q = 0 gives uniform
    weights, so dv_j = (sum_r dout_r) / L for every key j;
  * segment-order invariance, bf16-input widening, and the sampled-row mode
    agreeing with the full mode.
"""
import numpy as np
import torch

import oracle


def _pack(seed=0, lens=(3, 5, 0, 4, 1), heads=2, d=3, dv=2, q_zero=False):
    rng = np.random.default_rng(seed)
    T = int(sum(lens))
    q = np.zeros((T, heads, d)) if q_zero else rng.standard_normal((T, heads, d))
    k = rng.standard_normal((T, heads, d))
    v = rng.standard_normal((T, heads, dv))
    g = rng.standard_normal((T, heads, dv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, g, cu


def _bwd(lib, q, k, v, g, cu, scale):
    return oracle.varlen_attention_bwd(q, k, v, g, cu, scale, n_threads=2, lib=lib)


def check_finite_differences(lib):
    """dq, dk, dv equal the central differences of sum(out * G) (forward oracle, fp64)."""
    q, k, v, g, cu = _pack(seed=1)
    scale = 0.7
    dq, dk, dv = _bwd(lib, q, k, v, g, cu, scale)

    def f(x):
        out, _ = oracle.varlen_attention(x["q"], x["k"], x["v"], cu, scale, n_threads=1)
        return float(np.sum(out * g))

    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        base = {"q": q, "k": k, "v": v}
        num = np.zeros_like(base[name])
        for idx in np.ndindex(base[name].shape):
            plus = dict(base); plus[name] = base[name].copy(); plus[name][idx] += eps
            minus = dict(base); minus[name] = base[name].copy(); minus[name][idx] -= eps
            num[idx] = (f(plus) - f(minus)) / (2 * eps)
        err = float(np.max(np.abs(grad - num)))
        assert err < 1e-7, (name, err)


def check_autograd(lib):
    """fp64 torch autograd through the materialised block-diagonal attention."""
    q, k, v, g, cu = _pack(seed=2, lens=(7, 1, 0, 12, 5), heads=3, d=4, dv=3)
    scale = -0.45
    dq, dk, dv = _bwd(lib, q, k, v, g, cu, scale)
    T = q.shape[0]
    seg = np.zeros(T, dtype=np.int64)
    for i in range(len(cu) - 1):
        seg[cu[i]:cu[i + 1]] = i
    mask = torch.from_numpy(seg[:, None] == seg[None, :])
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    outs = []
    for h in range(q.shape[1]):
        s = scale * (tq[:, h, :] @ tk[:, h, :].T)
        s = s.masked_fill(~mask, float("-inf"))
        outs.append(torch.softmax(s, dim=-1) @ tv[:, h, :])
    out = torch.stack(outs, dim=1)
    (out * torch.from_numpy(g)).sum().backward()
    for name, a, b in (("q", dq, tq.grad), ("k", dk, tk.grad), ("v", dv, tv.grad)):
        err = float(np.max(np.abs(a - b.numpy())))
        assert err < 1e-12, (name, err)


def check_closed_forms(lib):
    """sum_j dk_j = 0 and sum_j dv_j = sum_r dout_r per segment and head."""
    q, k, v, g, cu = _pack(seed=3, lens=(9, 2, 16, 0, 5), heads=2, d=5, dv=4)
    dq, dk, dv = _bwd(lib, q, k, v, g, cu, 0.6)
    for i in range(len(cu) - 1):
        a, b = cu[i], cu[i + 1]
        if a == b:
            continue
        assert np.max(np.abs(dk[a:b].sum(axis=0))) < 1e-12
        assert np.max(np.abs(dv[a:b].sum(axis=0) - g[a:b].sum(axis=0))) < 1e-12


def check_special_cases(lib):
    """One-token segments: dq = dk = 0, dv = dout.  q = 0: dv_j = mean of dout over the segment times 1."""
    q, k, v, g, cu = _pack(seed=4, lens=(1, 1, 1), heads=2, d=3, dv=3)
    dq, dk, dv = _bwd(lib, q, k, v, g, cu, 1.3)
    assert np.max(np.abs(dq)) == 0.0 and np.max(np.abs(dk)) == 0.0
    assert np.max(np.abs(dv - g)) < 1e-15
    q, k, v, g, cu = _pack(seed=5, lens=(4, 6), heads=2, d=3, dv=2, q_zero=True)
    dq, dk, dv = _bwd(lib, q, k, v, g, cu, 0.9)
    assert np.max(np.abs(dk)) == 0.0  # dk_j = scale * sum_r dS_rj q_r with q = 0
    for i in range(len(cu) - 1):
        a, b = cu[i], cu[i + 1]
        expect = g[a:b].sum(axis=0) / (b - a)
        assert np.max(np.abs(dv[a:b] - expect[None])) < 1e-14


def check_permutation(lib):
    """Reordering the segments of the pack reorders the gradients, bit for bit."""
    lens = [5, 3, 8, 2]
    q, k, v, g, cu = _pack(seed=6, lens=tuple(lens), heads=2, d=4, dv=3)
    dq, dk, dv = _bwd(lib, q, k, v, g, cu, 0.8)
    perm = [2, 0, 3, 1]
    idx = np.concatenate([np.arange(cu[i], cu[i + 1]) for i in perm])
    cu2 = np.concatenate([[0], np.cumsum([lens[i] for i in perm])])
    dq2, dk2, dv2 = _bwd(lib, q[idx], k[idx], v[idx], g[idx], cu2, 0.8)
    assert np.array_equal(dq2, dq[idx]) and np.array_equal(dk2, dk[idx]) and np.array_equal(dv2, dv[idx])


def check_bf16_inputs_and_rows(lib):
    """bf16 inputs give the gradients of their exact fp64 values; the sampled-row mode
    returns the same dq rows as the full mode."""
    q, k, v, g, cu = _pack(seed=7, lens=(6, 11, 3), heads=2, d=4, dv=4)
    tb = [torch.from_numpy(x).to(torch.bfloat16) for x in (q, k, v, g)]
    full = oracle.varlen_attention_bwd(*tb, cu, 0.5, n_threads=2, lib=lib)
    wide = _bwd(lib, *[t.double().numpy() for t in tb], cu, 0.5)
    for a, b in zip(full, wide):
        assert np.array_equal(a, b)
    rows = (np.array([0, 7, 19, 12, 5], dtype=np.int64), np.array([1, 0, 1, 1, 0], dtype=np.int32))
    dq_rows = oracle.varlen_attention_bwd(*tb, cu, 0.5, rows=rows, n_threads=2, lib=lib)
    assert np.array_equal(dq_rows, full[0][rows[0], rows[1]])


ALL_CHECKS = [check_finite_differences, check_autograd, check_closed_forms, check_special_cases,
              check_permutation, check_bf16_inputs_and_rows]
