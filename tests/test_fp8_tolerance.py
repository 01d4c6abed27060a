"""The FP8 tolerance of tests/parity.py (fp8_sigma / fp8_check) against a CPU model of the
kernel's arithmetic: the model must pass, and plausible kernel mistakes must fail.

The model follows the FP8 kernel's steps as its header states them: keys in tiles of 128,
x = scale * log2(e) * (q_hat . k_hat), a shift m set by the first tile and moved only when a
tile's maximum exceeds it by more than 4, P8 = E4M3(2^(x - m + 4)), O = sum P8 v_hat, output =
O / sum P8, lse from the unrounded weights.  It is written in fp64 with the oracle's E4M3
rounding (test infrastructure), independent of the CUDA code.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
import workloads
from tests import parity

RESCALE, PSHIFT = 4.0, 4.0


def _model_rows(qh, kh, vh, cu, scale, tok, head, mistake=None):
    c = scale / np.log(2.0)
    out = np.empty((len(tok), vh.shape[2]))
    lse = np.empty(len(tok))
    for i, (t, h) in enumerate(zip(tok, head)):
        s = np.searchsorted(cu, t, side="right") - 1
        b, e = cu[s], cu[s + 1]
        if mistake == "last_key_dropped":
            e = max(b + 1, e - 1)
        x = (kh[b:e, h] @ qh[t, h]) * c
        m, l, lr, o = None, 0.0, 0.0, np.zeros(vh.shape[2])
        for j in range(0, e - b, 128):
            xt = x[j:j + 128]
            mx = xt.max()
            if m is None:
                m = mx
            elif mx > m + RESCALE:
                a = 2.0 ** (m - mx)
                l, lr, o, m = l * a, lr * a, o * a, mx
            p = 2.0 ** (xt - m + PSHIFT)
            p8 = fp8.e4m3_round(p.astype(np.float32))
            vt = vh[b + j:b + j + len(xt), h]
            if mistake == "v_scale_of_channel_0":
                vt = vt / vh.std(axis=0)[h] * vh.std(axis=0)[h][0]
            l += p.sum()
            lr += p8.sum()
            o += p8 @ vt
        out[i] = o / lr
        lse[i] = (m - PSHIFT + np.log2(l)) * np.log(2.0)
    return out, lse


def _setup(segs, heads, seed, outliers=False):
    cfg = dict(segments=segs, heads=heads, head_dim=128, seed=seed, scale=1 / np.sqrt(128))
    if outliers:
        cfg["key_outliers"] = dict(fraction=0.01, factor=8)
    p = workloads.make_inputs(cfg)
    qz = fp8.quantize_qkv(p["q"], p["k"], p["v"])
    # give the value channels different ranges, so a per-channel scale matters
    qh, kh, vh = fp8.dequantized_qkv(qz)
    vh = vh * np.linspace(0.5, 2.0, vh.shape[2])[None, None, :]
    cu = p["cu_seqlens"].numpy().astype(np.int64)
    rng = np.random.default_rng(seed)
    T = sum(segs)
    tok = rng.integers(0, T, 120)
    head = rng.integers(0, heads, 120).astype(np.int32)
    ref, rlse = oracle.varlen_attention(qh, kh, vh, cu, cfg["scale"], rows=(tok, head))
    sig, bias = parity.fp8_sigma(qh, kh, vh, cu, cfg["scale"], tok, head, ref)
    return qh, kh, vh, cu, cfg["scale"], tok, head, ref, rlse, (sig, bias)


@pytest.fixture(scope="module")
def packs():
    return {"ragged": _setup([300, 1, 129, 700], 2, 3), "outliers": _setup([2048], 2, 4, outliers=True)}


@pytest.mark.parametrize("name", ["ragged", "outliers"])
def test_model_of_the_kernel_passes(packs, name):
    qh, kh, vh, cu, scale, tok, head, ref, rlse, sig = packs[name]
    out, lse = _model_rows(qh, kh, vh, cu, scale, tok, head)
    # the kernel's output is bf16
    out = torch.from_numpy(out).to(torch.bfloat16).double().numpy()
    errs = parity.fp8_check(out, lse, ref, rlse, *sig, name)
    assert errs["worst_over_bound"] < 0.8


@pytest.mark.parametrize("mistake", ["last_key_dropped", "v_scale_of_channel_0"])
def test_kernel_mistakes_fail(packs, mistake):
    qh, kh, vh, cu, scale, tok, head, ref, rlse, sig = packs["ragged"]
    out, lse = _model_rows(qh, kh, vh, cu, scale, tok, head, mistake=mistake)
    with pytest.raises(AssertionError):
        parity.fp8_check(out, lse, ref, rlse, *sig, mistake)
