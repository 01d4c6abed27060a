"""Comparison helpers shared by the GPU parity tests, the smoke check and the benchmark.

Acceptance (stated for the packed attention forward): maximum absolute error of
the output <= 1.5e-2, relative Frobenius error <= 4e-3, and log-sum-exp within
an absolute error of 1e-3, against the fp64 oracle before any rounding.

Reading of the max-abs bound: the output is bf16, whose grid spacing (one ulp)
is 2^(e-7) for |x| in [2^e, 2^(e+1)).  For |x| >= 4 half an ulp is 2^-6 =
0.0156 > 1.5e-2, so even a perfectly rounded output could miss the bound.  The
per-element bound is therefore max(1.5e-2, one bf16 ulp of the oracle value):
the stated 1.5e-2 wherever the format can represent it (|x| < 2), and a
faithful rounding (within one ulp) where it cannot.
"""
import numpy as np

MAX_ABS = 1.5e-2
REL_FRO = 4e-3
LSE_ABS = 1e-3


def bf16_ulp(x):
    """Spacing of the bf16 grid at |x| (8 significant bits); 2^-133 below the normal range."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def errors(out_gpu, lse_gpu, out_ref, lse_ref):
    """out_gpu / lse_gpu: numpy arrays already gathered to the reference's shape."""
    o = np.asarray(out_gpu, dtype=np.float64)
    r = np.asarray(out_ref, dtype=np.float64)
    d = o - r
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    # worst error as a multiple of the per-element bound max(MAX_ABS, ulp)
    bound_ratio = float(np.max(np.abs(d) / np.maximum(MAX_ABS, bf16_ulp(r)))) if d.size else 0.0
    den = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))
    lse_abs = float(np.max(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref))) if np.size(lse_ref) else 0.0
    finite = bool(np.all(np.isfinite(o)) and np.all(np.isfinite(lse_gpu)))
    return dict(max_abs=max_abs, bound_ratio=bound_ratio, rel_fro=rel, lse_abs=lse_abs, finite=finite)


def check(errs, rel_fro=REL_FRO, lse_abs=LSE_ABS):
    assert errs["finite"], errs
    assert errs["bound_ratio"] <= 1.0, errs  # |out - oracle| <= max(1.5e-2, bf16 ulp) everywhere
    assert errs["rel_fro"] <= rel_fro, errs
    assert errs["lse_abs"] <= lse_abs, errs


def gather_rows(out, lse, tok, head):
    """Rows (token, head) of device tensors out [T, H, d] and lse [T, H] as fp64 numpy."""
    import torch
    t = torch.as_tensor(tok, dtype=torch.long, device=out.device)
    h = torch.as_tensor(head, dtype=torch.long, device=out.device)
    return (out[t, h].double().cpu().numpy(), lse[t, h].double().cpu().numpy())


# ---- gradients (pa_varlen_attn_bwd) against the fp64 gradient oracle
#
# No tolerance is given for the gradients; this one follows from the arithmetic.
# With u = 2^-9 (bf16 unit roundoff): P and dS are rounded to bf16 before the
# MMAs (one rounding per product term, u relative), D = dout . out uses the
# forward's bf16-rounded out (u relative in each term), the partial sums run in
# fp32, and each gradient is rounded to bf16 once (u).  The rounding errors of
# the terms are independent, so in the Frobenius norm they add to a few u:
# relative Frobenius error <= 1e-2 (about 5u).  Element-wise, a gradient can be
# a small difference of larger terms, so the bound is taken relative to the
# tensor's largest magnitude: |err| <= 2e-2 * max|ref| (about 10u).
BWD_REL_FRO = 1e-2
BWD_MAX_REL = 2e-2


def bwd_errors(got, ref):
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    d = g - r
    scale = float(np.max(np.abs(r))) if r.size else 0.0
    den = float(np.linalg.norm(r))
    return dict(max_abs=float(np.max(np.abs(d))) if d.size else 0.0, ref_max=scale,
                rel_fro=float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d)),
                finite=bool(np.all(np.isfinite(g))))


def bwd_check(errs, name=""):
    assert errs["finite"], (name, errs)
    assert errs["rel_fro"] <= BWD_REL_FRO, (name, errs)
    assert errs["max_abs"] <= BWD_MAX_REL * errs["ref_max"] + 1e-30, (name, errs)


# ---- projections (pa_qkv_rope_fwd, pa_linear_fwd) against the fp64 projection oracle
#
# bf16 x bf16 products are exact in fp32 and the fp32 sums over the hidden size add
# errors far below bf16's resolution; the rotation uses fp32 (cos, sin) rounded from
# fp64; the output is rounded to bf16 once (half an ulp: 2^-9 relative).  Bound per
# element: 2^-8 |ref| (twice the rounding) + 1e-4 rms(ref) for outputs near zero;
# relative Frobenius error <= 2e-3.
PROJ_REL = 2.0 ** -8
PROJ_ABS_RMS = 1e-4
PROJ_REL_FRO = 2e-3


def proj_check(got, ref, name=""):
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    d = np.abs(g - r)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    bound = PROJ_REL * np.abs(r) + PROJ_ABS_RMS * rms
    worst = float(np.max(d / np.maximum(bound, 1e-300))) if r.size else 0.0
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-300))
    errs = dict(worst_over_bound=worst, rel_fro=rel, finite=bool(np.all(np.isfinite(g))))
    assert errs["finite"], (name, errs)
    assert worst <= 1.0, (name, errs)
    assert rel <= PROJ_REL_FRO, (name, errs)
    return errs


# ---- FP8 variant (pa_varlen_attn_fwd_fp8) against the fp64 oracle of the
# dequantised operands (oracle/fp8.py)
#
# The kernel differs from that reference by rounding the softmax weights to E4M3
# before the P.V product, P8_j = P_j + d_j, and normalising by sum(P8).  To first order
# out_c - ref_c = sum_j d_j (v_jc - ref_c) / sum(P).  The bound below is taken with
# P_j = 2^(x_j - max x + 4), the kernel's weights at its smallest admissible shift (the
# row maximum at 2^4); a larger shift only scales the weights up, which keeps the
# relative error of normal values and can only move small weights out of the subnormal
# range.  Two terms:
#   * d_j as independent rounding errors, variance <= s_j^2 / 12 with s_j the E4M3
#     spacing at P_j (2^(e-3) on [2^e, 2^(e+1)), 2^-9 below 2^-6): a standard deviation
#     sigma_c = sqrt(sum_j s_j^2 / 12 (v_jc - ref_c)^2) / sum P per element;
#   * in the subnormal range (P_j < 2^-6) rounding is not zero-mean (every weight below
#     2^-10 flushes to zero), so those terms are also bounded deterministically, |d_j| <=
#     min(P_j, 2^-10): b_c = sum_j min(P_j, 2^-10) |v_jc - ref_c| / sum P.  (sigma keeps
#     their variance as well: the sum is conservative.)
# Bound per element: 7 sigma_c + b_c (a false alarm below 1e-11 per element for the
# Gaussian part) plus one bf16 ulp of ref_c for the output's rounding (half an ulp) and
# the fp32 accumulations;
# over all compared elements the relative Frobenius error is bounded by 1.25 times the
# predicted one (sigma and b) plus 2^-9.  lse uses unrounded weights: absolute error
# <= 1e-3 as for the bf16 path.
FP8_SIGMAS = 7.0
FP8_PSHIFT = 4.0
FP8_MIN_NORMAL = 2.0 ** -6
FP8_HALF_MIN_SUB = 2.0 ** -10


def _e4m3_spacing(p):
    e = np.floor(np.log2(np.maximum(p, 2.0 ** -30)))
    return np.where(p < FP8_MIN_NORMAL, 2.0 ** -9, np.exp2(e - 3))


def fp8_sigma(qh, kh, vh, cu, scale, tok, head, ref):
    """(sigma, bias) [n, d] of the FP8 kernel's output error at the rows (tok[i], head[i]):
    the standard deviation of the weights' rounding and the deterministic bound of the
    subnormal weights' rounding (fp64 dequantised operands qh, kh, vh [T, H, d]; ref [n, d] the
    oracle's rows)."""
    cu = np.asarray(cu, dtype=np.int64)
    tok = np.asarray(tok, dtype=np.int64)
    head = np.asarray(head, dtype=np.int64)
    ref = np.asarray(ref, dtype=np.float64)
    seg = np.searchsorted(cu, tok, side="right") - 1
    c = float(scale) / np.log(2.0)
    sig = np.zeros_like(ref)
    bias = np.zeros_like(ref)
    for s, h in {(int(a), int(b)) for a, b in zip(seg, head)}:
        sel = np.nonzero((seg == s) & (head == h))[0]
        b, e = cu[s], cu[s + 1]
        x = (qh[tok[sel], h] @ kh[b:e, h].T) * c                      # [n, L] log2 units
        p = np.exp2(x - x.max(axis=1, keepdims=True) + FP8_PSHIFT)
        sub = p < FP8_MIN_NORMAL
        var = _e4m3_spacing(p) ** 2 / 12.0
        v = vh[b:e, h]                                                # [L, d]
        o = ref[sel]
        acc = var @ (v * v) - 2.0 * o * (var @ v) + o * o * var.sum(axis=1, keepdims=True)
        tot = p.sum(axis=1, keepdims=True)
        sig[sel] = np.sqrt(np.maximum(acc, 0.0)) / tot
        w = np.where(sub, np.minimum(p, FP8_HALF_MIN_SUB), 0.0)       # [n, L]
        for r in range(len(sel)):
            nz = np.nonzero(w[r])[0]
            if nz.size:
                bias[sel[r]] = (w[r, nz] @ np.abs(v[nz] - o[r])) / tot[r, 0]
    return sig, bias


def fp8_check(out_gpu, lse_gpu, out_ref, lse_ref, sigma, bias, name=""):
    g = np.asarray(out_gpu, dtype=np.float64)
    r = np.asarray(out_ref, dtype=np.float64)
    d = np.abs(g - r)
    bound = FP8_SIGMAS * sigma + bias + bf16_ulp(r) + 1e-6
    worst = float(np.max(d / bound)) if r.size else 0.0
    den = max(float(np.linalg.norm(r)), 1e-300)
    rel = float(np.linalg.norm(g - r) / den)
    rel_pred = float((np.linalg.norm(sigma) + np.linalg.norm(bias)) / den)
    lse_abs = float(np.max(np.abs(np.asarray(lse_gpu, np.float64) - lse_ref))) if np.size(lse_ref) else 0.0
    errs = dict(worst_over_bound=worst, rel_fro=rel, rel_fro_predicted=rel_pred, max_abs=float(d.max()),
                lse_abs=lse_abs, finite=bool(np.all(np.isfinite(g)) and np.all(np.isfinite(lse_gpu))))
    assert errs["finite"], (name, errs)
    assert worst <= 1.0, (name, errs)
    assert rel <= 1.25 * rel_pred + 2.0 ** -9, (name, errs)
    assert lse_abs <= LSE_ABS, (name, errs)
    return errs
