"""Fits the polynomial used by the FMA-pipe exp2 of the attention kernel and
writes ``exp2_poly.cuh``.

Method: Cody-Waite style range reduction of exp2 (x = n + f, n = round(x),
|f| <= 1/2, 2^x = 2^n * 2^f) and a degree-3 polynomial p(f) ~ 2^f that
minimises the maximum *relative* error on [-1/2, 1/2], found with the Remez
exchange algorithm (equioscillation of the weighted error at deg + 2 points).
The coefficients are rounded to fp32; ``fp32_max_rel_error`` evaluates the
rounded polynomial in fp32 arithmetic (Horner with fused multiply-adds, as the
kernel does) against the fp64 exp2.

    python -m dit_resolution_packed_b200.csrc.fit_exp2_poly     # rewrites exp2_poly.cuh
"""
import os

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5
HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(HERE, "exp2_poly.cuh")


def _target(x):
    return np.exp2(x)


def remez(degree=DEGREE, lo=LO, hi=HI, iters=30, grid=200001):
    """Coefficients c[0..degree] (ascending powers) minimising max |p(x)/2^x - 1| on [lo, hi]."""
    n = degree + 2
    # initial reference: Chebyshev extrema mapped to [lo, hi]
    k = np.arange(n)
    ref = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * k / (n - 1))[::-1]
    xs = np.linspace(lo, hi, grid)
    c = None
    for _ in range(iters):
        # p(x_i) - g(x_i) = (-1)^i E g(x_i)  ->  sum_j c_j x_i^j - (-1)^i E g(x_i) = g(x_i)
        g = _target(ref)
        A = np.zeros((n, n))
        for j in range(degree + 1):
            A[:, j] = ref ** j
        A[:, degree + 1] = -((-1.0) ** np.arange(n)) * g
        sol = np.linalg.solve(A, g)
        c, E = sol[:degree + 1], sol[degree + 1]
        err = np.polyval(c[::-1], xs) / _target(xs) - 1.0
        # new reference: one extremum of the error per sign-alternating segment
        sign = np.sign(err)
        breaks = np.nonzero(np.diff(sign) != 0)[0] + 1
        segments = np.split(np.arange(grid), breaks)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segments if len(seg)]
        if len(ext) < n:
            break
        # keep the n consecutive extrema with the largest minimum |error|
        best, best_val = None, -1.0
        for s in range(len(ext) - n + 1):
            cand = ext[s:s + n]
            val = np.min(np.abs(err[cand]))
            if val > best_val:
                best, best_val = cand, val
        new_ref = xs[best]
        if np.allclose(new_ref, ref, atol=1e-12, rtol=0):
            break
        ref = new_ref
    return c


def fp32_max_rel_error(c32, samples=400001):
    """Max relative error of p(f) evaluated in fp32 (Horner, fused multiply-add) on [-1/2, 1/2]."""
    f = np.linspace(LO, HI, samples).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for cj in c32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(cj)).astype(np.float32)  # one rounding per fma
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def coefficients():
    c = remez()
    return [np.float32(x) for x in c]


def write_header(path=HEADER):
    c32 = coefficients()
    err = fp32_max_rel_error(c32)
    lines = [
        "// exp2_poly.cuh -- written by fit_exp2_poly.py; do not edit by hand.",
        "//",
        "// 2^f ~ C0 + f*(C1 + f*(C2 + f*C3)) on |f| <= 1/2: degree-3 minimax fit of the",
        "// relative error (Remez exchange), coefficients rounded to fp32.",
        f"// Max relative error of the fp32 evaluation (fused multiply-adds): {err:.3e}.",
        "#pragma once",
        "",
        "namespace pa {",
    ]
    for i, v in enumerate(c32):
        lines.append(f"constexpr float kExp2C{i} = {float(v)!r}f;")
    lines.append(f"constexpr float kExp2PolyMaxRelErr = {err:.6e}f;")
    lines.append("}  // namespace pa")
    with open(path, "w") as fh:
        fh.write("\n".join(lines) + "\n")
    return c32, err


if __name__ == "__main__":
    c32, err = write_header()
    print("coefficients", [float(x) for x in c32], "max rel err", err)
