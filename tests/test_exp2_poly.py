"""The FMA-pipe exp2 of the attention kernel (CPU emulation of its fp32 steps)."""
import re

import numpy as np

from dit_resolution_packed_b200.csrc import fit_exp2_poly as fit


def _header_constants():
    text = open(fit.HEADER).read()
    return [np.float32(float(v)) for v in re.findall(r"kExp2C\d = ([-0-9.e]+)f;", text)]


def test_header_matches_a_fresh_fit():
    assert _header_constants() == fit.coefficients()


def test_polynomial_relative_error_bound():
    assert fit.fp32_max_rel_error(_header_constants()) < 1e-4


def _emulated_exp2(x):
    """The kernel's sequence in fp32: clamp, magic-add rounding, Horner fma, exponent add."""
    c0, c1, c2, c3 = _header_constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    fma = lambda a, b, c: (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)
    p = fma(np.full_like(f, c3), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))) & np.uint64(0xFFFFFFFF)
    return bits.astype(np.uint32).view(np.float32)


def test_emulated_exp2_against_exp2_over_the_kernel_range():
    x = np.concatenate([np.linspace(-125.0, 8.5, 2000001), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 9) + 0.5, np.arange(-124, 9) - 0.5]).astype(np.float32)
    got = _emulated_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got / ref - 1.0)) < 1e-4


def test_clamp_keeps_tiny_inputs_tiny():
    got = _emulated_exp2(np.array([-126.0, -200.0, -1e30, -np.inf], dtype=np.float32)).astype(np.float64)
    assert np.all(got > 0) and np.all(got < 2.0 ** -124)
