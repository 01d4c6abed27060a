"""Plants plausible mistakes in copies of the FP8 oracle and requires its pins to catch each.

Every mutant is a textual edit of ``oracle/fp8.py`` loaded as a separate module (CPU only);
the checks of ``tests/oracle_fp8_pins.py`` must fail on every one of them.  (Forming the
product x * mult in fp64 is no mistake: a bf16 value times an fp32 multiplier is exact in fp64,
so rounding it to fp32 gives the fp32 product.)
"""
import importlib.util
import os

import pytest

import oracle
from tests import oracle_fp8_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "fp8.py")

MUTANTS = {
    "round_half_up": ("r = np.round(a / quantum) * quantum", "r = np.floor(a / quantum + 0.5) * quantum"),
    "truncate": ("r = np.round(a / quantum) * quantum", "r = np.floor(a / quantum) * quantum"),
    "no_saturation": ("r = np.minimum(r, E4M3_MAX)", "r = r"),
    "exponent_bias_8": ("_BIAS = 7", "_BIAS = 8"),
    "two_mantissa_bits": ("_MANT = 3", "_MANT = 2"),
    "subnormal_spacing_halved": ("_SUB_QUANTUM = 2.0 ** (_MIN_NORMAL_EXP - _MANT)",
                                 "_SUB_QUANTUM = 2.0 ** (_MIN_NORMAL_EXP - _MANT - 1)"),
    "subnormals_decoded_as_normals": ("mag = np.where(e == 0, m * _SUB_QUANTUM, (1.0 + m / 8.0) * np.exp2(e - _BIAS))",
                                      "mag = (1.0 + m / 8.0) * np.exp2(e - _BIAS)"),
    "v_per_tensor": ("av = (np.max(np.abs(vf), axis=0) if vf.shape[0] else np.zeros(vf.shape[1:])).astype(np.float32)",
                     "av = np.full(vf.shape[1:], np.max(np.abs(vf)) if vf.size else 0, dtype=np.float32)"),
    "mult_and_scale_swapped": ("    mult, _ = quant_params(amax)\n", "    _, mult = quant_params(amax)\n"),
    "q_dequantised_with_k_scale": ('return (dequantize(qz["q8"], qz["s_q"]),', 'return (dequantize(qz["q8"], qz["s_k"]),'),
    "zero_group_scale_zero": ("s = np.where(zero, np.float32(1), safe / np.float32(E4M3_MAX))",
                              "s = np.where(zero, np.float32(0), safe / np.float32(E4M3_MAX))"),
    "scale_inverted": ("s = np.where(zero, np.float32(1), safe / np.float32(E4M3_MAX))",
                       "s = np.where(zero, np.float32(1), np.float32(E4M3_MAX) / safe)"),
}


def _load(name, tmp_path):
    src = open(SRC).read()
    edits = MUTANTS[name] if isinstance(MUTANTS[name], list) else [MUTANTS[name]]
    for old, new in edits:
        assert src.count(old) == 1, f"mutation site of {name} not found exactly once"
        src = src.replace(old, new)
    # the copy lives outside the package: import the fp64 attention oracle absolutely
    src = src.replace("from . import varlen_attention", "from oracle import varlen_attention")
    path = tmp_path / f"fp8_mut_{name}.py"
    path.write_text(src)
    spec = importlib.util.spec_from_file_location(f"fp8_mut_{name}", str(path))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    mod = _load(name, tmp_path)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(mod)
        except (AssertionError, ValueError, FloatingPointError, IndexError):
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"
