"""Oracle of the FP8 (E4M3) variant of the packed attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and by the CPU legs of ``bench.py``;
never by the product package.  It shares no code with the CUDA path.

What the variant computes (FPS Attention slides of the Mage-Flow talk, "QK granularity"
and "V per channel, P per tensor": attention run on FP8 operands, with Q and K quantised
per tensor, V per channel and P per tensor).  Readings, since the slides give no formulas:

* E4M3 is the OCP FP8 format without infinities: 1 sign bit, 4 exponent bits (bias 7),
  3 mantissa bits; the largest finite value is 448 (exponent field 15, mantissa 110;
  mantissa 111 there is NaN); exponent field 0 holds the subnormals k * 2^-9.
* Quantising a tensor x with absolute maximum a (over the whole tensor for q and k, over
  all tokens of one (head, channel) column for v):
      mult = fp32(448 / a),   s = fp32(a / 448)       (both 1 when a == 0)
      code = E4M3(fp32(x * mult))                      round to nearest even, values
                                                       beyond 448 clamp to +-448
      x_hat = s * value(code)                          the dequantised input
  Every step is fp32 arithmetic with one rounding, so the codes are a deterministic
  function of the bf16 inputs.
* The attention of the variant is the exact block-diagonal attention (the fp64 oracle of
  this package) of q_hat, k_hat, v_hat with the caller's scale.  The kernel also rounds
  the softmax weights P to E4M3 (one static power-of-two scale for all of P); that
  rounding is the method's approximation and is left out here: the tests bound its
  effect by a tolerance derived from the E4M3 rounding error.
Pinned by ``tests/test_oracle_fp8_pins.py``.
"""
import numpy as np

from . import varlen_attention

E4M3_MAX = 448.0
_MANT = 3
_BIAS = 7
_MIN_NORMAL_EXP = 1 - _BIAS          # 2^-6
_SUB_QUANTUM = 2.0 ** (_MIN_NORMAL_EXP - _MANT)   # 2^-9


def _f32(x):
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        return x.float().numpy()
    if hasattr(x, "numpy") and not isinstance(x, np.ndarray):
        x = x.numpy()
    return np.asarray(x, dtype=np.float32)


def e4m3_decode(codes):
    """fp64 value of each E4M3 code (uint8), from the field layout; NaN for 0x7F / 0xFF."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> _MANT) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * _SUB_QUANTUM, (1.0 + m / 8.0) * np.exp2(e - _BIAS))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_round(x):
    """Nearest E4M3 value of each fp32 x (ties to even mantissa), clamped to +-448; fp64."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # np.log2 of an exact power of two is exact; guard the floor against a value just
    # below a binade edge all the same
    e = np.where(np.exp2(e) > a, e - 1, e)
    e = np.where(np.exp2(e + 1) <= a, e + 1, e)
    quantum = np.where(a < 2.0 ** _MIN_NORMAL_EXP, _SUB_QUANTUM, np.exp2(e - _MANT))
    r = np.round(a / quantum) * quantum          # x / quantum is exact; np.round is half-to-even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(x):
    """E4M3 code (uint8) of each fp32 x, rounded as ``e4m3_round``."""
    r = e4m3_round(x)
    a = np.abs(r)
    sign = np.signbit(r).astype(np.int64) << 7
    sub = a < 2.0 ** _MIN_NORMAL_EXP
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0))).astype(np.int64)
    m_sub = np.round(a / _SUB_QUANTUM).astype(np.int64)
    m_nrm = np.round((a / np.exp2(e) - 1.0) * 8.0).astype(np.int64)
    code = np.where(sub, m_sub, ((e + _BIAS) << _MANT) | m_nrm)
    return (sign | code).astype(np.uint8)


def quant_params(amax):
    """(mult, s) in fp32 for an absolute maximum (array or scalar)."""
    a = np.asarray(amax, dtype=np.float32)
    zero = a == 0
    safe = np.where(zero, np.float32(1), a).astype(np.float32)
    mult = np.where(zero, np.float32(1), np.float32(E4M3_MAX) / safe).astype(np.float32)
    s = np.where(zero, np.float32(1), safe / np.float32(E4M3_MAX)).astype(np.float32)
    return mult, s


def quantize(x, amax):
    """Codes of x (fp32-valued) with the given amax (broadcast against x)."""
    mult, _ = quant_params(amax)
    prod = (np.asarray(x, dtype=np.float32) * mult).astype(np.float32)   # one fp32 rounding
    flat = prod.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    step = 1 << 22                                   # bounded temporaries on large packs
    for i in range(0, flat.size, step):
        out[i:i + step] = e4m3_encode(flat[i:i + step])
    return out.reshape(prod.shape)


def qkv_amax(q, k, v):
    """(a_q, a_k, a_v): the absolute maxima of the whole q, the whole k and each (head,
    channel) column of v over all tokens (fp32; zero for an empty tensor)."""
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    aq = np.float32(np.max(np.abs(qf))) if qf.size else np.float32(0)
    ak = np.float32(np.max(np.abs(kf))) if kf.size else np.float32(0)
    av = (np.max(np.abs(vf), axis=0) if vf.shape[0] else np.zeros(vf.shape[1:])).astype(np.float32)
    return aq, ak, av


def quantize_qkv_with(q, k, v, aq, ak, av):
    """FP8 operands with the scales of given maxima (a_q, a_k scalars; a_v [H, d]): the
    quantisation of ``quantize_qkv`` with the maxima supplied instead of measured (delayed
    scaling).  An input above its group's maximum rounds to the code of +-448."""
    qf, kf, vf = _f32(q), _f32(k), _f32(v)
    aq, ak = np.float32(aq), np.float32(ak)
    av = np.asarray(av, dtype=np.float32)
    out = {"q8": quantize(qf, aq), "k8": quantize(kf, ak), "v8": quantize(vf, av[None, :, :])}
    out["s_q"] = quant_params(aq)[1]
    out["s_k"] = quant_params(ak)[1]
    out["s_v"] = quant_params(av)[1]
    return out


def quantize_qkv(q, k, v):
    """FP8 operands of the variant.

    q, k, v: [T, H, d] (bf16 tensors or fp32-valued arrays).  Returns a dict with
    q8, k8, v8 (uint8 codes [T, H, d]), s_q, s_k (fp32 scalars) and s_v (fp32 [H, d]).
    """
    return quantize_qkv_with(q, k, v, *qkv_amax(q, k, v))


def dequantize(codes, s):
    """s * value(code) in fp64 (s broadcast against the codes)."""
    return e4m3_decode(codes) * np.asarray(s, dtype=np.float64)


def dequantized_qkv(qz):
    """q_hat, k_hat, v_hat (fp64 [T, H, d]) of a ``quantize_qkv`` result."""
    return (dequantize(qz["q8"], qz["s_q"]), dequantize(qz["k8"], qz["s_k"]),
            dequantize(qz["v8"], qz["s_v"][None, :, :]))


def varlen_attention_fp8(q, k, v, cu_seqlens, scale, rows=None, n_threads=0):
    """(out, lse, qz): the exact attention of the dequantised FP8 operands, and the operands."""
    qz = quantize_qkv(q, k, v)
    qh, kh, vh = dequantized_qkv(qz)
    out, lse = varlen_attention(qh, kh, vh, cu_seqlens, scale, rows=rows, n_threads=n_threads)
    return out, lse, qz
