"""Pins of the FP8 oracle (oracle/fp8.py) against things other than itself: the E4M3
format's definition as PyTorch's float8_e4m3fn implements it, closed forms of the
quantiser, and exactly representable inputs for which the FP8 attention must equal the
plain fp64 oracle.

Each check takes the oracle module as its argument, so that tests/test_oracle_fp8_mutants.py
can run the same checks on copies of the oracle with planted mistakes."""
import numpy as np
import torch

import oracle
import workloads


def _torch_e4m3(x32):
    return torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(torch.float8_e4m3fn).float().numpy()


def check_decode_table_matches_torch(fp8):
    codes = np.arange(256, dtype=np.uint8)
    ours = fp8.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.sum(np.isnan(ours)) == 2
    assert fp8.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert fp8.e4m3_decode(np.array([0x38]))[0] == 1.0
    assert fp8.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert fp8.e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6


def check_encode_roundtrips_every_finite_code(fp8):
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = fp8.e4m3_decode(codes).astype(np.float32)
    got = fp8.e4m3_encode(vals)
    # +0 and -0 are distinct codes and both round-trip
    assert np.array_equal(got, codes)
    assert np.array_equal(fp8.e4m3_round(vals), vals.astype(np.float64))


def check_rounding_matches_torch_in_range(fp8):
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000) * 50,
        rng.standard_normal(20000) * 2.0 ** -7,               # subnormal range
        rng.uniform(-448, 448, 20000),
    ]).astype(np.float32)
    # exact ties: midpoints between neighbouring finite values of one sign
    vals = np.unique(fp8.e4m3_decode(np.arange(0x00, 0x7F, dtype=np.uint8)))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids]).astype(np.float32)
    assert np.array_equal(fp8.e4m3_round(x), _torch_e4m3(x).astype(np.float64))


def check_ties_go_to_even_mantissa_and_saturate(fp8):
    r = fp8.e4m3_round(np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, 464.0, 470.0, 1e9, -1e9],
                                dtype=np.float32))
    assert list(r) == [1.0, 1.25, 0.0, 2.0 ** -8, 448.0, 448.0, 448.0, -448.0]


def check_quant_params_closed_forms(fp8):
    mult, s = fp8.quant_params(np.array([448.0, 1.0, 0.0, 3.5], dtype=np.float32))
    assert list(mult) == [1.0, np.float32(448.0), 1.0, np.float32(128.0)]
    assert list(s) == [1.0, np.float32(1.0) / np.float32(448.0), 1.0, np.float32(3.5) / np.float32(448.0)]


def check_quantizer_axes_and_error_bound(fp8):
    q, k, v, _ = workloads.random_qkv(300, 3, 16, seed=5)
    v = v * torch.linspace(0.25, 4.0, 16).to(torch.bfloat16)       # channels of different ranges
    qz = fp8.quantize_qkv(q, k, v)
    qf, vf = q.float().numpy(), v.float().numpy()
    # the absolute maximum of each quantised group lands on +-448
    assert np.max(np.abs(fp8.e4m3_decode(qz["q8"]))) == 448.0
    per_ch = np.max(np.abs(fp8.e4m3_decode(qz["v8"])), axis=0)
    assert np.all(per_ch == 448.0)
    assert qz["s_v"].shape == (3, 16)
    assert np.array_equal(qz["s_v"], fp8.quant_params(np.max(np.abs(vf), axis=0))[1])
    # relative error of E4M3 round-to-nearest: at most 2^-4 for normal values
    qh = fp8.dequantize(qz["q8"], qz["s_q"])
    scaled = np.abs(qf) * float(fp8.quant_params(np.max(np.abs(qf)))[0])
    nrm = scaled >= 2.0 ** -6
    rel = np.abs(qh - qf)[nrm] / np.abs(qf)[nrm]
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)
    sub = ~nrm & (qf != 0)
    assert np.all(np.abs(qh - qf)[sub] <= 2.0 ** -10 * float(qz["s_q"]) * (1 + 1e-6))


def check_zero_tensor(fp8):
    z = torch.zeros(8, 2, 16, dtype=torch.bfloat16)
    qz = fp8.quantize_qkv(z, z, z)
    assert not qz["q8"].any() and qz["s_q"] == 1.0 and np.all(qz["s_v"] == 1.0)


def check_maxima_match_torch(fp8):
    q, k, v, _ = workloads.random_qkv(200, 3, 16, seed=8)
    aq, ak, av = fp8.qkv_amax(q, k, v)
    assert aq == q.float().abs().max().item() and ak == k.float().abs().max().item()
    assert np.array_equal(av, v.float().abs().amax(dim=0).numpy())


def check_given_maxima_against_torch(fp8):
    """Delayed scaling: with maxima above the data's, each code is PyTorch's E4M3 of the fp32
    product x * (448 / a); with maxima below it, what lies above a saturates to +-448 (codes
    0x7E / 0xFE) and the rest is PyTorch's E4M3 of the product."""
    q, k, v, _ = workloads.random_qkv(200, 3, 16, seed=9)
    aq, ak, av = fp8.qkv_amax(q, k, v)
    for f in (2.0, 0.5):
        gq, gk, gv = np.float32(aq * f), np.float32(ak * f), (av * np.float32(f)).astype(np.float32)
        qz = fp8.quantize_qkv_with(q, k, v, gq, gk, gv)
        for x, g, codes in ((q, gq, qz["q8"]), (k, gk, qz["k8"]), (v, gv[None, :, :], qz["v8"])):
            xf = x.float().numpy()
            mult = (np.float32(448.0) / np.asarray(g, dtype=np.float32)).astype(np.float32)
            prod = (xf * mult).astype(np.float32)
            over = np.abs(prod) > 448.0
            assert over.any() == (f < 1.0)
            dec = fp8.e4m3_decode(codes)
            assert np.all(dec[over] == np.sign(prod[over]) * 448.0)
            assert np.array_equal(dec[~over], _torch_e4m3(prod[~over]).astype(np.float64))
        assert qz["s_q"] == np.float32(gq) / np.float32(448.0)
        assert np.array_equal(qz["s_v"], (gv / np.float32(448.0)).astype(np.float32))


def _representable(fp8, rng, shape, top):
    """Random E4M3 values times `top` / 448 (a power of two), with the top value present."""
    codes = rng.integers(0, 0x7E, size=shape).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=shape).astype(np.uint8) << 7)
    vals = fp8.e4m3_decode(codes)
    vals.reshape(-1)[0] = 448.0
    return vals * (top / 448.0)


def check_exact_operands_give_plain_attention(fp8):
    """With operands already on the grid (amax a power of two times 448, per channel for v),
    dequantisation is exact and the FP8 attention is the plain fp64 attention."""
    rng = np.random.default_rng(3)
    T, H, d = 90, 2, 8
    cu = np.array([0, 40, 41, 90])
    q = _representable(fp8, rng, (T, H, d), 448.0)
    k = _representable(fp8, rng, (T, H, d), 448.0 * 2.0 ** -7)
    v = np.empty((T, H, d))
    for h in range(H):
        for c in range(d):
            col = _representable(fp8, rng, (T,), 448.0 * 2.0 ** (c % 5 - 2))
            v[:, h, c] = col
    out8, lse8, qz = fp8.varlen_attention_fp8(q.astype(np.float32), k.astype(np.float32), v.astype(np.float32),
                                              cu, 0.05)
    out, lse = oracle.varlen_attention(q, k, v, cu, 0.05)
    np.testing.assert_array_equal(out8, out)
    np.testing.assert_array_equal(lse8, lse)
    # a per-tensor scale for v would have lost these channels' low bits
    vz = fp8.quantize(v.astype(np.float32), np.float32(np.max(np.abs(v))))
    assert not np.array_equal(fp8.e4m3_decode(vz) * (np.max(np.abs(v)) / 448.0), v)


ALL_CHECKS = [check_decode_table_matches_torch, check_encode_roundtrips_every_finite_code, check_rounding_matches_torch_in_range, check_ties_go_to_even_mantissa_and_saturate, check_quant_params_closed_forms, check_quantizer_axes_and_error_bound, check_zero_tensor, check_exact_operands_give_plain_attention, check_maxima_match_torch, check_given_maxima_against_torch]
