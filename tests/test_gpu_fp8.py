"""GPU parity of the FP8 (E4M3) variant through the C ABI: the quantiser bit-exact
against the oracle's codes and scales, and the FP8 attention against the fp64 oracle
of the dequantised operands within the tolerance derived in tests/parity.py."""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
import workloads
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import dit_resolution_packed_b200 as m
    m.load_library()
    return m


def _key0(cu):
    """First key of each segment in the transposed V layout: 16*ceil(cu_s/16) + 16*s."""
    cu = np.asarray(cu, dtype=np.int64)
    s = np.arange(len(cu) - 1)
    return 16 * ((cu[:-1] + 15) // 16) + 16 * s


def _v8_from_vt(v8t, cu, heads, d=128):
    """[T, H, d] codes gathered back from the transposed buffer [H*d, keys]."""
    vt = v8t.cpu().numpy()
    cu = np.asarray(cu, dtype=np.int64)
    T = int(cu[-1])
    out = np.zeros((T, heads * d), dtype=np.uint8)
    for s, k0 in enumerate(_key0(cu)):
        L = int(cu[s + 1] - cu[s])
        out[cu[s]:cu[s + 1]] = vt[:, k0:k0 + L].T
    return out.reshape(T, heads, d)


def _vt_from_v8(v8, cu, keys):
    """The transposed buffer the quantiser would write, built from the oracle's codes."""
    T, H, d = v8.shape
    vt = np.zeros((H * d, keys), dtype=np.uint8)
    cu = np.asarray(cu, dtype=np.int64)
    flat = v8.reshape(T, H * d)
    for s, k0 in enumerate(_key0(cu)):
        L = int(cu[s + 1] - cu[s])
        vt[:, k0:k0 + L] = flat[cu[s]:cu[s + 1]].T
    return vt


def _oracle_operands_on_gpu(pa, qz, cu):
    T, H, d = qz["q8"].shape
    keys = pa.pa_fp8_vt_keys(len(cu) - 1, T)
    scales = np.zeros(4 + H * d, dtype=np.float32)
    scales[0], scales[1] = qz["s_q"], qz["s_k"]
    scales[4:] = qz["s_v"].reshape(-1)
    return dict(q8=torch.from_numpy(qz["q8"]).cuda(), k8=torch.from_numpy(qz["k8"]).cuda(),
                v8t=torch.from_numpy(_vt_from_v8(qz["v8"], cu, keys)).cuda(),
                scales=torch.from_numpy(scales).cuda())


def _run(pa, p, qz_dev=None):
    cu = p["cu_seqlens"].cuda()
    if qz_dev is None:
        qz_dev = pa.fp8_quantize_qkv(p["q"].cuda(), p["k"].cuda(), p["v"].cuda(), cu)
    out, lse = pa.varlen_attn_fwd_fp8(qz_dev, cu, p["max_seqlen"], p["scale"])
    assert pa.pa_get_error() == pa.PA_OK
    return qz_dev, out, lse


def _compare_full(p, out, lse, name, qz=None):
    qz = fp8.quantize_qkv(p["q"], p["k"], p["v"]) if qz is None else qz
    qh, kh, vh = fp8.dequantized_qkv(qz)
    cu = p["cu_seqlens"].numpy()
    ref, rlse = oracle.varlen_attention(qh, kh, vh, cu, p["scale"])
    T, H, _ = ref.shape
    tok = np.repeat(np.arange(T), H)
    head = np.tile(np.arange(H), T)
    sig, bias = parity.fp8_sigma(qh, kh, vh, cu, p["scale"], tok, head, ref.reshape(T * H, -1))
    return parity.fp8_check(out.double().cpu().numpy().reshape(T * H, -1), lse.double().cpu().numpy().reshape(-1),
                            ref.reshape(T * H, -1), rlse.reshape(-1), sig, bias, name)


def _compare_rows(p, out, lse, tok, head, name, qz):
    qh, kh, vh = fp8.dequantized_qkv(qz)
    cu = p["cu_seqlens"].numpy()
    ref, rlse = oracle.varlen_attention(qh, kh, vh, cu, p["scale"], rows=(tok, head))
    sig, bias = parity.fp8_sigma(qh, kh, vh, cu, p["scale"], tok, head, ref)
    go, gl = parity.gather_rows(out, lse, tok, head)
    return parity.fp8_check(go, gl, ref, rlse, sig, bias, name)


def _check_quantiser(pa, p, qz_dev, rows=None, qz=None):
    qz = fp8.quantize_qkv(p["q"], p["k"], p["v"]) if qz is None else qz
    T, H, d = qz["q8"].shape
    sc = qz_dev["scales"].cpu().numpy()
    assert sc[0] == qz["s_q"] and sc[1] == qz["s_k"] and sc[2] == 0 and sc[3] == 0
    assert np.array_equal(sc[4:], qz["s_v"].reshape(-1))
    sel = slice(None) if rows is None else rows
    assert np.array_equal(qz_dev["q8"].cpu().numpy()[sel], qz["q8"][sel])
    assert np.array_equal(qz_dev["k8"].cpu().numpy()[sel], qz["k8"][sel])
    v8 = _v8_from_vt(qz_dev["v8t"], p["cu_seqlens"].numpy(), H)
    assert np.array_equal(v8[sel], qz["v8"][sel])


PACKS = {
    "two_images": ([256, 108], 2),
    "ragged": ([1, 127, 128, 129, 300, 0, 513, 17], 3),
    "one_tile": ([128], 1),
    "odd_starts": ([5, 250, 3, 700, 9], 2),
    "empty_ends": ([0, 0, 300, 0, 129, 0], 2),
    # more segments than the scheduler stages in shared memory (4096)
    "many_segments": ([int(n) for n in np.random.default_rng(5).integers(0, 40, 5000)], 1),
}


@pytest.mark.parametrize("name", sorted(PACKS))
def test_quantiser_bit_exact(pa, name):
    segs, H = PACKS[name]
    p = workloads.random_pack(segs, H, 128, seed=41)
    qz_dev, _, _ = _run(pa, p)
    _check_quantiser(pa, p, qz_dev)


@pytest.mark.parametrize("name", sorted(PACKS))
def test_fp8_attention_on_oracle_operands(pa, name):
    """The attention kernel alone, fed the oracle's codes and scales."""
    segs, H = PACKS[name]
    p = workloads.random_pack(segs, H, 128, seed=43)
    qz = fp8.quantize_qkv(p["q"], p["k"], p["v"])
    _, out, lse = _run(pa, p, _oracle_operands_on_gpu(pa, qz, p["cu_seqlens"].numpy()))
    _compare_full(p, out, lse, name, qz)


@pytest.mark.parametrize("name", sorted(PACKS))
def test_fp8_end_to_end(pa, name):
    segs, H = PACKS[name]
    p = workloads.random_pack(segs, H, 128, seed=47)
    _, out, lse = _run(pa, p)
    _compare_full(p, out, lse, name)


def test_negative_scale(pa):
    p = workloads.random_pack([300, 77], 2, 128, seed=5, scale=-0.09)
    _, out, lse = _run(pa, p)
    _compare_full(p, out, lse, "negative scale")


def test_zero_queries_give_the_mean_of_v(pa):
    """q = 0: every weight is exactly 2^4 in E4M3, so out is the mean of the dequantised
    value rows and lse = ln L."""
    p = workloads.random_pack([200, 1, 333], 2, 128, seed=9)
    p["q"] = torch.zeros_like(p["q"])
    qz_dev, out, lse = _run(pa, p)
    qz = fp8.quantize_qkv(p["q"], p["k"], p["v"])
    vh = fp8.dequantize(qz["v8"], qz["s_v"][None])
    cu = p["cu_seqlens"].numpy()
    o = out.double().cpu().numpy()
    ls = lse.double().cpu().numpy()
    for s in range(len(cu) - 1):
        b, e = cu[s], cu[s + 1]
        mean = vh[b:e].mean(axis=0)
        np.testing.assert_allclose(o[b:e], np.broadcast_to(mean, o[b:e].shape), rtol=2.0 ** -8, atol=1e-6)
        np.testing.assert_allclose(ls[b:e], math.log(e - b), atol=1e-4)  # fp32 log2 of the sum


def test_identical_value_rows_are_reproduced(pa):
    """All value rows of a segment equal: out is that row (convex combination with the
    E4M3 weights the MMA used), whatever q and k."""
    p = workloads.random_pack([384, 129], 2, 128, seed=13)
    cu = p["cu_seqlens"].numpy()
    for s in range(len(cu) - 1):
        p["v"][cu[s]:cu[s + 1]] = p["v"][cu[s]]
    _, out, _ = _run(pa, p)
    qz = fp8.quantize_qkv(p["q"], p["k"], p["v"])
    vh = fp8.dequantize(qz["v8"], qz["s_v"][None])
    o = out.double().cpu().numpy()
    for s in range(len(cu) - 1):
        b, e = cu[s], cu[s + 1]
        np.testing.assert_allclose(o[b:e], np.broadcast_to(vh[b], o[b:e].shape), rtol=2.0 ** -8, atol=1e-6)


def test_rejects_head_dim_64(pa):
    p = workloads.random_pack([64], 1, 64, seed=1)
    with pytest.raises(pa.PackAttnError):
        pa.fp8_quantize_qkv(p["q"].cuda(), p["k"].cuda(), p["v"].cuda(), p["cu_seqlens"].cuda())


def test_bad_cu_seqlens_reported(pa):
    p = workloads.random_pack([100, 100], 1, 128, seed=2)
    qz_dev = pa.fp8_quantize_qkv(p["q"].cuda(), p["k"].cuda(), p["v"].cuda(), p["cu_seqlens"].cuda())
    bad = torch.tensor([0, 150, 120], dtype=torch.int32).cuda()
    pa.varlen_attn_fwd_fp8(qz_dev, bad, 200, 0.1)
    assert pa.pa_get_error() == pa.PA_ERR_CU_SEQLENS
    assert pa.pa_get_error() == pa.PA_OK


@pytest.mark.parametrize("config", ["mixed", "training", "interactive"])
def test_fp8_full_size_sampled(pa, config):
    """The benchmark's launch configuration at full size, checked on sampled rows
    (quantiser codes on a band of tokens)."""
    cfg = workloads.load_config(config)
    p = workloads.make_inputs(cfg)
    qz_dev, out, lse = _run(pa, p)
    qz = fp8.quantize_qkv(p["q"], p["k"], p["v"])
    T = sum(cfg["segments"])
    _check_quantiser(pa, p, qz_dev, rows=slice(max(0, T // 2 - 700), T // 2 + 700), qz=qz)
    tok, head = workloads.sampled_rows(cfg, per_head=48)
    errs = _compare_rows(p, out, lse, tok.numpy(), head.numpy(), config, qz)
    assert errs["rel_fro"] < 0.05


# ---- delayed scaling: scales from given maxima, this call's maxima returned

def _amax_vec(aq, ak, av):
    a = np.zeros(4 + av.size, dtype=np.float32)
    a[0], a[1] = aq, ak
    a[4:] = av.reshape(-1)
    return a


@pytest.mark.parametrize("factor", [2.0, 1.0, 0.5])
@pytest.mark.parametrize("name", ["ragged", "odd_starts", "empty_ends"])
def test_delayed_quantiser_bit_exact(pa, name, factor):
    """Codes and scales from given maxima (above the data's: no saturation; equal: the
    current-scaling result; below: saturation at +-448) match the oracle bit for bit, and the
    returned maxima are the data's exactly."""
    segs, H = PACKS[name]
    p = workloads.random_pack(segs, H, 128, seed=53)
    aq, ak, av = fp8.qkv_amax(p["q"], p["k"], p["v"])
    gq, gk, gv = np.float32(aq * factor), np.float32(ak * factor), (av * np.float32(factor)).astype(np.float32)
    cu = p["cu_seqlens"].cuda()
    qz_dev = pa.fp8_quantize_qkv_delayed(p["q"].cuda(), p["k"].cuda(), p["v"].cuda(), cu,
                                         torch.from_numpy(_amax_vec(gq, gk, gv)).cuda())
    assert pa.pa_get_error() == pa.PA_OK
    qz = fp8.quantize_qkv_with(p["q"], p["k"], p["v"], gq, gk, gv)
    _check_quantiser(pa, p, qz_dev, qz=qz)
    assert np.array_equal(qz_dev["amax"].cpu().numpy(), _amax_vec(aq, ak, av))
    if factor == 1.0:  # the same operands as the current-scaling quantiser
        ref = pa.fp8_quantize_qkv(p["q"].cuda(), p["k"].cuda(), p["v"].cuda(), cu)
        for key in ("q8", "k8", "scales"):
            assert torch.equal(ref[key], qz_dev[key]), key
        # v8t: the segments' keys (the keys between segments are never written)
        cun = p["cu_seqlens"].numpy()
        assert np.array_equal(_v8_from_vt(ref["v8t"], cun, H), _v8_from_vt(qz_dev["v8t"], cun, H))


def test_delayed_quantiser_two_steps_end_to_end(pa):
    """A loop of two steps: step 1 quantises with step 0's maxima (returned by step 0's
    call from all-ones maxima) and the FP8 attention on its operands meets the FP8 bound
    against the oracle of the dequantised operands."""
    segs, H = [300, 129, 17, 700], 2
    p0 = workloads.random_pack(segs, H, 128, seed=61)
    p1 = workloads.random_pack(segs, H, 128, seed=62)
    cu = p0["cu_seqlens"].cuda()
    ones = torch.ones(4 + H * 128, dtype=torch.float32, device="cuda")
    z0 = pa.fp8_quantize_qkv_delayed(p0["q"].cuda(), p0["k"].cuda(), p0["v"].cuda(), cu, ones)
    z1 = pa.fp8_quantize_qkv_delayed(p1["q"].cuda(), p1["k"].cuda(), p1["v"].cuda(), cu, z0["amax"])
    out, lse = pa.varlen_attn_fwd_fp8(z1, cu, p1["max_seqlen"], p1["scale"])
    assert pa.pa_get_error() == pa.PA_OK
    a0 = fp8.qkv_amax(p0["q"], p0["k"], p0["v"])
    assert np.array_equal(z0["amax"].cpu().numpy(), _amax_vec(*a0))
    qz = fp8.quantize_qkv_with(p1["q"], p1["k"], p1["v"], *a0)
    _check_quantiser(pa, p1, z1, qz=qz)
    _compare_full(p1, out, lse, "delayed two steps", qz)


def test_delayed_quantiser_empty_pack_zeroes_amax(pa):
    H = 2
    amax_in = torch.ones(4 + H * 128, dtype=torch.float32, device="cuda")
    amax_out = torch.full((4 + H * 128,), 7.0, dtype=torch.float32, device="cuda")
    e = torch.empty(0, H, 128, dtype=torch.bfloat16, device="cuda")
    e8 = torch.empty(0, H, 128, dtype=torch.uint8, device="cuda")
    cu = torch.zeros(1, dtype=torch.int32, device="cuda")
    vt = torch.empty(H * 128, 0, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(4 + H * 128, dtype=torch.float32, device="cuda")
    rc = pa.pa_fp8_quantize_qkv_delayed(e, e, e, cu, amax_in, amax_out, e8, e8, vt, sc)
    assert rc == pa.PA_OK and pa.pa_get_error() == pa.PA_OK
    assert not amax_out.any()
