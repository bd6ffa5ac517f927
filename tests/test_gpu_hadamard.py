"""GPU parity of the block-local Walsh-Hadamard rotation (each 16 / 32 / 128
block along K rotated before quantization; activation side times 1/n, weight
side unscaled, so the GEMM is unchanged).  Codes and scales bit-exact against
the oracle's FP32 butterflies followed by its FP32-input quantizers; products
on every GEMM kernel (CTA pair for M > 128, one CTA for M <= 128, split-K
decode for M <= 16; INT4 kernel) within 1 bf16 ulp + 1e-5 * sum|a w|; the
rotation cancels in the product."""
import numpy as np
import pytest

from tests import helpers as H
from w4a4_quantized_gemm_token_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_quantized_gemm_token_b200 as w4  # noqa: E402

BLOCK = {w4.NVFP4: 16, w4.MXFP4: 32, w4.INT4: 128}


def dev(bits):
    return H.to_dev_bf16(bits)


def _oracle_quant(orc, Xb, fmt, mode, act_side):
    xr = orc.rotate_blocks(Xb, BLOCK[fmt], act_side=act_side)
    if fmt == w4.NVFP4:
        return orc.quant_nvfp4_f32(xr, mode)
    if fmt == w4.MXFP4:
        return orc.quant_mxfp4_f32(xr)
    return orc.quant_int4_f32(xr)


def _compare(q, ref, fmt, M, K):
    codes = q.codes.cpu().numpy()[: M * K // 2].reshape(M, K // 2)
    np.testing.assert_array_equal(codes, ref[0])
    if fmt == w4.INT4:
        sc = H.int4_scales(q.scales.cpu().numpy().view(np.float32), M, K)
        np.testing.assert_array_equal(sc.view(np.uint32), ref[1].view(np.uint32))
    else:
        g = BLOCK[fmt]
        np.testing.assert_array_equal(H.unswizzle_scales(q.scales.cpu().numpy(), M, K, g), ref[1])
        assert np.all(H.padding_scales(q.scales.cpu().numpy(), M, K, g) == 0)
    if fmt == w4.NVFP4:
        np.testing.assert_array_equal(q.s2.cpu().numpy()[: len(ref[2])], ref[2])


CASES = [(w4.NVFP4, w4.SCALE_TOKEN), (w4.NVFP4, w4.SCALE_TENSOR), (w4.MXFP4, 0), (w4.INT4, 0)]


@pytest.mark.parametrize("M,K", [(1, 128), (5, 384), (130, 1024), (300, 2816), (17, 8192)])
@pytest.mark.parametrize("fmt,mode", CASES)
def test_rotated_activation_quant_bitexact(orc, M, K, fmt, mode):
    X = synth.activations("qwen25_7b_int4" if fmt == w4.INT4 else "llama2_70b", M, K, seed=41)
    q = w4.quantize_act(dev(X), fmt, mode if fmt == w4.NVFP4 else w4.SCALE_TENSOR, hadamard=True)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _compare(q, _oracle_quant(orc, X, fmt, mode, True), fmt, M, K)


@pytest.mark.parametrize("fmt", [w4.NVFP4, w4.MXFP4, w4.INT4])
def test_rotated_weight_quant_bitexact(orc, fmt):
    N, K = 384, 1280
    Wb = synth.weights("llama2_70b", N, K, seed=42)
    q = w4.quantize_weight(dev(Wb), fmt, hadamard=True)
    torch.cuda.synchronize()
    _compare(q, _oracle_quant(orc, Wb, fmt, 0, False), fmt, N, K)


def test_rotated_special_values(orc):
    """Zero and negative-zero blocks, one outlier per block, values spanning a
    wide exponent range (the butterflies round), bf16 extremes."""
    K = 256
    r = np.random.default_rng(43)
    rows = [np.zeros(K), -np.zeros(K), np.where(np.arange(K) % 16 == 3, 50.0, 0.01),
            synth.normal((1, K), 1.0, 43, 1)[0] * np.exp2(r.integers(-14, 15, size=K)),
            np.r_[[3e38], np.zeros(K - 1)], np.linspace(-7, 7, K)]
    X = synth.f32_to_bf16_bits(np.array(rows, np.float32))
    for fmt, mode in CASES:
        q = w4.quantize_act(dev(X), fmt, mode if fmt == w4.NVFP4 else w4.SCALE_TENSOR, hadamard=True)
        torch.cuda.synchronize()
        _compare(q, _oracle_quant(orc, X, fmt, mode, True), fmt, len(rows), K)


def _gemm_ref(orc, fmt, Xa, Xw, mode):
    if fmt == w4.NVFP4:
        ca, sa, s2a = _oracle_quant(orc, Xa, fmt, mode, True)
        cw, sw, s2w = _oracle_quant(orc, Xw, fmt, 0, False)
        return orc.gemm_nvfp4(ca, sa, s2a, mode, cw, sw, s2w)
    ca, sa = _oracle_quant(orc, Xa, fmt, 0, True)
    cw, sw = _oracle_quant(orc, Xw, fmt, 0, False)
    return (orc.gemm_mxfp4 if fmt == w4.MXFP4 else orc.gemm_int4)(ca, sa, cw, sw)


# M = 1, 16: split-K decode; 100: one-CTA kernel; 300: CTA pair (INT4: its own kernel)
@pytest.mark.parametrize("M", [1, 16, 100, 300])
@pytest.mark.parametrize("fmt,mode", CASES)
def test_rotated_linear_parity(orc, M, fmt, mode):
    N, K = 384, 1280
    Xa = synth.activations("llama2_70b", M, K, seed=44)
    Xw = synth.weights("llama2_70b", N, K, seed=44)
    Wq = w4.quantize_weight(dev(Xw), fmt, hadamard=True)
    Y = w4.linear(dev(Xa), Wq, mode)
    Yg = w4.gemm(w4.quantize_act(dev(Xa), fmt, mode if fmt == w4.NVFP4 else w4.SCALE_TENSOR, hadamard=True), Wq)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _, yref, absd = _gemm_ref(orc, fmt, Xa, Xw, mode)
    for name, out in (("linear", Y), ("gemm", Yg)):
        bad = H.gemm_violations(H.to_np_u16(out), yref, absd)
        assert not bad.any(), f"{name}: {bad.sum()} of {bad.size} outside tolerance"


@pytest.mark.parametrize("fmt", [w4.NVFP4, w4.MXFP4, w4.INT4])
def test_rotation_cancels_in_the_product(fmt):
    """Rotated activations times rotated weights approximate X W^T as well as
    the unrotated product does (the rotation itself cancels: H H^T = n I)."""
    M, N, K = 64, 256, 2048
    Xa = synth.activations("qwen25_7b_int4", M, K, seed=45)
    Xw = synth.weights("qwen25_7b_int4", N, K, seed=45)
    exact = synth.bf16_bits_to_f32(Xa).astype(np.float64) @ synth.bf16_bits_to_f32(Xw).astype(np.float64).T
    mode = w4.SCALE_TOKEN if fmt == w4.NVFP4 else 0
    errs = []
    for rot in (False, True):
        Wq = w4.quantize_weight(dev(Xw), fmt, hadamard=rot)
        Y = H.bf16_to_f64(H.to_np_u16(w4.linear(dev(Xa), Wq, mode)))
        errs.append(np.abs(Y - exact).mean() / np.abs(exact).mean())
    assert errs[1] < 1.5 * errs[0] and errs[1] < 0.3, errs


def test_rotated_segments_bitexact(orc):
    """Per-segment NVFP4 weights with rotation: each segment is the rotated
    tensor rule on its rows."""
    K = 1024
    Wb, seg = synth.fused_weights((256, 128, 128), (1.0, 4.0, 0.25), K, seed=46)
    N = seg[-1]
    q = w4.quantize_weight_segments(dev(Wb), seg, hadamard=True)
    torch.cuda.synchronize()
    xr = orc.rotate_blocks(Wb, 16, act_side=False)
    codes = q.codes.cpu().numpy()[: N * K // 2].reshape(N, K // 2)
    sc = H.unswizzle_scales(q.scales.cpu().numpy(), N, K, 16)
    s2 = q.s2.cpu().numpy()[:N]
    for i in range(3):
        r0, r1 = seg[i], seg[i + 1]
        oc, osc, os2 = orc.quant_nvfp4_f32(xr[r0:r1], 0)
        np.testing.assert_array_equal(codes[r0:r1], oc)
        np.testing.assert_array_equal(sc[r0:r1], osc)
        assert np.all(s2[r0:r1] == os2[0])


def test_rotated_sampled_at_llama_qkv_size(orc):
    """Llama-2-70B qkv (8192 -> 10240) at 4096 tokens, NVFP4 per token, rotated:
    the activation quantization compared in full, the product on sampled rows."""
    M, N, K = 4096, 10240, 8192
    Xa = synth.activations("llama2_70b", M, K, seed=0)
    Xw = synth.weights("llama2_70b", N, K, seed=0)
    Wq = w4.quantize_weight(dev(Xw), w4.NVFP4, hadamard=True)
    q = w4.quantize_act(dev(Xa), w4.NVFP4, w4.SCALE_TOKEN, hadamard=True)
    Y = w4.linear(dev(Xa), Wq, w4.SCALE_TOKEN)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    ref = _oracle_quant(orc, Xa, w4.NVFP4, 1, True)
    _compare(q, ref, w4.NVFP4, M, K)
    pick = np.array([0, 1, 255, 256, 2047, 4095])
    cw, sw, s2w = _oracle_quant(orc, Xw, w4.NVFP4, 0, False)
    _, yref, absd = orc.gemm_nvfp4(ref[0][pick], ref[1][pick], ref[2][pick], 1, cw, sw, s2w)
    bad = H.gemm_violations(H.to_np_u16(Y)[pick], yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"
