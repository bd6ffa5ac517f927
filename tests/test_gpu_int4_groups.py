"""GPU parity of INT4 with coarser scale groups (256, 512 elements; "Depth
Registers..." thelatestinai page, para 2: APEX4's rho-aware granularity): codes
and scales bit-exact against the oracle's grouped rule (with and without the
block-local rotation), the grouped GEMM (several 128-element MMA stages
accumulated per rescale) within 1 bf16 ulp + 1e-5 * sum|a w| of the oracle."""
import numpy as np
import pytest

from tests import helpers as H
from w4a4_quantized_gemm_token_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_quantized_gemm_token_b200 as w4  # noqa: E402


def dev(bits):
    return H.to_dev_bf16(bits)


def _scales(q, rows, cols, G):
    ld = H.pad128(rows)
    buf = q.scales.cpu().numpy().view(np.float32)[: (cols // G) * ld].reshape(cols // G, ld)
    return buf[:, :rows].T


def _check(q, ref, rows, cols, G):
    np.testing.assert_array_equal(q.codes.cpu().numpy()[: rows * cols // 2].reshape(rows, cols // 2), ref[0])
    np.testing.assert_array_equal(_scales(q, rows, cols, G).view(np.uint32), ref[1].view(np.uint32))


@pytest.mark.parametrize("M,K", [(1, 512), (130, 1024), (300, 3584), (17, 18944)])
@pytest.mark.parametrize("G", [256, 512])
def test_grouped_quant_bitexact(orc, M, K, G):
    X = synth.activations("qwen25_7b_int4", M, K, seed=81)
    q = w4.quantize_act(dev(X), w4.INT4, 0, group=G)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _check(q, orc.quant_int4_g(X, G), M, K, G)
    Wb = synth.weights("qwen25_7b_int4", 256, K, seed=81)
    qw = w4.quantize_weight(dev(Wb), w4.INT4, group=G)
    torch.cuda.synchronize()
    _check(qw, orc.quant_int4_g(Wb, G), 256, K, G)


@pytest.mark.parametrize("G", [256, 512])
def test_grouped_quant_rotated_and_special(orc, G):
    """Zero groups, one outlier, wide exponent spread; and the rotated form
    (128-element rotation blocks inside G-element scale groups)."""
    K = 1024
    r = np.random.default_rng(82)
    rows = [np.zeros(K), np.where(np.arange(K) == 300, -40.0, 0.02), np.linspace(-9, 9, K),
            synth.normal((1, K), 1.0, 82, 1)[0] * np.exp2(r.integers(-12, 13, size=K))]
    X = synth.f32_to_bf16_bits(np.array(rows, np.float32))
    q = w4.quantize_act(dev(X), w4.INT4, 0, group=G)
    qr = w4.quantize_act(dev(X), w4.INT4, 0, group=G, hadamard=True)
    torch.cuda.synchronize()
    _check(q, orc.quant_int4_g(X, G), len(rows), K, G)
    _check(qr, orc.quant_int4_f32_g(orc.rotate_blocks(X, 128, act_side=True), G), len(rows), K, G)


@pytest.mark.parametrize("M", [1, 100, 300])
@pytest.mark.parametrize("G", [256, 512])
def test_grouped_linear_parity(orc, M, G):
    N, K = 384, 3584
    Xa = synth.activations("qwen25_7b_int4", M, K, seed=83)
    Xw = synth.weights("qwen25_7b_int4", N, K, seed=83)
    Wq = w4.quantize_weight(dev(Xw), w4.INT4, group=G)
    Y = w4.linear(dev(Xa), Wq, 0)
    Yg = w4.gemm(w4.quantize_act(dev(Xa), w4.INT4, 0, group=G), Wq)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    ca, sa = orc.quant_int4_g(Xa, G)
    cw, sw = orc.quant_int4_g(Xw, G)
    _, yref, absd = orc.gemm_int4_g(ca, sa, cw, sw, G)
    for name, out in (("linear", Y), ("gemm", Yg)):
        bad = H.gemm_violations(H.to_np_u16(out), yref, absd)
        assert not bad.any(), f"{name}: {bad.sum()} of {bad.size} outside tolerance"


def test_grouped_rotated_linear_parity(orc):
    M, N, K, G = 200, 256, 2048, 512
    Xa = synth.activations("qwen25_7b_int4", M, K, seed=84)
    Xw = synth.weights("qwen25_7b_int4", N, K, seed=84)
    Wq = w4.quantize_weight(dev(Xw), w4.INT4, group=G, hadamard=True)
    Y = w4.linear(dev(Xa), Wq, 0)
    torch.cuda.synchronize()
    ca, sa = orc.quant_int4_f32_g(orc.rotate_blocks(Xa, 128, act_side=True), G)
    cw, sw = orc.quant_int4_f32_g(orc.rotate_blocks(Xw, 128, act_side=False), G)
    _, yref, absd = orc.gemm_int4_g(ca, sa, cw, sw, G)
    bad = H.gemm_violations(H.to_np_u16(Y), yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"


def test_grouped_sampled_at_qwen_w2_size(orc):
    """Qwen2.5-7B w2 (18944 -> 3584) at 2048 tokens with groups of 512: the
    activation quantization in full, the product on sampled rows."""
    M, N, K, G = 2048, 3584, 18944, 512
    Xa = synth.activations("qwen25_7b_int4", M, K, seed=0)
    Xw = synth.weights("qwen25_7b_int4", N, K, seed=0)
    Wq = w4.quantize_weight(dev(Xw), w4.INT4, group=G)
    q = w4.quantize_act(dev(Xa), w4.INT4, 0, group=G)
    Y = w4.linear(dev(Xa), Wq, 0)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    ca, sa = orc.quant_int4_g(Xa, G)
    _check(q, (ca, sa), M, K, G)
    pick = np.array([0, 1, 127, 128, 1023, 2047])
    cw, sw = orc.quant_int4_g(Xw, G)
    _, yref, absd = orc.gemm_int4_g(ca[pick], sa[pick], cw, sw, G)
    bad = H.gemm_violations(H.to_np_u16(Y)[pick], yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"
