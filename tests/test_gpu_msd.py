"""GPU parity of the multi-pass MXFP4 decomposition ("APEX4: Efficient Pure
W4A4 LLM Inference via Intra-SM Compute Rebalancing" page, para 1, MSD):
codes and scales of every pass bit-exact against the oracle; the weight side
[W | W | ...] equal to the oracle's MXFP4 of the repeated matrix; the product
on every GEMM kernel (CTA pair for M > 128, one CTA for M <= 128, split-K
decode for M <= 16) within 1 bf16 ulp + 1e-5 * sum|a w| of the oracle."""
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


def _check_act(orc, Xb, passes):
    M, K = Xb.shape
    q = w4.quantize_act_msd(dev(Xb), passes)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    oc, osc = orc.quant_mxfp4_msd(Xb, passes=passes)
    cols = passes * K
    np.testing.assert_array_equal(q.codes.cpu().numpy()[: M * cols // 2].reshape(M, cols // 2), oc)
    np.testing.assert_array_equal(H.unswizzle_scales(q.scales.cpu().numpy(), M, cols, 32), osc)
    assert np.all(H.padding_scales(q.scales.cpu().numpy(), M, cols, 32) == 0)
    return q


@pytest.mark.parametrize("M,K", [(1, 128), (5, 384), (130, 1024), (300, 2816), (17, 8192)])
@pytest.mark.parametrize("passes", [1, 2, 3])
def test_msd_quant_bitexact(orc, M, K, passes):
    X = synth.activations("swiglu300m" if K == 1024 else "llama2_70b", M, K, seed=31)
    _check_act(orc, X, passes)


def test_msd_quant_special_values(orc):
    """Zero blocks, negative zeros, grid-exact blocks (zero residual), values
    near the bf16 extremes and tiny values inside large blocks."""
    K = 256
    rows = [np.zeros(K), -np.zeros(K), synth.e2m1_grid_values((K,), 3, 1) * 4.0,
            np.linspace(-7, 7, K), np.r_[[3e38], np.full(K - 1, 1e-30)], np.r_[[1e-38], np.full(K - 1, -1e-40)],
            synth.normal((1, K), 1.0, 5, 1)[0] * np.exp2(np.arange(K) % 64 - 32)]
    rows[2][::32] = 24.0
    X = synth.f32_to_bf16_bits(np.array(rows, np.float32))
    for passes in (2, 3):
        _check_act(orc, X, passes)


def test_msd_weights_repeat_the_mxfp4_weights(orc):
    N, K = 384, 1024
    Wb = synth.weights("llama2_70b", N, K, seed=32)
    q = w4.quantize_weight_msd(dev(Wb), 2)
    torch.cuda.synchronize()
    cw, sw = orc.quant_mxfp4(Wb)
    np.testing.assert_array_equal(q.codes.cpu().numpy()[: N * K].reshape(N, K), np.concatenate([cw, cw], 1))
    np.testing.assert_array_equal(H.unswizzle_scales(q.scales.cpu().numpy(), N, 2 * K, 32), np.concatenate([sw, sw], 1))


def _ref(orc, Xa, Xw, passes):
    ca, sa = orc.quant_mxfp4_msd(Xa, passes=passes)
    cw, sw = orc.quant_mxfp4(Xw)
    return orc.gemm_mxfp4(ca, sa, np.concatenate([cw] * passes, 1), np.concatenate([sw] * passes, 1))


# M = 1 and 16: split-K decode; 100: one-CTA kernel; 300: CTA pair
@pytest.mark.parametrize("M", [1, 16, 100, 300])
@pytest.mark.parametrize("passes", [2, 3])
def test_msd_linear_parity(orc, M, passes):
    N, K = 384, 1280
    Xa = synth.activations("llama2_70b", M, K, seed=33)
    Xw = synth.weights("llama2_70b", N, K, seed=33)
    Wq = w4.quantize_weight_msd(dev(Xw), passes)
    Y = w4.linear_msd(dev(Xa), Wq, passes)
    Yg = w4.gemm(w4.quantize_act_msd(dev(Xa), passes), Wq)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _, yref, absd = _ref(orc, Xa, Xw, passes)
    for name, out in (("linear", Y), ("gemm", Yg)):
        bad = H.gemm_violations(H.to_np_u16(out), yref, absd)
        assert not bad.any(), f"{name}: {bad.sum()} of {bad.size} outside tolerance"


def test_msd_two_passes_beat_one_pass_on_the_product(orc):
    """The decomposition's purpose: the two-pass product is closer to the
    unquantized-activation product (X in bf16 times the quantized weights)."""
    M, N, K = 64, 256, 2048
    Xa = synth.activations("llama2_70b", M, K, seed=34)
    Xw = synth.weights("llama2_70b", N, K, seed=34)
    cw, sw = orc.quant_mxfp4(Xw)
    exact = synth.bf16_bits_to_f32(Xa).astype(np.float64) @ orc.dequant_mxfp4(cw, sw).T
    Wq1, Wq2 = w4.quantize_weight(dev(Xw), w4.MXFP4), w4.quantize_weight_msd(dev(Xw), 2)
    Y1 = H.bf16_to_f64(H.to_np_u16(w4.linear(dev(Xa), Wq1, 0)))
    Y2 = H.bf16_to_f64(H.to_np_u16(w4.linear_msd(dev(Xa), Wq2, 2)))
    e1, e2 = np.abs(Y1 - exact).mean(), np.abs(Y2 - exact).mean()
    assert e2 < e1 / 3, (e1, e2)


def test_msd_sampled_at_llama_qkv_size(orc):
    """Llama-2-70B qkv (8192 -> 10240) at 4096 tokens, two passes: the
    activation passes compared in full, the product on sampled rows."""
    M, N, K = 4096, 10240, 8192
    Xa = synth.activations("llama2_70b", M, K, seed=0)
    Xw = synth.weights("llama2_70b", N, K, seed=0)
    Wq = w4.quantize_weight_msd(dev(Xw), 2)
    q = _check_act(orc, Xa, 2)
    Y = w4.linear_msd(dev(Xa), Wq, 2)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    pick = np.array([0, 1, 255, 256, 2047, 4095])
    _, yref, absd = _ref(orc, Xa[pick], Xw, 2)
    bad = H.gemm_violations(H.to_np_u16(Y)[pick], yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"
    del q
