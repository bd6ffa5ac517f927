"""GPU parity of NVFP4 weights with one global scale per row segment (fused
q/k/v or gate/up modules, "Daily Papers" page, para 4, Minima: one NVFP4
global scale per module).  Quantization bit-exact against the oracle's
per-segment rule; the GEMM and the fused linear on every kernel that can read
the weights (CTA pair for M > 128, one CTA for M <= 128, split-K decode for
M <= 16) within 1 bf16 ulp + 1e-5 * sum|a w| of the oracle's per-row-scale
product; one segment reproduces the tensor-scale path bit for bit."""
import numpy as np
import pytest

from tests import helpers as H
from w4a4_quantized_gemm_token_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_quantized_gemm_token_b200 as w4  # noqa: E402

# q | k | v in the proportions of Llama-2-70B's fused qkv (8 : 1 : 1), scaled down
SEG_ROWS, GAINS = (512, 128, 128), (1.0, 4.0, 0.25)


def dev(bits):
    return H.to_dev_bf16(bits)


def _codes(q, rows):
    return q.codes.cpu().numpy()[: rows * q.cols // 2].reshape(rows, q.cols // 2)


@pytest.mark.parametrize("K", [256, 1280, 8192])
def test_segment_quant_bitexact(orc, K):
    Wb, seg = synth.fused_weights(SEG_ROWS, GAINS, K, seed=7)
    N = seg[-1]
    q = w4.quantize_weight_segments(dev(Wb), seg)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    oc, osc, os2 = orc.quant_nvfp4_segments(Wb, seg)
    np.testing.assert_array_equal(_codes(q, N), oc)
    np.testing.assert_array_equal(H.unswizzle_scales(q.scales.cpu().numpy(), N, K, 16), osc)
    np.testing.assert_array_equal(q.s2.cpu().numpy()[:N], os2)
    # three different scales, constant inside each segment
    assert len(set(os2.tolist())) == 3


def test_segment_quant_with_residual_channels(orc):
    """[W | W[:,S]] per segment: the appended channels take their segment's scale."""
    K, nS = 1024, 128
    Wb, seg = synth.fused_weights(SEG_ROWS, GAINS, K, seed=8)
    N = seg[-1]
    S_np = orc.select_channels(synth.calibration("qwen25_3b_aug", K, rows=256), nS)
    q = w4.quantize_weight_segments(dev(Wb), seg, S=torch.from_numpy(S_np).cuda())
    torch.cuda.synchronize()
    oc, osc, os2 = orc.quant_nvfp4_segments(np.concatenate([Wb, Wb[:, S_np]], 1), seg)
    np.testing.assert_array_equal(_codes(q, N), oc)
    np.testing.assert_array_equal(H.unswizzle_scales(q.scales.cpu().numpy(), N, K + nS, 16), osc)
    np.testing.assert_array_equal(q.s2.cpu().numpy()[:N], os2)


def _ref(orc, Xa, Wb, seg, a_mode, S=None):
    ca, sa, s2a = orc.quant_nvfp4(Xa, mode=a_mode)
    if S is not None:
        rc, rs = orc.augment_nvfp4(Xa, S, ca, sa, s2a, a_mode)
        ca, sa = np.concatenate([ca, rc], 1), np.concatenate([sa, rs], 1)
        Wb = np.concatenate([Wb, Wb[:, S]], 1)
    cw, sw, s2w = orc.quant_nvfp4_segments(Wb, seg)
    return orc.gemm_nvfp4(ca, sa, s2a, a_mode, cw, sw, s2w)


# M = 1 and 16: split-K decode; 100: one-CTA kernel; 300: CTA pair
@pytest.mark.parametrize("M", [1, 16, 100, 300])
@pytest.mark.parametrize("a_mode", [w4.SCALE_TOKEN, w4.SCALE_TENSOR])
def test_segment_linear_parity(orc, M, a_mode):
    K = 1280
    Xa = synth.activations("llama2_70b", M, K, seed=13)
    Wb, seg = synth.fused_weights(SEG_ROWS, GAINS, K, seed=13)
    Wq = w4.quantize_weight_segments(dev(Wb), seg)
    Y = w4.linear(dev(Xa), Wq, a_mode)
    Yg = w4.gemm(w4.quantize_act(dev(Xa), w4.NVFP4, a_mode), Wq)
    Yn = w4.linear_noalloc(dev(Xa), Wq, a_mode) if M <= 16 else Y
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _, yref, absd = _ref(orc, Xa, Wb, seg, a_mode)
    for name, out in (("linear", Y), ("gemm", Yg), ("noalloc", Yn)):
        bad = H.gemm_violations(H.to_np_u16(out), yref, absd)
        assert not bad.any(), f"{name}: {bad.sum()} of {bad.size} outside tolerance at {np.argwhere(bad)[:4]}"


@pytest.mark.parametrize("M", [16, 300])
def test_segment_linear_with_residual_channels(orc, M):
    K, nS = 1024, 128
    Xa = synth.activations("qwen25_3b_aug", M, K, seed=6)
    Wb, seg = synth.fused_weights(SEG_ROWS, GAINS, K, model="qwen25_3b_aug", seed=6)
    S_np = orc.select_channels(synth.calibration("qwen25_3b_aug", K, rows=256), nS)
    S = torch.from_numpy(S_np).cuda()
    Wq = w4.quantize_weight_segments(dev(Wb), seg, S=S)
    Y = w4.linear(dev(Xa), Wq, w4.SCALE_TOKEN, S=S)
    torch.cuda.synchronize()
    _, yref, absd = _ref(orc, Xa, Wb, seg, w4.SCALE_TOKEN, S=S_np)
    bad = H.gemm_violations(H.to_np_u16(Y), yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"


@pytest.mark.parametrize("M", [1, 16, 100, 300, 600])
def test_one_segment_is_the_tensor_scale_path(M):
    """A single segment quantizes like w4a4_quantize_weight and, since the
    epilogue forms alpha = s2_A * s2_B[n] the same way, gives identical bytes."""
    N, K = 768, 1024
    Xa = dev(synth.activations("llama2_70b", M, K, seed=17))
    Wb = dev(synth.weights("llama2_70b", N, K, seed=17))
    Wt = w4.quantize_weight(Wb, w4.NVFP4)
    Wr = w4.quantize_weight_segments(Wb, [0, N])
    torch.cuda.synchronize()
    assert torch.equal(Wt.codes, Wr.codes) and torch.equal(Wt.scales, Wr.scales)
    assert torch.all(Wr.s2[:N] == Wt.s2[0])
    Yt = w4.linear(Xa, Wt, w4.SCALE_TOKEN)
    Yr = w4.linear(Xa, Wr, w4.SCALE_TOKEN)
    torch.cuda.synchronize()
    assert torch.equal(Yt.view(torch.int16), Yr.view(torch.int16))


def test_segments_sampled_at_llama_qkv_size(orc):
    """Llama-2-70B fused qkv (10240 x 8192, segments 8192 | 1024 | 1024) at 4096
    tokens: quantization compared in full per segment, the product on sampled
    output rows, each against the oracle."""
    K = 8192
    rows, gains = synth.FUSED["llama2_70b"]["qkv"]
    Wb, seg = synth.fused_weights(rows, gains, K, seed=0)
    N = seg[-1]
    M = 4096
    Xa = synth.activations("llama2_70b", M, K, seed=0)
    Wq = w4.quantize_weight_segments(dev(Wb), seg)
    Y = w4.linear(dev(Xa), Wq, w4.SCALE_TOKEN)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    oc, osc, os2 = orc.quant_nvfp4_segments(Wb, seg)
    q_s2 = Wq.s2.cpu().numpy()[:N]
    np.testing.assert_array_equal(q_s2, os2)
    np.testing.assert_array_equal(_codes(Wq, N), oc)
    np.testing.assert_array_equal(H.unswizzle_scales(Wq.scales.cpu().numpy(), N, K, 16), osc)
    assert len(set(q_s2.tolist())) == 3
    pick = np.array([0, 1, 255, 256, 2047, 4095])
    ca, sa, s2a = orc.quant_nvfp4(Xa[pick], mode=1)
    _, yref, absd = orc.gemm_nvfp4(ca, sa, s2a, 1, oc, osc, os2)
    bad = H.gemm_violations(H.to_np_u16(Y)[pick], yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"
