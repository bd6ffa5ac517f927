"""GPU parity at the workloads' full sizes, through the calls the benchmark
times (w4a4_linear on weights from w4a4_quantize_weight).  The oracle checks
sampled rows: activation rows are quantized independently (per token), so a
sampled row's codes, scales and s2 are compared bit for bit; weight rows with
a tensor scale are compared after the scale itself (amax over the whole
matrix) is checked; GEMM outputs of the sampled rows are compared over all N
within 1 bf16 ulp + 1e-5 * sum|a w|."""
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


def _rows(M):
    return np.unique(np.array([0, 1, M // 2, M - 1]))[: M]


def _nv_rows(q, rows, cols):
    """Codes, unswizzled scales and s2 of the given rows of an NVFP4 tensor."""
    codes = q.codes.cpu().numpy()[: q.rows * cols // 2].reshape(q.rows, cols // 2)[rows]
    sc = H.unswizzle_scales(q.scales.cpu().numpy(), q.rows, cols, 16)[rows]
    return codes, sc


_WQ_CACHE = {}


def _oracle_weights(orc, key, Wb):
    """The oracle's NVFP4 tensor-scale quantization of a whole weight matrix,
    computed once per matrix."""
    if key not in _WQ_CACHE:
        _WQ_CACHE.clear()  # one matrix at a time (they are large)
        _WQ_CACHE[key] = orc.quant_nvfp4(Wb, mode=0)
    return _WQ_CACHE[key]


def _check_nvfp4_linear(orc, Xa, Wb, a_mode, Xq_dev, Wq, Y, key):
    """Sampled-row parity of one NVFP4 linear: activation rows, weight rows,
    the weight tensor scale, and the output rows."""
    M, K = Xa.shape
    N = Wb.shape[0]
    rows = _rows(M)
    # weights: the tensor scale from the whole matrix, then sampled rows with it
    w = synth.bf16_bits_to_f32(Wb)
    s2w = orc.lib().orc_nvfp4_s2_from_amax(float(np.abs(w).max()))
    assert np.float32(Wq.s2.cpu().numpy()[0]) == np.float32(s2w)
    wrows = _rows(N)
    cw_s, sw_s, _ = orc.quant_nvfp4(Wb[wrows], mode=0, static_s2=np.array([s2w], np.float32))
    gc, gs = _nv_rows(Wq, wrows, K)
    np.testing.assert_array_equal(gc, cw_s)
    np.testing.assert_array_equal(gs, sw_s)
    # activations (per token rows are independent; a tensor scale is checked whole)
    if a_mode == w4.SCALE_TOKEN:
        ca, sa, s2a = orc.quant_nvfp4(Xa[rows], mode=1)
    else:
        x = synth.bf16_bits_to_f32(Xa)
        s2x = np.float32(orc.lib().orc_nvfp4_s2_from_amax(float(np.abs(x).max())))
        ca, sa, s2a = orc.quant_nvfp4(Xa[rows], mode=0, static_s2=np.array([s2x], np.float32))
    if Xq_dev is not None:
        gc, gs = _nv_rows(Xq_dev, rows, K)
        np.testing.assert_array_equal(gc, ca)
        np.testing.assert_array_equal(gs, sa)
    # the product of the sampled rows with all of W (the oracle quantizes W whole)
    cw, sw, s2 = _oracle_weights(orc, key, Wb)
    _, yref, absd = orc.gemm_nvfp4(ca, sa, s2a, a_mode, cw, sw, s2)
    bad = H.gemm_violations(H.to_np_u16(Y)[rows], yref, absd)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outputs outside tolerance"


def test_mxfp4_small_gemm_in_full(orc):
    """16 x 256 by 256 x 256 MXFP4, X ~ N(0,1), W ~ N(0,0.02), seed 0: every
    code, scale and output."""
    Xa = synth.activations("mxfp4_small", 16, 256, seed=0)
    Xw = synth.weights("mxfp4_small", 256, 256, seed=0)
    A = w4.quantize_act(dev(Xa), w4.MXFP4, 0)
    B = w4.quantize_weight(dev(Xw), w4.MXFP4)
    Y = w4.linear(dev(Xa), B, 0)
    torch.cuda.synchronize()
    ca, sa = orc.quant_mxfp4(Xa)
    cw, sw = orc.quant_mxfp4(Xw)
    np.testing.assert_array_equal(A.codes.cpu().numpy()[: 16 * 128].reshape(16, 128), ca)
    np.testing.assert_array_equal(H.unswizzle_scales(A.scales.cpu().numpy(), 16, 256, 32), sa)
    np.testing.assert_array_equal(B.codes.cpu().numpy()[: 256 * 128].reshape(256, 128), cw)
    _, yref, absd = orc.gemm_mxfp4(ca, sa, cw, sw)
    assert not H.gemm_violations(H.to_np_u16(Y), yref, absd).any()


@pytest.mark.parametrize("li", range(5))
def test_swiglu300m_layer_tensor_scales(orc, li):
    """300M SwiGLU decoder linears at M = 4096, NVFP4 with a tensor scale on
    both sides (X ~ N(0,1) with 8 channels x50)."""
    name, K, N = synth.SHAPES["swiglu300m"][li]
    M = 4096
    Xa = synth.activations("swiglu300m", M, K, seed=0, tensor_id=200 + li)
    Wb = synth.weights("swiglu300m", N, K, seed=0, tensor_id=100 + li)
    Wq = w4.quantize_weight(dev(Wb), w4.NVFP4)
    Xq = w4.quantize_act(dev(Xa), w4.NVFP4, w4.SCALE_TENSOR)
    Y = w4.linear(dev(Xa), Wq, w4.SCALE_TENSOR)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _check_nvfp4_linear(orc, Xa, Wb, w4.SCALE_TENSOR, Xq, Wq, Y, ("swiglu300m", li))


# ordered by linear, so each weight matrix is quantized by the oracle once
LLAMA_CASES = [(M, li) for li in range(5) for M in (1, 16, 256, 4096)] + [(16384, 4)]


@pytest.fixture(scope="module")
def llama_weights():
    """The Llama-2-70B layer's weight bits (seed 0), drawn once for the module."""
    return [synth.weights("llama2_70b", N, K, seed=0, tensor_id=100 + li)
            for li, (name, K, N) in enumerate(synth.SHAPES["llama2_70b"])]


@pytest.mark.parametrize("M,li", LLAMA_CASES)
def test_llama2_70b_linears(orc, llama_weights, M, li):
    """Llama-2-70B linears, per-token NVFP4 activations (0.5 * Student-t(4)),
    at every token count of the workload: decode (M <= 16), the CTA pair."""
    name, K, N = synth.SHAPES["llama2_70b"][li]
    Wb = llama_weights[li]
    Xa = synth.activations("llama2_70b", M, K, seed=0, tensor_id=200 + li)
    Wq = w4.quantize_weight(dev(Wb), w4.NVFP4)
    Xq = w4.quantize_act(dev(Xa), w4.NVFP4, w4.SCALE_TOKEN)
    Y = w4.linear(dev(Xa), Wq, w4.SCALE_TOKEN)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _check_nvfp4_linear(orc, Xa, Wb, w4.SCALE_TOKEN, Xq, Wq, Y, ("llama2_70b", li))


@pytest.mark.parametrize("li", range(4))
def test_qwen25_7b_int4_g128(orc, li):
    """INT4-g128 Qwen2.5-7B linears at M = 2048 (X ~ N(0,1), 0.5% channels
    x20): sampled activation and weight rows bit-exact (every row is
    quantized on its own), sampled output rows within tolerance."""
    name, K, N = synth.SHAPES["qwen25_7b_int4"][li]
    M = 2048
    Xa = synth.activations("qwen25_7b_int4", M, K, seed=0, tensor_id=200 + li)
    Wb = synth.weights("qwen25_7b_int4", N, K, seed=0, tensor_id=100 + li)
    Wq = w4.quantize_weight(dev(Wb), w4.INT4)
    Xq = w4.quantize_act(dev(Xa), w4.INT4, 0)
    Y = w4.linear(dev(Xa), Wq, 0)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    rows, wrows = _rows(M), _rows(N)
    ca, sa = orc.quant_int4(Xa[rows])
    cw_s, sw_s = orc.quant_int4(Wb[wrows])
    for q, r, c, s in ((Xq, rows, ca, sa), (Wq, wrows, cw_s, sw_s)):
        codes = q.codes.cpu().numpy()[: q.rows * K // 2].reshape(q.rows, K // 2)[r]
        np.testing.assert_array_equal(codes, c)
        sc = H.int4_scales(q.scales.cpu().numpy().view(np.float32), q.rows, K)[r]
        np.testing.assert_array_equal(sc.view(np.uint32), s.view(np.uint32))
    cw, sw = orc.quant_int4(Wb)
    _, yref, absd = orc.gemm_int4(ca, sa, cw, sw)
    bad = H.gemm_violations(H.to_np_u16(Y)[rows], yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"


@pytest.mark.parametrize("li", range(3))
def test_qwen25_3b_augmented(orc, li):
    """Dual-stage NVFP4 augmentation, Qwen2.5-3B shapes at M = 8192, the 256
    channels chosen from the seed-1 calibration batch ("APEX4..." page, para 2:
    ARCQuant).  Bit for bit on sampled rows: the augmented activation codes and
    block scales over all K + 256 columns (first stage, then the residual
    stage, as the fused linear runs them), the row scales, and the weight codes
    and block scales of [W | W[:, S]]; the sampled output rows within the GEMM
    tolerance."""
    name, K, N = synth.SHAPES["qwen25_3b_aug"][li]
    M, nS = 8192, 256
    cols = K + nS
    S_np = orc.select_channels(synth.calibration("qwen25_3b_aug", K), nS)
    S = torch.from_numpy(S_np).cuda()
    np.testing.assert_array_equal(w4.select_channels(dev(synth.calibration("qwen25_3b_aug", K)), nS).cpu().numpy(),
                                  S_np)
    Xa = synth.activations("qwen25_3b_aug", M, K, seed=0, tensor_id=200 + li)
    Wb = synth.weights("qwen25_3b_aug", N, K, seed=0, tensor_id=100 + li)
    Xd = dev(Xa)
    Wq = w4.quantize_weight(dev(Wb), w4.NVFP4, S=S)
    Xq = w4.quantize_act(Xd, w4.NVFP4, w4.SCALE_TOKEN, cols=cols)
    w4.augment_residual(Xd, S, Xq)
    Y = w4.linear(Xd, Wq, w4.SCALE_TOKEN, S=S)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    rows = _rows(M)
    ca, sa, s2a = orc.quant_nvfp4(Xa[rows], mode=1)
    rc, rs = orc.augment_nvfp4(Xa[rows], S_np, ca, sa, s2a, 1)
    ca, sa = np.concatenate([ca, rc], 1), np.concatenate([sa, rs], 1)
    gc, gs = _nv_rows(Xq, rows, cols)
    np.testing.assert_array_equal(gc, ca)
    np.testing.assert_array_equal(gs, sa)
    np.testing.assert_array_equal(Xq.s2.cpu().numpy()[rows], s2a)
    cw, sw, s2w = orc.quant_nvfp4(np.ascontiguousarray(np.concatenate([Wb, Wb[:, S_np]], 1)), mode=0)
    assert np.float32(Wq.s2.cpu().numpy()[0]) == np.float32(s2w[0])
    wrows = _rows(N)
    gc, gs = _nv_rows(Wq, wrows, cols)
    np.testing.assert_array_equal(gc, cw[wrows])
    np.testing.assert_array_equal(gs, sw[wrows])
    _, yref, absd = orc.gemm_nvfp4(ca, sa, s2a, 1, cw, sw, s2w)
    bad = H.gemm_violations(H.to_np_u16(Y)[rows], yref, absd)
    assert not bad.any(), f"{bad.sum()} bad"
    # the linear's quantizer computes the residual stage in the same launch:
    # its product equals the two-call path's byte for byte
    Y2 = w4.gemm(Xq, Wq)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("M", [4096, 600])
def test_llama2_70b_tensor_scale_both_quantizer_paths(orc, llama_weights, M):
    """NVFP4 with a tensor activation scale at the o projection's K = 8192:
    M = 4096 rows do not fit in shared memory across the SMs (amax pass, then
    the row-ring quantizer); M = 600 do (one cooperative pass).  Sampled rows
    bit-exact against the oracle with the tensor's amax, outputs within
    tolerance."""
    name, K, N = synth.SHAPES["llama2_70b"][1]
    Wb = llama_weights[1]
    Xa = synth.activations("llama2_70b", M, K, seed=5, tensor_id=300)
    Wq = w4.quantize_weight(dev(Wb), w4.NVFP4)
    Xq = w4.quantize_act(dev(Xa), w4.NVFP4, w4.SCALE_TENSOR)
    Y = w4.linear(dev(Xa), Wq, w4.SCALE_TENSOR)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _check_nvfp4_linear(orc, Xa, Wb, w4.SCALE_TENSOR, Xq, Wq, Y, ("llama2_70b", 1))
