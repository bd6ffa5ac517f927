"""GPU edge cases of the fused linear and the GEMM: the largest K the library
accepts (65536), the smallest N (one 128-row weight tile), M = 0 (a no-op
that leaves Y untouched), activation rows with a stride larger than K, and
every GEMM kernel (decode M <= 16, one CTA M <= 128, CTA pair) at these
boundaries, each against the oracle within 1 bf16 ulp + 1e-5 * sum|a w|."""
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


def _nvfp4_ref(orc, Xa, Xw):
    ca, sa, s2a = orc.quant_nvfp4(Xa, mode=1)
    cw, sw, s2w = orc.quant_nvfp4(Xw, mode=0)
    return orc.gemm_nvfp4(ca, sa, s2a, 1, cw, sw, s2w)


@pytest.mark.parametrize("M", [1, 16, 130])
def test_largest_k(orc, M):
    """K = 65536, the library's limit (the decode kernel's 3-D boxes, the
    pair kernel's raster over a long K, 4096 scale atoms per row)."""
    N, K = 128, 65536
    Xa = synth.activations("llama2_70b", M, K, seed=91)
    Xw = synth.weights("llama2_70b", N, K, seed=91)
    Y = w4.linear(dev(Xa), w4.quantize_weight(dev(Xw), w4.NVFP4), w4.SCALE_TOKEN)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _, yref, absd = _nvfp4_ref(orc, Xa, Xw)
    assert not H.gemm_violations(H.to_np_u16(Y), yref, absd).any()


@pytest.mark.parametrize("M", [1, 100, 257])
@pytest.mark.parametrize("fmt", [w4.NVFP4, w4.MXFP4, w4.INT4])
def test_one_weight_tile(orc, M, fmt):
    """N = 128: a single weight tile (half of a pair tile's columns)."""
    N, K = 128, 512
    Xa = synth.activations("llama2_70b", M, K, seed=92)
    Xw = synth.weights("llama2_70b", N, K, seed=92)
    mode = w4.SCALE_TOKEN if fmt == w4.NVFP4 else 0
    Y = w4.linear(dev(Xa), w4.quantize_weight(dev(Xw), fmt), mode)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    if fmt == w4.NVFP4:
        _, yref, absd = _nvfp4_ref(orc, Xa, Xw)
    elif fmt == w4.MXFP4:
        ca, sa = orc.quant_mxfp4(Xa)
        cw, sw = orc.quant_mxfp4(Xw)
        _, yref, absd = orc.gemm_mxfp4(ca, sa, cw, sw)
    else:
        ca, sa = orc.quant_int4(Xa)
        cw, sw = orc.quant_int4(Xw)
        _, yref, absd = orc.gemm_int4(ca, sa, cw, sw)
    assert not H.gemm_violations(H.to_np_u16(Y), yref, absd).any()


def test_zero_tokens_leave_y_untouched():
    N, K = 256, 512
    Wq = w4.quantize_weight(dev(synth.weights("llama2_70b", N, K, seed=93)), w4.NVFP4)
    X = torch.zeros(0, K, dtype=torch.bfloat16, device="cuda")
    Y = torch.full((1, N), 7.0, dtype=torch.bfloat16, device="cuda")
    w4.linear(X, Wq, w4.SCALE_TOKEN, Y=Y[:0])
    q = w4.quantize_act(X, w4.NVFP4, w4.SCALE_TOKEN)
    w4.gemm(q, Wq, Y[:0])
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    assert torch.all(Y == 7.0)


@pytest.mark.parametrize("M", [3, 200])
def test_strided_activation_rows(orc, M):
    """X rows with a stride of K + 64 elements (a slice of a wider tensor)."""
    N, K = 256, 1024
    Xfull = synth.activations("llama2_70b", M, K + 64, seed=94)
    Xa = np.ascontiguousarray(Xfull[:, :K])
    Xw = synth.weights("llama2_70b", N, K, seed=94)
    Xd = dev(Xfull)[:, :K]
    assert Xd.stride(0) == K + 64
    Y = w4.linear(Xd, w4.quantize_weight(dev(Xw), w4.NVFP4), w4.SCALE_TOKEN)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _, yref, absd = _nvfp4_ref(orc, Xa, Xw)
    assert not H.gemm_violations(H.to_np_u16(Y), yref, absd).any()


def test_output_row_stride(orc):
    """Y written into a wider buffer (ldy > N): the columns past N stay untouched."""
    M, N, K = 40, 256, 512
    Xa = synth.activations("llama2_70b", M, K, seed=95)
    Xw = synth.weights("llama2_70b", N, K, seed=95)
    big = torch.full((M, N + 64), 3.0, dtype=torch.bfloat16, device="cuda")
    w4.linear(dev(Xa), w4.quantize_weight(dev(Xw), w4.NVFP4), w4.SCALE_TOKEN, Y=big[:, :N])
    torch.cuda.synchronize()
    assert torch.all(big[:, N:] == 3.0)
    _, yref, absd = _nvfp4_ref(orc, Xa, Xw)
    assert not H.gemm_violations(H.to_np_u16(big[:, :N].contiguous()), yref, absd).any()
