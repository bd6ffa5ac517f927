"""Every finite bf16 value through the GPU quantizers, bit for bit against the
oracle.

The E2M1 and E4M3 conversions the quantizers use are hardware instructions
(round to nearest even, saturating, sign kept).  These tests feed every one
of the 65280 finite bf16 bit patterns (both zeros, the subnormals, every
E2M1 midpoint) through each activation quantizer in two arrangements:

* blocks with a fixed maximum, so that the element scale is exactly 1 and
  the E2M1 (or INT4) conversion sees the bf16 value itself: MXFP4 blocks
  led by 6.0 (shared exponent floor(log2 6) - 2 = 0), NVFP4 blocks led by
  6.0 with a static second-level scale of 1 (block scale E4M3(6/6/1) = 1),
  INT4 groups led by 7.0 (scale 7/7 = 1).  Values whose magnitude exceeds
  the leader change the block's scale and are still compared;
* the values in ascending bit order, packed into blocks as they come, under
  every scale mode, so each block scale (E4M3 or E8M0) is exercised over the
  whole bf16 range.

Formats: the "Daily Papers" page, para 4 (Minima: NVFP4 with 16-element
blocks, E4M3 block scales and a global scale) and the "Depth Registers..."
thelatestinai page, para 1 (the open MXFP4 standard); the element and scale
encodings are those of the OCP Microscaling and NVFP4 definitions.
"""
import numpy as np
import pytest

from tests import helpers as H

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_quantized_gemm_token_b200 as w4  # noqa: E402
from tests.test_gpu_parity import check_quant  # noqa: E402


def finite_bf16():
    """All finite bf16 bit patterns (exponent field below 0xFF), ascending."""
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


def led_blocks(values, block, leader, K):
    """Rows of K elements: blocks of `block` elements whose first element is
    `leader` (bf16 bits) and whose others are the given values in order
    (the last block padded with zeros)."""
    per = block - 1
    nblk = -(-len(values) // per)
    out = np.zeros((nblk, block), np.uint16)
    out[:, 0] = leader
    flat = out[:, 1:].reshape(-1)
    flat[: len(values)] = values
    out[:, 1:] = flat.reshape(nblk, per)
    flat = out.reshape(-1)
    rows = -(-len(flat) // K)
    X = np.zeros(rows * K, np.uint16)
    X[: len(flat)] = flat
    return X.reshape(rows, K)


def sorted_rows(values, K):
    rows = -(-len(values) // K)
    X = np.zeros(rows * K, np.uint16)
    X[: len(values)] = values
    return X.reshape(rows, K)


BF16_SIX, BF16_SEVEN = 0x40C0, 0x40E0


def test_finite_bf16_count():
    v = finite_bf16()
    assert len(v) == 65280
    f = H.bf16_to_f64(v)
    assert np.isfinite(f).all()
    # every E2M1 midpoint and both zeros are among them
    for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0):
        assert (f == m).any() and (f == -m).any()
    assert ((v == 0x0000) | (v == 0x8000)).sum() == 2


def test_every_bf16_at_unit_scale_mxfp4(orc):
    X = led_blocks(finite_bf16(), 32, BF16_SIX, 4096)
    check_quant(orc, X, w4.MXFP4)


def test_every_bf16_at_unit_scale_nvfp4(orc):
    X = led_blocks(finite_bf16(), 16, BF16_SIX, 4096)
    check_quant(orc, X, w4.NVFP4, w4.SCALE_TENSOR, static=np.array([1.0], np.float32))


def test_every_bf16_at_unit_scale_int4(orc):
    X = led_blocks(finite_bf16(), 128, BF16_SEVEN, 4096)
    check_quant(orc, X, w4.INT4)


def test_unit_scale_blocks_really_have_unit_scale(orc):
    """The arrangement does what it says: a led block whose values stay below
    the leader gets E8M0 code 127 (2^0), E4M3 scale 0x38 (1.0), INT4 scale 1."""
    vals = np.array([0x3E80, 0xBF40, 0x0001, 0x8000], np.uint16)  # 0.25, -0.75, tiny, -0
    Xm = led_blocks(vals, 32, BF16_SIX, 128)
    _, sm = orc.quant_mxfp4(Xm)
    assert sm[0, 0] == 127
    Xn = led_blocks(vals, 16, BF16_SIX, 128)
    _, sn, _ = orc.quant_nvfp4(Xn, mode=0, static_s2=np.array([1.0], np.float32))
    assert sn[0, 0] == 0x38
    Xi = led_blocks(vals, 128, BF16_SEVEN, 128)
    _, si = orc.quant_int4(Xi)
    assert si[0, 0] == np.float32(1.0)


@pytest.mark.parametrize("fmt,mode", [(w4.NVFP4, w4.SCALE_TOKEN), (w4.NVFP4, w4.SCALE_TENSOR),
                                      (w4.MXFP4, 0), (w4.INT4, 0)])
def test_every_bf16_in_ascending_blocks(orc, fmt, mode):
    check_quant(orc, sorted_rows(finite_bf16(), 4096), fmt, mode)


def test_every_bf16_nvfp4_static_scales(orc):
    """Static second-level scales far from 1 push the block-scale quotient
    through E4M3's subnormal and saturating ranges."""
    X = sorted_rows(finite_bf16(), 4096)
    for s in (1.0, 2.0 ** -20, 2.0 ** 20, 0.0123):
        check_quant(orc, X, w4.NVFP4, w4.SCALE_TENSOR, static=np.array([s], np.float32))
