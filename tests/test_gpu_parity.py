"""GPU parity: every kernel through the C-ABI against the C oracle on the same
seeded inputs.  Codes and scales bit-exact; GEMM outputs within
1 bf16 ulp + 1e-5 * sum|a w|.  Sizes span several tiles and ragged tails."""
import numpy as np
import pytest

from tests import helpers as H
from w4a4_quantized_gemm_token_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import w4a4_quantized_gemm_token_b200 as w4  # noqa: E402

FMT_NAMES = {w4.NVFP4: "nvfp4", w4.MXFP4: "mxfp4", w4.INT4: "int4"}


def dev(bits):
    return H.to_dev_bf16(bits)


def check_quant(orc, Xb, fmt, mode=w4.SCALE_TOKEN, static=None, cols=None):
    """Quantize on the GPU and compare codes / scales / s2 with the oracle."""
    M, K = Xb.shape
    st = None if static is None else torch.from_numpy(np.asarray(static, np.float32)).cuda()
    q = w4.quantize_act(dev(Xb), fmt, mode, static_s2=st, cols=cols)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    cols = q.cols
    codes = q.codes.cpu().numpy()[: M * cols // 2].reshape(M, cols // 2)[:, : K // 2]
    if fmt == w4.NVFP4:
        oc, osc, os2 = orc.quant_nvfp4(Xb, mode=mode, static_s2=static)
        np.testing.assert_array_equal(codes, oc)
        sc = H.unswizzle_scales(q.scales.cpu().numpy(), M, cols, 16)[:, : K // 16]
        np.testing.assert_array_equal(sc, osc)
        s2 = q.s2.cpu().numpy()
        np.testing.assert_array_equal(s2[: len(os2)], os2)
        assert np.all(H.padding_scales(q.scales.cpu().numpy(), M, cols, 16) == 0)
    elif fmt == w4.MXFP4:
        oc, osc = orc.quant_mxfp4(Xb)
        np.testing.assert_array_equal(codes, oc)
        sc = H.unswizzle_scales(q.scales.cpu().numpy(), M, cols, 32)[:, : K // 32]
        np.testing.assert_array_equal(sc, osc)
        assert np.all(H.padding_scales(q.scales.cpu().numpy(), M, cols, 32) == 0)
    else:
        oc, osc = orc.quant_int4(Xb)
        np.testing.assert_array_equal(codes, oc)
        sc = H.int4_scales(q.scales.cpu().numpy().view(np.float32), M, cols)[:, : K // 128]
        np.testing.assert_array_equal(sc.view(np.uint32), osc.view(np.uint32))
    return q


QUANT_SHAPES = [(1, 128), (5, 384), (130, 1024), (300, 2816), (17, 8192), (3, 28672), (2, 40960)]


@pytest.mark.parametrize("M,K", QUANT_SHAPES)
@pytest.mark.parametrize("fmt,mode", [(w4.NVFP4, w4.SCALE_TOKEN), (w4.NVFP4, w4.SCALE_TENSOR),
                                      (w4.MXFP4, 0), (w4.INT4, 0)])
def test_quant_bitexact(orc, M, K, fmt, mode):
    X = synth.activations("swiglu300m" if K == 1024 else "llama2_70b", M, K, seed=3)
    check_quant(orc, X, fmt, mode)


def test_quant_static_scales(orc):
    X = synth.activations("llama2_70b", 70, 512, seed=4)
    check_quant(orc, X, w4.NVFP4, w4.SCALE_TENSOR, static=np.array([0.0123], np.float32))
    s = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.linspace(1e-3, 0.1, 70)))
    check_quant(orc, X, w4.NVFP4, w4.SCALE_TOKEN, static=s)


def test_quant_special_values(orc):
    """Ties of the E2M1 grid hit exactly (static s2 = 1, block amax 6 -> scale 1),
    signed zeros, tiny negatives, all-zero blocks and rows, huge and subnormal values."""
    ties = [6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5, -.25, -.75, -1.25, -1.75, -2.5, -3.5, -5, -0.0]
    neg = [-6, -0.1, -0.0, 0.0, 1e-3, -1e-3, 0.2, -0.2, 3, -3, 4, 0.5, -0.5, 1, -1, 2]
    rows = [ties * 8, neg * 8, [0.0] * 128, [1e30] + [0.0] * 127,
            [1e-40, -3e-39] + [0.0] * 126, list(np.linspace(-7, 7, 128))]
    X = synth.f32_to_bf16_bits(np.array(rows, np.float32))
    for fmt in (w4.MXFP4, w4.INT4):
        check_quant(orc, X, fmt)
    check_quant(orc, X, w4.NVFP4, w4.SCALE_TENSOR, static=np.array([1.0], np.float32))
    check_quant(orc, X, w4.NVFP4, w4.SCALE_TOKEN)
    check_quant(orc, X, w4.NVFP4, w4.SCALE_TENSOR)


def test_quant_empty_and_strided(orc):
    X = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    q = w4.quantize_act(X, w4.NVFP4, w4.SCALE_TOKEN)
    assert q.rows == 0
    # row stride larger than K
    Xb = synth.activations("llama2_70b", 33, 512, seed=9)
    big = torch.zeros(33, 640, dtype=torch.bfloat16, device="cuda")
    big[:, :512] = dev(Xb)
    q = w4.quantize_act(big[:, :512], w4.NVFP4, w4.SCALE_TOKEN)
    oc, osc, os2 = orc.quant_nvfp4(Xb, mode=1)
    np.testing.assert_array_equal(q.codes.cpu().numpy()[: 33 * 256].reshape(33, 256), oc)


def _gemm_case(orc, fmt, M, N, K, model="llama2_70b", a_mode=w4.SCALE_TOKEN, seed=0):
    Xa = synth.activations(model, M, K, seed=seed)
    Xw = synth.weights(model, N, K, seed=seed)
    A = w4.quantize_act(dev(Xa), fmt, a_mode)
    B = w4.quantize_weight(dev(Xw), fmt)
    Y = w4.gemm(A, B)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    if fmt == w4.NVFP4:
        ca, sa, s2a = orc.quant_nvfp4(Xa, mode=a_mode)
        cw, sw, s2w = orc.quant_nvfp4(Xw, mode=0)
        _, yref, absd = orc.gemm_nvfp4(ca, sa, s2a, a_mode, cw, sw, s2w)
    elif fmt == w4.MXFP4:
        ca, sa = orc.quant_mxfp4(Xa)
        cw, sw = orc.quant_mxfp4(Xw)
        _, yref, absd = orc.gemm_mxfp4(ca, sa, cw, sw)
    else:
        ca, sa = orc.quant_int4(Xa)
        cw, sw = orc.quant_int4(Xw)
        _, yref, absd = orc.gemm_int4(ca, sa, cw, sw)
    bad = H.gemm_violations(H.to_np_u16(Y), yref, absd)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outside tolerance, first at {np.argwhere(bad)[:5]}"
    return Y, yref


GEMM_SHAPES = [(16, 256, 256), (1, 128, 256), (9, 256, 640), (128, 256, 128), (200, 384, 640), (257, 512, 2048), (2304, 2304, 256),
               (130, 1024, 1024)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
@pytest.mark.parametrize("fmt", [w4.NVFP4, w4.MXFP4, w4.INT4])
def test_gemm_parity(orc, fmt, M, N, K):
    _gemm_case(orc, fmt, M, N, K)


def test_gemm_nvfp4_tensor_scales(orc):
    _gemm_case(orc, w4.NVFP4, 300, 512, 1024, model="swiglu300m", a_mode=w4.SCALE_TENSOR)


def test_gemm_textbook_exact(orc):
    """E2M1-grid operands, static s2 = 1: the GEMM is an exact integer matmul."""
    M, N, K = 130, 256, 512
    A = synth.e2m1_grid_values((M, K), 5, 1)
    B = synth.e2m1_grid_values((N, K), 5, 2)
    A[:, ::16] = 6.0
    B[:, 3::16] = -6.0
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    qa = w4.quantize_act(dev(synth.f32_to_bf16_bits(A)), w4.NVFP4, w4.SCALE_TENSOR, static_s2=one)
    qb = w4.QTensor(w4.NVFP4, N, K, w4.SCALE_TENSOR)
    w4.quantize_weight(dev(synth.f32_to_bf16_bits(B)), w4.NVFP4, out=qb)
    Y = w4.gemm(qa, qb)
    exact = (2 * A).astype(np.int64) @ (2 * B).astype(np.int64).T / 4.0
    yb = H.bf16_to_f64(H.to_np_u16(Y))
    assert np.all(np.abs(yb - exact) <= H.ulp_bf16(exact) * 0.5)


def _linear_ref(orc, fmt, Xa, Xw, a_mode, S=None):
    if fmt == w4.NVFP4:
        ca, sa, s2a = orc.quant_nvfp4(Xa, mode=a_mode)
        if S is not None:
            Kx = Xa.shape[1]
            rc, rs = orc.augment_nvfp4(Xa, S, ca, sa, s2a, a_mode)
            ca, sa = np.concatenate([ca, rc], 1), np.concatenate([sa, rs], 1)
            Xw = np.concatenate([Xw, Xw[:, S]], 1)
        cw, sw, s2w = orc.quant_nvfp4(Xw, mode=0)
        return orc.gemm_nvfp4(ca, sa, s2a, a_mode, cw, sw, s2w)
    if fmt == w4.MXFP4:
        ca, sa = orc.quant_mxfp4(Xa)
        cw, sw = orc.quant_mxfp4(Xw)
        return orc.gemm_mxfp4(ca, sa, cw, sw)
    ca, sa = orc.quant_int4(Xa)
    cw, sw = orc.quant_int4(Xw)
    return orc.gemm_int4(ca, sa, cw, sw)


@pytest.mark.parametrize("M", [1, 7, 16, 17, 300])
@pytest.mark.parametrize("fmt,mode", [(w4.NVFP4, w4.SCALE_TOKEN), (w4.NVFP4, w4.SCALE_TENSOR),
                                      (w4.MXFP4, 0), (w4.INT4, 0)])
def test_linear_parity(orc, fmt, mode, M):
    N, K = 384, 1280
    Xa = synth.activations("llama2_70b", M, K, seed=11)
    Xw = synth.weights("llama2_70b", N, K, seed=11)
    Wq = w4.quantize_weight(dev(Xw), fmt)
    Y = w4.linear(dev(Xa), Wq, mode)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _, yref, absd = _linear_ref(orc, fmt, Xa, Xw, mode)
    bad = H.gemm_violations(H.to_np_u16(Y), yref, absd)
    assert not bad.any(), f"{bad.sum()} bad of {bad.size}"


def test_select_channels_parity(orc):
    Xc = synth.calibration("qwen25_3b_aug", 2048, rows=512)
    S = w4.select_channels(dev(Xc), 256)
    np.testing.assert_array_equal(S.cpu().numpy(), orc.select_channels(Xc, 256))


@pytest.mark.parametrize("mode", [w4.SCALE_TOKEN, w4.SCALE_TENSOR])
def test_augment_parity(orc, mode):
    M, K, N, nS = 200, 1024, 256, 128
    Xa = synth.activations("qwen25_3b_aug", M, K, seed=5)
    Xw = synth.weights("qwen25_3b_aug", N, K, seed=5)
    S_np = orc.select_channels(synth.calibration("qwen25_3b_aug", K, rows=512), nS)
    S = torch.from_numpy(S_np).cuda()
    # two-call form: quantize into an augmented tensor, then the residual stage
    Xq = w4.quantize_act(dev(Xa), w4.NVFP4, mode, cols=K + nS)
    w4.augment_residual(dev(Xa), S, Xq)
    torch.cuda.synchronize()
    ca, sa, s2a = orc.quant_nvfp4(Xa, mode=mode)
    rc, rs = orc.augment_nvfp4(Xa, S_np, ca, sa, s2a, mode)
    codes = Xq.codes.cpu().numpy()[: M * (K + nS) // 2].reshape(M, (K + nS) // 2)
    np.testing.assert_array_equal(codes[:, : K // 2], ca)
    np.testing.assert_array_equal(codes[:, K // 2:], rc)
    sc = H.unswizzle_scales(Xq.scales.cpu().numpy(), M, K + nS, 16)
    np.testing.assert_array_equal(sc, np.concatenate([sa, rs], 1))
    # weights [W | W[:,S]] and the augmented GEMM, then the fused linear
    Wq = w4.quantize_weight(dev(Xw), w4.NVFP4, S=S)
    Y1 = w4.gemm(Xq, Wq)
    Y2 = w4.linear(dev(Xa), Wq, mode, S=S)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    _, yref, absd = _linear_ref(orc, w4.NVFP4, Xa, Xw, mode, S=S_np)
    for Y in (Y1, Y2):
        bad = H.gemm_violations(H.to_np_u16(Y), yref, absd)
        assert not bad.any(), f"{bad.sum()} bad"
    # the linear (whose per-token quantizer computes the residual stage in the
    # same launch) multiplies the same operands as the two-call path: the
    # same GEMM kernel gives the same bytes
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("M,K,nS,order", [(1, 1024, 128, "asc"), (37, 2048, 256, "asc"), (300, 2816, 384, "asc"),
                                           (5, 11008, 256, "asc"), (200, 2048, 256, "desc"),
                                           (130, 4096, 128, "perm"), (70, 4096, 256, "asc")])
def test_fused_residual_stage_matches_two_calls(orc, M, K, nS, order):
    """The fused linear's residual channels equal the separate second stage
    (w4a4_augment_residual after w4a4_quantize_act) bit for bit: the two
    paths' products agree byte for byte at every token count, on the
    decode, one-CTA and CTA-pair GEMMs, whatever the order of the channels."""
    N = 256
    Xa = synth.activations("qwen25_3b_aug", M, K, seed=17)
    Xw = synth.weights("qwen25_3b_aug", N, K, seed=17)
    S = w4.select_channels(dev(synth.calibration("qwen25_3b_aug", K, rows=512)), nS)
    if order == "desc":
        S = S.flip(0).contiguous()
    elif order == "perm":
        S = S[torch.from_numpy(np.random.default_rng(5).permutation(nS)).to(S.device)].contiguous()
    Wq = w4.quantize_weight(dev(Xw), w4.NVFP4, S=S)
    Xd = dev(Xa)
    Xq = w4.quantize_act(Xd, w4.NVFP4, w4.SCALE_TOKEN, cols=K + nS)
    w4.augment_residual(Xd, S, Xq)
    Y1 = w4.gemm(Xq, Wq)
    Y2 = w4.linear(Xd, Wq, w4.SCALE_TOKEN, S=S)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    if M > 16:  # same GEMM kernel on both paths (the decode variant has its own reduction order)
        assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    _, yref, absd = _linear_ref(orc, w4.NVFP4, Xa, Xw, w4.SCALE_TOKEN, S=S.cpu().numpy())
    for Y in (Y1, Y2):
        bad = H.gemm_violations(H.to_np_u16(Y), yref, absd)
        assert not bad.any(), f"{bad.sum()} bad"


@pytest.mark.parametrize("bad", [2048 + 5, -3])
def test_out_of_range_channel_is_channel_zero_and_reported(bad):
    """A channel index outside [0, K) in a device-side S is taken as channel 0
    and reported by w4a4_device_status as an invalid argument: the fused
    linear, the two-call path and the weight gather give exactly the bytes of
    the list with that index replaced by 0."""
    M, N, K, nS = 70, 256, 2048, 128
    Xd = dev(synth.activations("qwen25_3b_aug", M, K, seed=23))
    Wd = dev(synth.weights("qwen25_3b_aug", N, K, seed=23))
    S = w4.select_channels(dev(synth.calibration("qwen25_3b_aug", K, rows=512)), nS)
    S_bad = S.clone()
    S_bad[37] = bad
    S_fix = S.clone()
    S_fix[37] = 0
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    W_bad = w4.quantize_weight(Wd, w4.NVFP4, S=S_bad)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.ERR_INVALID_ARG
    W_fix = w4.quantize_weight(Wd, w4.NVFP4, S=S_fix)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    assert torch.equal(W_bad.codes, W_fix.codes) and torch.equal(W_bad.scales, W_fix.scales)
    Y_fix = w4.linear(Xd, W_fix, w4.SCALE_TOKEN, S=S_fix)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    Y_bad = w4.linear(Xd, W_fix, w4.SCALE_TOKEN, S=S_bad)  # fused second stage
    torch.cuda.synchronize()
    assert w4.device_status() == w4.ERR_INVALID_ARG
    assert torch.equal(Y_bad.view(torch.int16), Y_fix.view(torch.int16))
    Xq = w4.quantize_act(Xd, w4.NVFP4, w4.SCALE_TOKEN, cols=K + nS)
    w4.augment_residual(Xd, S_bad, Xq)  # the separate second stage
    torch.cuda.synchronize()
    assert w4.device_status() == w4.ERR_INVALID_ARG
    Xq2 = w4.quantize_act(Xd, w4.NVFP4, w4.SCALE_TOKEN, cols=K + nS)
    w4.augment_residual(Xd, S_fix, Xq2)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    assert torch.equal(Xq.codes, Xq2.codes) and torch.equal(Xq.scales, Xq2.scales)


def test_determinism_and_poisoned_output(orc):
    """Two runs give identical bytes; every output element is written (NaN poison)."""
    M, N, K = 300, 768, 1024
    Xa = dev(synth.activations("llama2_70b", M, K, seed=21))
    Wq = w4.quantize_weight(dev(synth.weights("llama2_70b", N, K, seed=21)), w4.NVFP4)
    for fmt in (w4.NVFP4,):
        Y1 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        Y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear(Xa, Wq, w4.SCALE_TOKEN, Y=Y1)
        w4.linear(Xa, Wq, w4.SCALE_TOKEN, Y=Y2)
        torch.cuda.synchronize()
        assert not torch.isnan(Y1).any()
        assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    for Mdec in (1, 16):
        Y1 = torch.full((Mdec, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear(Xa[:Mdec], Wq, w4.SCALE_TOKEN, Y=Y1)
        torch.cuda.synchronize()
        assert not torch.isnan(Y1).any()


def test_bounded_wait_reports_timeout(orc):
    """A k-tile that is never loaded makes the consumer's bounded wait expire:
    the kernel returns, the host reads W4A4_ERR_DEVICE_TIMEOUT, and the context
    stays usable for a correct GEMM afterwards."""
    M, N, K = 128, 256, 512
    Xa = synth.activations("llama2_70b", M, K, seed=2)
    Xw = synth.weights("llama2_70b", N, K, seed=2)
    A = w4.quantize_act(dev(Xa), w4.NVFP4, w4.SCALE_TOKEN)
    B = w4.quantize_weight(dev(Xw), w4.NVFP4)
    A2 = w4.quantize_act(dev(synth.activations("llama2_70b", 2 * M, K, seed=3)), w4.NVFP4, w4.SCALE_TOKEN)
    Ai = w4.quantize_act(dev(Xa), w4.INT4, 0)
    Bi = w4.quantize_weight(dev(Xw), w4.INT4)
    torch.cuda.synchronize()
    try:
        w4.debug_set(skip_k_tile=1, wait_limit_ns=200_000_000)
        w4.gemm(A, B)
        assert w4.device_status() == w4.ERR_DEVICE_TIMEOUT
        w4.gemm(Ai, Bi)
        assert w4.device_status() == w4.ERR_DEVICE_TIMEOUT
        w4.gemm(A2, B)  # M > 128: the CTA-pair kernel
        assert w4.device_status() == w4.ERR_DEVICE_TIMEOUT
    finally:
        w4.debug_set(-1, 0)
    Y = w4.gemm(A, B)
    assert w4.device_status() == w4.OK
    w4.gemm(A2, B)
    assert w4.device_status() == w4.OK
    ca, sa, s2a = orc.quant_nvfp4(Xa, mode=1)
    cw, sw, s2w = orc.quant_nvfp4(Xw, mode=0)
    _, yref, absd = orc.gemm_nvfp4(ca, sa, s2a, 1, cw, sw, s2w)
    assert not H.gemm_violations(H.to_np_u16(Y), yref, absd).any()


def test_abi_errors_on_gpu():
    X = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4A4Error) as e:
        w4.quantize_act(X[:, 1:129], w4.NVFP4, w4.SCALE_TOKEN)   # misaligned start
    assert e.value.status == w4.ERR_MISALIGNED
    Wq = w4.quantize_weight(torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda"), w4.NVFP4)
    with pytest.raises(w4.W4A4Error) as e:
        w4.linear(X, Wq, w4.SCALE_TOKEN, ws=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == w4.ERR_WORKSPACE


@pytest.mark.parametrize("fmt", [w4.NVFP4, w4.MXFP4, w4.INT4])
@pytest.mark.parametrize("N,K,nS", [(200, 1024, 128), (130, 2048, 256), (1, 384, 384)])
def test_weight_gather_bitexact(orc, fmt, N, K, nS):
    """w4a4_quantize_weight with channels S: [W | W[:, S]] quantized as one
    tensor of K + nS columns ("APEX4..." page, para 2: ARCQuant duplicates the
    weight columns of the augmented channels), bit for bit at ragged N.  The
    duplicated columns form blocks of their own, so their codes are compared
    against the oracle's quantization of the concatenated matrix, not copied
    from the first K columns."""
    Xw = synth.weights("qwen25_3b_aug", N, K, seed=11)
    S_np = np.sort(np.random.default_rng(7).choice(K, nS, replace=False)).astype(np.int32)
    S = torch.from_numpy(S_np).cuda()
    Wq = w4.quantize_weight(dev(Xw), fmt, S=S)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    cols = K + nS
    Wcat = np.ascontiguousarray(np.concatenate([Xw, Xw[:, S_np]], 1))
    codes = Wq.codes.cpu().numpy()[: N * cols // 2].reshape(N, cols // 2)
    if fmt == w4.NVFP4:
        oc, osc, os2 = orc.quant_nvfp4(Wcat, mode=0)
        np.testing.assert_array_equal(codes, oc)
        np.testing.assert_array_equal(H.unswizzle_scales(Wq.scales.cpu().numpy(), N, cols, 16), osc)
        assert np.float32(Wq.s2.cpu().numpy()[0]) == np.float32(os2[0])
        assert np.all(H.padding_scales(Wq.scales.cpu().numpy(), N, cols, 16) == 0)
    elif fmt == w4.MXFP4:
        oc, osc = orc.quant_mxfp4(Wcat)
        np.testing.assert_array_equal(codes, oc)
        np.testing.assert_array_equal(H.unswizzle_scales(Wq.scales.cpu().numpy(), N, cols, 32), osc)
    else:
        oc, osc = orc.quant_int4(Wcat)
        np.testing.assert_array_equal(codes, oc)
        sc = H.int4_scales(Wq.scales.cpu().numpy().view(np.float32), N, cols)
        np.testing.assert_array_equal(sc.view(np.uint32), osc.view(np.uint32))
