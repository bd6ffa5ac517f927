"""Host-side checks of the C-ABI library that need no GPU: it loads, exports
every entry point the header declares, and rejects bad arguments before
touching a device."""
import ctypes as C
import os
import re

import pytest

import w4a4_quantized_gemm_token_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a4.h")


@pytest.fixture(scope="module")
def L():
    from w4a4_quantized_gemm_token_b200 import build
    build.build()
    return w4.lib()


def declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|void|const char\*)\s+(w4a4_\w+)\s*\(", text, re.M)))


def test_header_lists_entry_points():
    names = declared()
    assert set(names) == set(w4.EXPORTS), names


def test_every_declared_symbol_exported(L):
    for name in declared():
        assert hasattr(L, name), name


def test_status_strings(L):
    assert w4.status_string(w4.OK) == "ok"
    assert "timed out" in w4.status_string(w4.ERR_DEVICE_TIMEOUT)
    assert w4.status_string(99) == "unknown status"


def test_qtensor_bytes(L):
    c, s, t = w4.qtensor_bytes(w4.NVFP4, 200, 1024, w4.SCALE_TOKEN)
    assert (c, s, t) == (200 * 512, 256 * 64, 800)
    c, s, t = w4.qtensor_bytes(w4.NVFP4, 200, 1024, w4.SCALE_TENSOR)
    assert t == 16  # the scale and three scratch words
    c, s, t = w4.qtensor_bytes(w4.MXFP4, 1, 256, 0)
    assert (c, s, t) == (128, 128 * 8, 0)
    c, s, t = w4.qtensor_bytes(w4.INT4, 130, 384, 0)
    assert (c, s, t) == (130 * 192, 3 * 256 * 4, 0)
    with pytest.raises(w4.W4A4Error):
        w4.qtensor_bytes(w4.NVFP4, 4, 100, 0)
    with pytest.raises(w4.W4A4Error):
        w4.qtensor_bytes(7, 4, 128, 0)


def test_workspace_sizes(L):
    assert w4.linear_workspace(4096, 10240, 8192, w4.NVFP4) >= 4096 * 4096 + 4096 * 512
    assert w4.linear_workspace(16, 10240, 8192, w4.NVFP4) >= 16 * 10240 * 4
    assert w4.linear_workspace(16, 100, 8192, w4.NVFP4) == 0        # N not a multiple of 128
    assert w4.linear_workspace(16, 256, 8192, w4.NVFP4, 100) == 0   # nS not a multiple of 128


def _qt(fmt, rows, cols, mode=0, codes=16, scales=16, s2=16):
    return w4.QTensorStruct(fmt, rows, cols, w4.GROUP[fmt], mode, 0, codes, scales, s2)


def test_argument_errors_before_any_device_work(L):
    q = _qt(w4.NVFP4, 4, 256, w4.SCALE_TOKEN)
    ref = C.byref(q)
    # bad K, bad group, bad format, rows mismatch: all rejected on the host
    assert L.w4a4_quantize_act(C.c_void_p(16), 4, 100, 128, 0, 16, 1, None, ref, None) == w4.ERR_INVALID_ARG
    assert L.w4a4_quantize_act(C.c_void_p(16), 4, 256, 256, 0, 32, 1, None, ref, None) == w4.ERR_INVALID_ARG
    assert L.w4a4_quantize_act(C.c_void_p(16), 5, 256, 256, 0, 16, 1, None, ref, None) == w4.ERR_INVALID_ARG
    assert L.w4a4_quantize_act(C.c_void_p(16), 4, 256, 200, 0, 16, 1, None, ref, None) == w4.ERR_INVALID_ARG
    # misaligned X
    assert L.w4a4_quantize_act(C.c_void_p(18), 4, 256, 256, 0, 16, 1, None, ref, None) == w4.ERR_MISALIGNED
    # M == 0 is a no-op
    q0 = _qt(w4.NVFP4, 0, 256, w4.SCALE_TOKEN)
    assert L.w4a4_quantize_act(None, 0, 256, 256, 0, 16, 1, None, C.byref(q0), None) == w4.OK
    # gemm: format mismatch, K mismatch, N not a multiple of 128
    a = _qt(w4.NVFP4, 4, 256, w4.SCALE_TOKEN)
    b = _qt(w4.MXFP4, 256, 256)
    assert L.w4a4_gemm(C.byref(a), C.byref(b), C.c_void_p(16), 256, None) == w4.ERR_INVALID_ARG
    b = _qt(w4.NVFP4, 256, 512, w4.SCALE_TENSOR)
    assert L.w4a4_gemm(C.byref(a), C.byref(b), C.c_void_p(16), 256, None) == w4.ERR_INVALID_ARG
    b = _qt(w4.NVFP4, 200, 256, w4.SCALE_TENSOR)
    assert L.w4a4_gemm(C.byref(a), C.byref(b), C.c_void_p(16), 256, None) == w4.ERR_INVALID_ARG
    # NVFP4 weights with one scale per row need those scales 16-byte aligned
    b = _qt(w4.NVFP4, 256, 256, w4.SCALE_TOKEN, s2=20)
    assert L.w4a4_gemm(C.byref(a), C.byref(b), C.c_void_p(16), 256, None) == w4.ERR_MISALIGNED
    # linear: workspace too small, residual channels with a non-NVFP4 weight
    W = _qt(w4.NVFP4, 256, 256, w4.SCALE_TENSOR)
    assert L.w4a4_linear(C.c_void_p(16), 4, 256, 256, C.byref(W), 1, None, 0, C.c_void_p(16), 256,
                         C.c_void_p(256), 16, None) == w4.ERR_WORKSPACE
    Wm = _qt(w4.MXFP4, 256, 384)
    assert L.w4a4_linear(C.c_void_p(16), 4, 256, 256, C.byref(Wm), 1, C.c_void_p(16), 128, C.c_void_p(16), 256,
                         C.c_void_p(256), 1 << 20, None) == w4.ERR_INVALID_ARG
    # the static-scratch linear: sizes beyond its scratch, null weights
    Wbig = _qt(w4.NVFP4, 1024, 8192, w4.SCALE_TENSOR)
    assert L.w4a4_linear_noalloc(C.c_void_p(16), 4096, 8192, 8192, C.byref(Wbig), 1, None, 0, C.c_void_p(16),
                                 1024, None) == w4.ERR_WORKSPACE
    assert L.w4a4_linear_noalloc(C.c_void_p(16), 4, 256, 256, None, 1, None, 0, C.c_void_p(16), 256,
                                 None) == w4.ERR_INVALID_ARG
    # S with nS not a multiple of 128
    assert L.w4a4_augment_residual(C.c_void_p(16), 4, 256, 256, C.c_void_p(16), 64, ref, None) == w4.ERR_INVALID_ARG
    # channel selection: workspace too small
    assert L.w4a4_select_channels(C.c_void_p(16), 4, 256, 256, 16, C.c_void_p(16), C.c_void_p(16), 8,
                                  None) == w4.ERR_WORKSPACE


def test_no_device_means_error_not_fallback(L):
    """With valid arguments but no usable GPU the library reports an error
    instead of computing anything on the host."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    q = _qt(w4.NVFP4, 4, 256, w4.SCALE_TOKEN)
    rc = L.w4a4_quantize_act(C.c_void_p(16), 4, 256, 256, 0, 16, 1, None, C.byref(q), None)
    assert rc in (w4.ERR_CUDA, w4.ERR_ARCH)


def test_segment_weight_arguments(L):
    """Per-segment weight scales: the segment list, the output's scale mode and
    the alignment of its per-row scales are checked on the host."""
    def seg_call(seg, out, N=512, K=256, S=None, nS=0):
        arr = (C.c_int32 * len(seg))(*seg)
        return L.w4a4_quantize_weight_segments(C.c_void_p(16), N, K, K, arr, len(seg) - 1, S, nS,
                                               C.byref(out), None)
    out = _qt(w4.NVFP4, 512, 256, w4.SCALE_TOKEN)
    for bad in ([0, 256, 256, 512],   # empty segment
                [0, 200, 512],        # boundary not a multiple of 128
                [0, 256, 384],        # does not end at N
                [128, 512],           # does not start at 0
                [0],                  # no segment
                [0, 384, 256, 512]):  # not ascending
        assert seg_call(bad, out) == w4.ERR_INVALID_ARG, bad
    # the output must be NVFP4 with one s2 per row
    assert seg_call([0, 512], _qt(w4.NVFP4, 512, 256, w4.SCALE_TENSOR)) == w4.ERR_INVALID_ARG
    assert seg_call([0, 512], _qt(w4.MXFP4, 512, 256)) == w4.ERR_INVALID_ARG
    assert seg_call([0, 512], _qt(w4.NVFP4, 512, 256, w4.SCALE_TOKEN, s2=20)) == w4.ERR_MISALIGNED
    # residual channels: cols must be K + nS, nS a multiple of 128
    assert seg_call([0, 512], out, S=C.c_void_p(16), nS=128) == w4.ERR_INVALID_ARG
    aug = _qt(w4.NVFP4, 512, 384, w4.SCALE_TOKEN)
    assert seg_call([0, 512], aug, S=C.c_void_p(16), nS=64) == w4.ERR_INVALID_ARG


def test_msd_arguments(L):
    """Multi-pass MXFP4: pass count, output format and width are checked on the host."""
    out = _qt(w4.MXFP4, 4, 512)
    X = C.c_void_p(16)
    assert L.w4a4_quantize_act_msd(X, 4, 256, 256, 0, C.byref(out), None) == w4.ERR_INVALID_ARG   # passes < 1
    assert L.w4a4_quantize_act_msd(X, 4, 256, 256, 5, C.byref(out), None) == w4.ERR_INVALID_ARG   # passes > 4
    assert L.w4a4_quantize_act_msd(X, 4, 256, 256, 3, C.byref(out), None) == w4.ERR_INVALID_ARG   # cols != 3K
    nv = _qt(w4.NVFP4, 4, 512, w4.SCALE_TOKEN)
    assert L.w4a4_quantize_act_msd(X, 4, 256, 256, 2, C.byref(nv), None) == w4.ERR_INVALID_ARG    # not MXFP4
    assert L.w4a4_quantize_act_msd(C.c_void_p(18), 4, 256, 256, 2, C.byref(out), None) == w4.ERR_MISALIGNED
    W = _qt(w4.MXFP4, 256, 512)
    assert L.w4a4_quantize_weight_msd(X, 256, 256, 256, 3, C.byref(W), None) == w4.ERR_INVALID_ARG
    assert L.w4a4_linear_msd(X, 4, 256, 256, C.byref(W), 3, C.c_void_p(16), 256, C.c_void_p(256), 1 << 20,
                             None) == w4.ERR_INVALID_ARG
    assert L.w4a4_linear_msd(X, 4, 256, 256, C.byref(W), 2, C.c_void_p(16), 256, C.c_void_p(256), 16,
                             None) == w4.ERR_WORKSPACE


def test_hadamard_flag_arguments(L):
    """The rotation flag: unknown bits rejected; operands must agree; no
    rotation with residual channels or the multi-pass decomposition."""
    X = C.c_void_p(16)
    bad = _qt(w4.NVFP4, 4, 256, w4.SCALE_TOKEN)
    bad.flags = 2
    assert L.w4a4_quantize_act(X, 4, 256, 256, 0, 16, 1, None, C.byref(bad), None) == w4.ERR_INVALID_ARG
    a = _qt(w4.NVFP4, 4, 256, w4.SCALE_TOKEN)
    a.flags = w4.FLAG_HADAMARD
    b = _qt(w4.NVFP4, 256, 256, w4.SCALE_TENSOR)
    assert L.w4a4_gemm(C.byref(a), C.byref(b), C.c_void_p(16), 256, None) == w4.ERR_INVALID_ARG
    Wr = _qt(w4.NVFP4, 256, 384, w4.SCALE_TENSOR)
    Wr.flags = w4.FLAG_HADAMARD
    assert L.w4a4_quantize_weight(X, 256, 256, 256, 0, 16, C.c_void_p(16), 128, C.byref(Wr), None) == w4.ERR_INVALID_ARG
    assert L.w4a4_linear(X, 4, 256, 256, C.byref(Wr), 1, C.c_void_p(16), 128, C.c_void_p(16), 256,
                         C.c_void_p(256), 1 << 20, None) == w4.ERR_INVALID_ARG
    m = _qt(w4.MXFP4, 4, 512)
    m.flags = w4.FLAG_HADAMARD
    assert L.w4a4_quantize_act_msd(X, 4, 256, 256, 2, C.byref(m), None) == w4.ERR_INVALID_ARG


def test_int4_group_choice_and_checks(L):
    """rho-aware INT4 group size: 128 up to rho = 16, doubled per doubling, at
    most 512; groups other than 128/256/512, or not dividing K, are rejected."""
    assert [w4.int4_group_for_rho(r) for r in (0, 8, 16, 17, 32, 33, 60, 64, 1000)] == \
        [128, 128, 128, 256, 256, 512, 512, 512, 512]
    X = C.c_void_p(16)
    q = _qt(w4.INT4, 4, 1024)
    q.group = 384
    assert L.w4a4_quantize_act(X, 4, 1024, 1024, w4.INT4, 384, 0, None, C.byref(q), None) == w4.ERR_INVALID_ARG
    q = _qt(w4.INT4, 4, 384)
    q.group = 256
    assert L.w4a4_quantize_act(X, 4, 384, 384, w4.INT4, 256, 0, None, C.byref(q), None) == w4.ERR_INVALID_ARG
    a = _qt(w4.INT4, 4, 1024)
    a.group = 512
    b = _qt(w4.INT4, 256, 1024)
    assert L.w4a4_gemm(C.byref(a), C.byref(b), C.c_void_p(16), 256, None) == w4.ERR_INVALID_ARG  # groups differ


def test_noalloc_scratch_size_matches_header():
    """The binding's copy of the no-alloc scratch size is the header's."""
    import re
    hdr = open(os.path.join(ROOT, "include", "w4a4.h")).read()
    m = re.search(r"#define\s+W4A4_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", hdr)
    assert m, "W4A4_NOALLOC_SCRATCH_BYTES not found"
    import w4a4_quantized_gemm_token_b200 as w4
    assert w4.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
