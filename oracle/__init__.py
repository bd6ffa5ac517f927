"""Python access to the C oracle (oracle.c) through ctypes.

TEST INFRASTRUCTURE ONLY.  The oracle is the plain CPU restatement of the
W4A4 quantized linear layer that the GPU library is checked against.  Only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this module; the library package never does.

All arrays are numpy arrays; bf16 tensors travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc) when it is missing or stale."""
    stale = (not os.path.exists(_LIB) or
             os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _declare(_lib)
    return _lib


_u8p = C.POINTER(C.c_uint8)
_u16p = C.POINTER(C.c_uint16)
_i32p = C.POINTER(C.c_int32)
_f32p = C.POINTER(C.c_float)
_f64p = C.POINTER(C.c_double)


def _declare(L):
    L.orc_e2m1_encode.argtypes = [C.c_float]; L.orc_e2m1_encode.restype = C.c_uint8
    L.orc_e2m1_decode.argtypes = [C.c_uint8]; L.orc_e2m1_decode.restype = C.c_float
    L.orc_e4m3_encode.argtypes = [C.c_float]; L.orc_e4m3_encode.restype = C.c_uint8
    L.orc_e4m3_decode.argtypes = [C.c_uint8]; L.orc_e4m3_decode.restype = C.c_float
    L.orc_e8m0_decode.argtypes = [C.c_uint8]; L.orc_e8m0_decode.restype = C.c_float
    L.orc_floor_log2.argtypes = [C.c_float]; L.orc_floor_log2.restype = C.c_int
    L.orc_bf16_to_f32.argtypes = [C.c_uint16]; L.orc_bf16_to_f32.restype = C.c_float
    L.orc_f64_to_bf16.argtypes = [C.c_double]; L.orc_f64_to_bf16.restype = C.c_uint16
    L.orc_nvfp4_s2_from_amax.argtypes = [C.c_float]; L.orc_nvfp4_s2_from_amax.restype = C.c_float
    L.orc_quant_nvfp4.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, C.c_int, _f32p, _u8p, _u8p, _f32p]
    L.orc_quant_nvfp4_segments.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, _i32p, C.c_int, _u8p, _u8p, _f32p]
    L.orc_gemm_nvfp4_wrows.argtypes = [_u8p, _u8p, _f32p, C.c_int, _u8p, _u8p, _f32p, C.c_int,
                                       C.c_int, C.c_int, C.c_int, _u16p, _f64p, _f64p]
    L.orc_quant_mxfp4.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, _u8p, _u8p]
    L.orc_quant_mxfp4_msd.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, C.c_int, _u8p, _u8p]
    L.orc_rotate_blocks.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, _f32p]
    L.orc_quant_nvfp4_f32.argtypes = [_f32p, C.c_int, C.c_int, C.c_int, _u8p, _u8p, _f32p]
    L.orc_quant_mxfp4_f32.argtypes = [_f32p, C.c_int, C.c_int, _u8p, _u8p]
    L.orc_quant_int4_f32.argtypes = [_f32p, C.c_int, C.c_int, _u8p, _f32p]
    L.orc_quant_int4_g.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, C.c_int, _u8p, _f32p]
    L.orc_quant_int4_f32_g.argtypes = [_f32p, C.c_int, C.c_int, C.c_int, _u8p, _f32p]
    L.orc_gemm_int4_g.argtypes = [_u8p, _f32p, _u8p, _f32p, C.c_int, C.c_int, C.c_int, C.c_int, _u16p, _f64p, _f64p]
    L.orc_quant_int4.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, _u8p, _f32p]
    L.orc_dequant_nvfp4.argtypes = [_u8p, _u8p, _f32p, C.c_int, C.c_int, C.c_int, _f64p]
    L.orc_dequant_mxfp4.argtypes = [_u8p, _u8p, C.c_int, C.c_int, _f64p]
    L.orc_dequant_int4.argtypes = [_u8p, _f32p, C.c_int, C.c_int, _f64p]
    L.orc_gemm_nvfp4.argtypes = [_u8p, _u8p, _f32p, C.c_int, _u8p, _u8p, _f32p,
                                 C.c_int, C.c_int, C.c_int, _u16p, _f64p, _f64p]
    L.orc_gemm_mxfp4.argtypes = [_u8p, _u8p, _u8p, _u8p, C.c_int, C.c_int, C.c_int, _u16p, _f64p, _f64p]
    L.orc_gemm_int4.argtypes = [_u8p, _f32p, _u8p, _f32p, C.c_int, C.c_int, C.c_int, _u16p, _f64p, _f64p]
    L.orc_augment_nvfp4.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, _i32p, C.c_int,
                                    _u8p, _u8p, _f32p, C.c_int, _u8p, _u8p]
    L.orc_select_channels.argtypes = [_u16p, C.c_int, C.c_int, C.c_int, _i32p]
    for name in ("orc_quant_nvfp4", "orc_quant_mxfp4", "orc_quant_int4", "orc_gemm_nvfp4",
                 "orc_gemm_mxfp4", "orc_gemm_int4", "orc_augment_nvfp4", "orc_select_channels"):
        getattr(L, name).restype = C.c_int


def _p(a, ptr_t):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ptr_t)


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"oracle {name} rejected its arguments (rc={rc})")


def _bf16(x):
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16, "bf16 tensors are passed as uint16 bit patterns"
    return x


# ---- scalar helpers (vectorised by a python loop; small inputs only) -------
def e2m1_encode(v: float) -> int:
    return int(lib().orc_e2m1_encode(float(v)))


def e2m1_decode(c: int) -> float:
    return float(lib().orc_e2m1_decode(int(c)))


def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_decode(c: int) -> float:
    return float(lib().orc_e4m3_decode(int(c)))


def e8m0_decode(c: int) -> float:
    return float(lib().orc_e8m0_decode(int(c)))


def floor_log2(a: float) -> int:
    return int(lib().orc_floor_log2(float(a)))


def f64_to_bf16(v: float) -> int:
    return int(lib().orc_f64_to_bf16(float(v)))


def nvfp4_s2_from_amax(a: float) -> float:
    return float(lib().orc_nvfp4_s2_from_amax(float(a)))


# ---- quantizers -------------------------------------------------------------
def quant_nvfp4(X, mode: int, static_s2=None):
    """X: uint16 [M, K] bf16 bits.  mode 0 = tensor scale, 1 = per-token scale.
    Returns (codes [M, K/2] u8, scales [M, K/16] u8 (E4M3), s2 f32 [1] or [M])."""
    X = _bf16(X)
    M, K = X.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 16), np.uint8)
    s2 = np.zeros(M if mode == 1 else 1, np.float32)
    ss = None if static_s2 is None else np.ascontiguousarray(static_s2, np.float32)
    _check(lib().orc_quant_nvfp4(_p(X, _u16p), M, K, K, mode, _p(ss, _f32p), _p(codes, _u8p),
                                 _p(scales, _u8p), _p(s2, _f32p)), "quant_nvfp4")
    return codes, scales, s2


def quant_nvfp4_segments(X, seg):
    """Row segments [seg[i], seg[i+1]) quantized as separate NVFP4 tensors.
    Returns (codes, scales, s2 per row [M])."""
    X = _bf16(X)
    M, K = X.shape
    seg = np.ascontiguousarray(seg, np.int32)
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 16), np.uint8)
    s2 = np.zeros(M, np.float32)
    _check(lib().orc_quant_nvfp4_segments(_p(X, _u16p), M, K, K, _p(seg, _i32p), len(seg) - 1, _p(codes, _u8p),
                                          _p(scales, _u8p), _p(s2, _f32p)), "quant_nvfp4_segments")
    return codes, scales, s2


def quant_mxfp4(X):
    """Returns (codes [M, K/2] u8, scales [M, K/32] u8 (E8M0))."""
    X = _bf16(X)
    M, K = X.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 32), np.uint8)
    _check(lib().orc_quant_mxfp4(_p(X, _u16p), M, K, K, _p(codes, _u8p), _p(scales, _u8p)),
           "quant_mxfp4")
    return codes, scales


def quant_mxfp4_msd(X, passes=2):
    """Multi-pass MXFP4: pass p quantizes the residual of passes 0..p-1 into
    columns [p*K, (p+1)*K).  Returns (codes [M, passes*K/2], scales
    [M, passes*K/32])."""
    X = _bf16(X)
    M, K = X.shape
    codes = np.zeros((M, passes * K // 2), np.uint8)
    scales = np.zeros((M, passes * K // 32), np.uint8)
    _check(lib().orc_quant_mxfp4_msd(_p(X, _u16p), M, K, K, passes, _p(codes, _u8p), _p(scales, _u8p)),
           "quant_mxfp4_msd")
    return codes, scales


def rotate_blocks(X, n, act_side):
    """Block-local Walsh-Hadamard rotation (FP32 butterflies) of bf16 X, blocks
    of n along K; times 1/n on the activation side.  Returns float32 [M, K]."""
    X = _bf16(X)
    M, K = X.shape
    out = np.zeros((M, K), np.float32)
    _check(lib().orc_rotate_blocks(_p(X, _u16p), M, K, K, n, 1 if act_side else 0, _p(out, _f32p)), "rotate_blocks")
    return out


def quant_nvfp4_f32(Xf, mode=1):
    Xf = np.ascontiguousarray(Xf, np.float32)
    M, K = Xf.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 16), np.uint8)
    s2 = np.zeros(max(M, 1) if mode == 1 else 1, np.float32)
    _check(lib().orc_quant_nvfp4_f32(_p(Xf, _f32p), M, K, mode, _p(codes, _u8p), _p(scales, _u8p), _p(s2, _f32p)),
           "quant_nvfp4_f32")
    return codes, scales, s2


def quant_mxfp4_f32(Xf):
    Xf = np.ascontiguousarray(Xf, np.float32)
    M, K = Xf.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 32), np.uint8)
    _check(lib().orc_quant_mxfp4_f32(_p(Xf, _f32p), M, K, _p(codes, _u8p), _p(scales, _u8p)), "quant_mxfp4_f32")
    return codes, scales


def quant_int4_f32(Xf):
    Xf = np.ascontiguousarray(Xf, np.float32)
    M, K = Xf.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 128), np.float32)
    _check(lib().orc_quant_int4_f32(_p(Xf, _f32p), M, K, _p(codes, _u8p), _p(scales, _f32p)), "quant_int4_f32")
    return codes, scales


def quant_int4_g(X, G):
    """INT4 with groups of G elements: (codes [M, K/2], scales [M, K/G] f32)."""
    X = _bf16(X)
    M, K = X.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // G), np.float32)
    _check(lib().orc_quant_int4_g(_p(X, _u16p), M, K, K, G, _p(codes, _u8p), _p(scales, _f32p)), "quant_int4_g")
    return codes, scales


def quant_int4_f32_g(Xf, G):
    Xf = np.ascontiguousarray(Xf, np.float32)
    M, K = Xf.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // G), np.float32)
    _check(lib().orc_quant_int4_f32_g(_p(Xf, _f32p), M, K, G, _p(codes, _u8p), _p(scales, _f32p)), "quant_int4_f32_g")
    return codes, scales


def gemm_int4_g(ca, sa, cw, sw, G, want_ref=True):
    M, K = ca.shape[0], ca.shape[1] * 2
    N = cw.shape[0]
    Y, yref, absd = _gemm_out(M, N, want_ref)
    c = np.ascontiguousarray
    _check(lib().orc_gemm_int4_g(_p(c(ca), _u8p), _p(c(sa, np.float32), _f32p), _p(c(cw), _u8p),
                                 _p(c(sw, np.float32), _f32p), M, N, K, G, _p(Y, _u16p), _p(yref, _f64p),
                                 _p(absd, _f64p)), "gemm_int4_g")
    return Y, yref, absd


def quant_int4(X):
    """Returns (codes [M, K/2] u8 two's-complement nibbles, scales [M, K/128] f32)."""
    X = _bf16(X)
    M, K = X.shape
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 128), np.float32)
    _check(lib().orc_quant_int4(_p(X, _u16p), M, K, K, _p(codes, _u8p), _p(scales, _f32p)),
           "quant_int4")
    return codes, scales


def dequant_nvfp4(codes, scales, s2, mode):
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((M, K), np.float64)
    lib().orc_dequant_nvfp4(_p(np.ascontiguousarray(codes), _u8p), _p(np.ascontiguousarray(scales), _u8p),
                            _p(np.ascontiguousarray(s2, np.float32), _f32p), mode, M, K, _p(out, _f64p))
    return out


def dequant_mxfp4(codes, scales):
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((M, K), np.float64)
    lib().orc_dequant_mxfp4(_p(np.ascontiguousarray(codes), _u8p), _p(np.ascontiguousarray(scales), _u8p),
                            M, K, _p(out, _f64p))
    return out


def dequant_int4(codes, scales):
    M, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((M, K), np.float64)
    lib().orc_dequant_int4(_p(np.ascontiguousarray(codes), _u8p),
                           _p(np.ascontiguousarray(scales, np.float32), _f32p), M, K, _p(out, _f64p))
    return out


# ---- GEMM references --------------------------------------------------------
def _gemm_out(M, N, want_ref):
    Y = np.zeros((M, N), np.uint16)
    yref = np.zeros((M, N), np.float64) if want_ref else None
    absd = np.zeros((M, N), np.float64) if want_ref else None
    return Y, yref, absd


def gemm_nvfp4(ca, sa, s2a, a_mode, cw, sw, s2w, want_ref=True):
    """Returns (Y bf16 bits [M,N], exact value [M,N], |alpha|*sum|a w| [M,N]).
    s2w: one weight scale ([1]) or one per output row ([N])."""
    M, K = ca.shape[0], ca.shape[1] * 2
    N = cw.shape[0]
    Y, yref, absd = _gemm_out(M, N, want_ref)
    c = np.ascontiguousarray
    s2w = c(s2w, np.float32)
    w_mode = 1 if s2w.size == N and N > 1 else 0
    _check(lib().orc_gemm_nvfp4_wrows(_p(c(ca), _u8p), _p(c(sa), _u8p), _p(c(s2a, np.float32), _f32p), a_mode,
                                      _p(c(cw), _u8p), _p(c(sw), _u8p), _p(s2w, _f32p), w_mode,
                                      M, N, K, _p(Y, _u16p), _p(yref, _f64p), _p(absd, _f64p)), "gemm_nvfp4")
    return Y, yref, absd


def gemm_mxfp4(ca, sa, cw, sw, want_ref=True):
    M, K = ca.shape[0], ca.shape[1] * 2
    N = cw.shape[0]
    Y, yref, absd = _gemm_out(M, N, want_ref)
    c = np.ascontiguousarray
    _check(lib().orc_gemm_mxfp4(_p(c(ca), _u8p), _p(c(sa), _u8p), _p(c(cw), _u8p), _p(c(sw), _u8p),
                                M, N, K, _p(Y, _u16p), _p(yref, _f64p), _p(absd, _f64p)), "gemm_mxfp4")
    return Y, yref, absd


def gemm_int4(ca, sa, cw, sw, want_ref=True):
    M, K = ca.shape[0], ca.shape[1] * 2
    N = cw.shape[0]
    Y, yref, absd = _gemm_out(M, N, want_ref)
    c = np.ascontiguousarray
    _check(lib().orc_gemm_int4(_p(c(ca), _u8p), _p(c(sa, np.float32), _f32p), _p(c(cw), _u8p),
                               _p(c(sw, np.float32), _f32p), M, N, K, _p(Y, _u16p), _p(yref, _f64p),
                               _p(absd, _f64p)), "gemm_int4")
    return Y, yref, absd


# ---- augmentation -----------------------------------------------------------
def augment_nvfp4(X, S, codes, scales, s2, mode):
    """Second stage of the dual-stage NVFP4 quantization.
    Returns (rcodes [M, nS/2], rscales [M, nS/16])."""
    X = _bf16(X)
    M, K = X.shape
    S = np.ascontiguousarray(S, np.int32)
    nS = S.shape[0]
    rc = np.zeros((M, nS // 2), np.uint8)
    rs = np.zeros((M, nS // 16), np.uint8)
    c = np.ascontiguousarray
    _check(lib().orc_augment_nvfp4(_p(X, _u16p), M, K, K, _p(S, _i32p), nS, _p(c(codes), _u8p),
                                   _p(c(scales), _u8p), _p(c(s2, np.float32), _f32p), mode,
                                   _p(rc, _u8p), _p(rs, _u8p)), "augment_nvfp4")
    return rc, rs


def select_channels(Xcal, nS):
    Xcal = _bf16(Xcal)
    Mc, K = Xcal.shape
    S = np.zeros(nS, np.int32)
    _check(lib().orc_select_channels(_p(Xcal, _u16p), Mc, K, nS, _p(S, _i32p)), "select_channels")
    return S
