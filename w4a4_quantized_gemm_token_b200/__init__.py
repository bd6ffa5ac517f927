"""B200 (sm_100a) W4A4 quantized linear layer: Python binding of lib/libw4a4.so.

Argument marshalling only: every step (quantization, GEMM, augmentation,
channel selection) runs in the library's CUDA kernels; PyTorch provides the
device memory and the current stream.  There is no CPU path: when the shared
library is missing, importing the functions below raises.

Formats: NVFP4 (E2M1 + E4M3 per 16 + FP32 second-level scale), MXFP4
(E2M1 + E8M0 per 32), INT4 (two's complement, FP32 scale amax/7 per 128).
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "lib", "libw4a4.so")

NVFP4, MXFP4, INT4 = 0, 1, 2
GROUP = {NVFP4: 16, MXFP4: 32, INT4: 128}
SCALE_TENSOR, SCALE_TOKEN = 0, 1
FLAG_HADAMARD = 1  # blocks rotated by a Walsh-Hadamard matrix before quantization

OK, ERR_INVALID_ARG, ERR_MISALIGNED, ERR_WORKSPACE, ERR_ARCH, ERR_CUDA, ERR_DEVICE_TIMEOUT = range(7)

# every entry point declared in include/w4a4.h
EXPORTS = ("w4a4_qtensor_bytes", "w4a4_quantize_act", "w4a4_quantize_weight", "w4a4_gemm",
           "w4a4_linear_workspace", "w4a4_linear", "w4a4_augment_residual", "w4a4_select_channels",
           "w4a4_device_status", "w4a4_debug_set", "w4a4_status_string", "w4a4_linear_noalloc",
           "w4a4_quantize_weight_segments", "w4a4_quantize_act_msd", "w4a4_quantize_weight_msd",
           "w4a4_linear_msd", "w4a4_int4_group_for_rho")


class W4A4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class QTensorStruct(C.Structure):
    _fields_ = [("format", C.c_int32), ("rows", C.c_int32), ("cols", C.c_int32), ("group", C.c_int32),
                ("scale_mode", C.c_int32), ("flags", C.c_int32), ("codes", C.c_void_p),
                ("scales", C.c_void_p), ("s2", C.c_void_p)]


_lib = None


def lib():
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"W4A4 CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m w4a4_quantized_gemm_token_b200.build)")
        L = C.CDLL(LIB_PATH)
        vp, i, sz = C.c_void_p, C.c_int, C.c_size_t
        qp = C.POINTER(QTensorStruct)
        L.w4a4_qtensor_bytes.argtypes = [i, i, i, i, C.POINTER(sz), C.POINTER(sz), C.POINTER(sz)]
        L.w4a4_quantize_act.argtypes = [vp, i, i, i, i, i, i, vp, qp, vp]
        L.w4a4_quantize_weight.argtypes = [vp, i, i, i, i, i, vp, i, qp, vp]
        L.w4a4_quantize_weight_segments.argtypes = [vp, i, i, i, C.POINTER(C.c_int32), i, vp, i, qp, vp]
        L.w4a4_gemm.argtypes = [qp, qp, vp, i, vp]
        L.w4a4_int4_group_for_rho.argtypes = [C.c_double]
        L.w4a4_quantize_act_msd.argtypes = [vp, i, i, i, i, qp, vp]
        L.w4a4_quantize_weight_msd.argtypes = [vp, i, i, i, i, qp, vp]
        L.w4a4_linear_msd.argtypes = [vp, i, i, i, qp, i, vp, i, vp, sz, vp]
        L.w4a4_linear_workspace.argtypes = [i, i, i, i, i]
        L.w4a4_linear_workspace.restype = sz
        L.w4a4_linear.argtypes = [vp, i, i, i, qp, i, vp, i, vp, i, vp, sz, vp]
        L.w4a4_linear_noalloc.argtypes = [vp, i, i, i, qp, i, vp, i, vp, i, vp]
        L.w4a4_augment_residual.argtypes = [vp, i, i, i, vp, i, qp, vp]
        L.w4a4_select_channels.argtypes = [vp, i, i, i, i, vp, vp, sz, vp]
        L.w4a4_device_status.argtypes = [vp]
        L.w4a4_debug_set.argtypes = [i, C.c_ulonglong]
        L.w4a4_debug_set.restype = None
        L.w4a4_status_string.argtypes = [i]
        L.w4a4_status_string.restype = C.c_char_p
        for name in ("w4a4_qtensor_bytes", "w4a4_quantize_act", "w4a4_quantize_weight", "w4a4_gemm",
                     "w4a4_linear", "w4a4_augment_residual", "w4a4_select_channels", "w4a4_device_status",
                     "w4a4_linear_noalloc", "w4a4_quantize_weight_segments", "w4a4_quantize_act_msd",
                     "w4a4_quantize_weight_msd", "w4a4_linear_msd", "w4a4_int4_group_for_rho"):
            getattr(L, name).restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().w4a4_status_string(int(status)).decode()


def _check(rc: int, where: str):
    if rc != OK:
        raise W4A4Error(rc, where)


def _stream():
    import torch
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def qtensor_bytes(fmt: int, rows: int, cols: int, scale_mode: int = SCALE_TENSOR):
    c, s, t = C.c_size_t(), C.c_size_t(), C.c_size_t()
    _check(lib().w4a4_qtensor_bytes(fmt, rows, cols, scale_mode, C.byref(c), C.byref(s), C.byref(t)),
           "w4a4_qtensor_bytes")
    return c.value, s.value, t.value


class QTensor:
    """A quantized tensor whose buffers are torch uint8/float32 device tensors."""

    def __init__(self, fmt: int, rows: int, cols: int, scale_mode: int = SCALE_TENSOR, device="cuda", flags: int = 0,
                 group: int | None = None):
        import torch
        cb, sb, tb = qtensor_bytes(fmt, rows, cols, scale_mode)
        self.format, self.rows, self.cols, self.scale_mode, self.flags = fmt, rows, cols, scale_mode, flags
        self.group = group or GROUP[fmt]
        self.codes = torch.zeros(max(cb, 16), dtype=torch.uint8, device=device)
        self.scales = torch.zeros(max(sb, 16), dtype=torch.uint8, device=device)
        self.s2 = torch.zeros(max(tb // 4, 4), dtype=torch.float32, device=device) if tb else None
        self.struct = QTensorStruct(fmt, rows, cols, self.group, scale_mode if fmt == NVFP4 else 0, flags,
                                    self.codes.data_ptr(), self.scales.data_ptr(),
                                    self.s2.data_ptr() if self.s2 is not None else None)

    @property
    def ref(self):
        return C.byref(self.struct)


def quantize_act(X, fmt: int, scale_mode: int = SCALE_TOKEN, static_s2=None, out: QTensor | None = None,
                 cols: int | None = None, hadamard: bool = False, group: int | None = None) -> QTensor:
    """X: bf16 [M, K] CUDA tensor (row stride may exceed K).  hadamard: rotate
    each quantization block first (activation side, times 1/block)."""
    M, K = X.shape
    if out is None:
        out = QTensor(fmt, M, cols or K, scale_mode if fmt == NVFP4 else SCALE_TENSOR, X.device,
                      FLAG_HADAMARD if hadamard else 0, group)
    _check(lib().w4a4_quantize_act(_ptr(X), M, K, X.stride(0), fmt, out.group, scale_mode, _ptr(static_s2),
                                   out.ref, _stream()), "w4a4_quantize_act")
    return out


def quantize_weight(W, fmt: int, S=None, out: QTensor | None = None, hadamard: bool = False,
                    group: int | None = None) -> QTensor:
    """W: bf16 [N, K]; S: optional int32 CUDA tensor of augmented channels;
    hadamard: rotate each quantization block first (weight side, unscaled)."""
    N, K = W.shape
    nS = 0 if S is None else S.numel()
    if out is None:
        out = QTensor(fmt, N, K + nS, SCALE_TENSOR, W.device, FLAG_HADAMARD if hadamard else 0, group)
    _check(lib().w4a4_quantize_weight(_ptr(W), N, K, W.stride(0), fmt, out.group, _ptr(S), nS, out.ref,
                                      _stream()), "w4a4_quantize_weight")
    return out


def quantize_weight_segments(W, seg, S=None, out: QTensor | None = None, hadamard: bool = False) -> QTensor:
    """NVFP4 weights of a fused module, one global scale per row segment.

    W: bf16 [N, K]; seg: host sequence of N-row boundaries [0, ..., N], each a
    multiple of 128 (e.g. [0, q_rows, q_rows + k_rows, N] for fused q/k/v);
    S: optional int32 CUDA tensor of augmented channels.  The result stores
    one s2 per row (scale_mode TOKEN)."""
    N, K = W.shape
    nS = 0 if S is None else S.numel()
    seg = [int(v) for v in seg]
    if out is None:
        out = QTensor(NVFP4, N, K + nS, SCALE_TOKEN, W.device, FLAG_HADAMARD if hadamard else 0)
    arr = (C.c_int32 * len(seg))(*seg)
    _check(lib().w4a4_quantize_weight_segments(_ptr(W), N, K, W.stride(0), arr, len(seg) - 1, _ptr(S), nS,
                                               out.ref, _stream()), "w4a4_quantize_weight_segments")
    return out


def quantize_act_msd(X, passes: int = 2, out: QTensor | None = None) -> QTensor:
    """Multi-pass MXFP4 activations: pass p (the residual of the earlier
    passes) in columns [p*K, (p+1)*K)."""
    M, K = X.shape
    if out is None:
        out = QTensor(MXFP4, M, passes * K, SCALE_TENSOR, X.device)
    _check(lib().w4a4_quantize_act_msd(_ptr(X), M, K, X.stride(0), passes, out.ref, _stream()),
           "w4a4_quantize_act_msd")
    return out


def quantize_weight_msd(W, passes: int = 2, out: QTensor | None = None) -> QTensor:
    """MXFP4 weights repeated `passes` times along K, for the multi-pass product."""
    N, K = W.shape
    if out is None:
        out = QTensor(MXFP4, N, passes * K, SCALE_TENSOR, W.device)
    _check(lib().w4a4_quantize_weight_msd(_ptr(W), N, K, W.stride(0), passes, out.ref, _stream()),
           "w4a4_quantize_weight_msd")
    return out


def linear_msd(X, Wq: QTensor, passes: int = 2, Y=None, ws=None):
    """The multi-pass MXFP4 linear layer (Wq from quantize_weight_msd)."""
    import torch
    M, K = X.shape
    if Y is None:
        Y = torch.empty(M, Wq.rows, dtype=torch.bfloat16, device=X.device)
    need = linear_workspace(M, Wq.rows, K, MXFP4, (passes - 1) * K)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _check(lib().w4a4_linear_msd(_ptr(X), M, K, X.stride(0), Wq.ref, passes, _ptr(Y), Y.stride(0), _ptr(ws),
                                 ws.numel(), _stream()), "w4a4_linear_msd")
    return Y


def gemm(A: QTensor, B: QTensor, Y=None):
    import torch
    if Y is None:
        Y = torch.empty(A.rows, B.rows, dtype=torch.bfloat16, device=A.codes.device)
    _check(lib().w4a4_gemm(A.ref, B.ref, _ptr(Y), Y.stride(0), _stream()), "w4a4_gemm")
    return Y


def int4_group_for_rho(rho: float) -> int:
    """INT4 scale-group size for a tensor-core / CUDA-core throughput ratio rho."""
    return int(lib().w4a4_int4_group_for_rho(float(rho)))


def linear_workspace(M: int, N: int, K: int, fmt: int, nS: int = 0) -> int:
    return int(lib().w4a4_linear_workspace(M, N, K, fmt, nS))


def linear(X, Wq: QTensor, scale_mode: int = SCALE_TOKEN, S=None, Y=None, ws=None):
    """Quantize X per token in Wq's format (plus the residual channels S) and
    multiply with Wq: the fused W4A4 linear layer."""
    import torch
    M, K = X.shape
    nS = 0 if S is None else S.numel()
    if Y is None:
        Y = torch.empty(M, Wq.rows, dtype=torch.bfloat16, device=X.device)
    need = linear_workspace(M, Wq.rows, K, Wq.format, nS)
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _check(lib().w4a4_linear(_ptr(X), M, K, X.stride(0), Wq.ref, scale_mode, _ptr(S), nS, _ptr(Y), Y.stride(0),
                             _ptr(ws), ws.numel(), _stream()), "w4a4_linear")
    return Y


def linear_noalloc(X, Wq: QTensor, scale_mode: int = SCALE_TOKEN, S=None, Y=None):
    """linear() with the library's static per-device scratch instead of a
    workspace (sizes up to NOALLOC_SCRATCH_BYTES of workspace; calls on one
    device must not overlap)."""
    import torch
    M, K = X.shape
    nS = 0 if S is None else S.numel()
    if Y is None:
        Y = torch.empty(M, Wq.rows, dtype=torch.bfloat16, device=X.device)
    _check(lib().w4a4_linear_noalloc(_ptr(X), M, K, X.stride(0), Wq.ref, scale_mode, _ptr(S), nS, _ptr(Y),
                                     Y.stride(0), _stream()), "w4a4_linear_noalloc")
    return Y


NOALLOC_SCRATCH_BYTES = 16 << 20


def augment_residual(X, S, Xaug: QTensor) -> QTensor:
    M, K = X.shape
    _check(lib().w4a4_augment_residual(_ptr(X), M, K, X.stride(0), _ptr(S), S.numel(), Xaug.ref, _stream()),
           "w4a4_augment_residual")
    return Xaug


def select_channels(Xcal, nS: int, ws=None):
    import torch
    Mc, K = Xcal.shape
    S = torch.empty(max(nS, 1), dtype=torch.int32, device=Xcal.device)
    if ws is None:
        ws = torch.empty(8 * K, dtype=torch.uint8, device=Xcal.device)
    _check(lib().w4a4_select_channels(_ptr(Xcal), Mc, K, Xcal.stride(0), nS, _ptr(S), _ptr(ws), ws.numel(),
                                      _stream()), "w4a4_select_channels")
    return S[:nS]


def device_status() -> int:
    """Synchronize the current stream; return (and clear) the device error status."""
    return int(lib().w4a4_device_status(_stream()))


def debug_set(skip_k_tile: int = -1, wait_limit_ns: int = 0):
    lib().w4a4_debug_set(int(skip_k_tile), int(wait_limit_ns))
