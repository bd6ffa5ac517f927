"""w4a4_linear_noalloc (static per-device scratch) against w4a4_linear (caller
workspace): same kernels, so the outputs must be identical bit for bit, on
two calls in a row with different inputs.  Collected last on purpose: it must
pass both alone and after every other GPU test has used the device."""
import numpy as np
import pytest
import torch

import w4a4_quantized_gemm_token_b200 as w4
from w4a4_quantized_gemm_token_b200 import synth

pytestmark = pytest.mark.gpu


def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


CASES = [
    # (workload, M, K, N, fmt, mode)
    ("llama2_70b", 1, 8192, 10240, w4.NVFP4, w4.SCALE_TOKEN),
    ("llama2_70b", 16, 8192, 10240, w4.NVFP4, w4.SCALE_TOKEN),
    ("llama2_70b", 7, 1280, 384, w4.NVFP4, w4.SCALE_TENSOR),
    ("llama2_70b", 16, 1024, 2048, w4.MXFP4, 0),
    ("qwen25_7b_int4", 33, 3584, 4608, w4.INT4, 0),
    ("llama2_70b", 300, 2048, 1024, w4.NVFP4, w4.SCALE_TOKEN),
]


@pytest.mark.parametrize("model,M,K,N,fmt,mode", CASES)
def test_noalloc_matches_workspace_path_twice(model, M, K, N, fmt, mode):
    assert w4.linear_workspace(M, N, K, fmt) <= w4.NOALLOC_SCRATCH_BYTES
    Wq = w4.quantize_weight(dev(synth.weights(model, N, K, seed=21)), fmt)
    for call in range(2):
        X = dev(synth.activations(model, M, K, seed=40 + call))
        ref = w4.linear(X, Wq, mode)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.linear_noalloc(X, Wq, mode, Y=Y)
        torch.cuda.synchronize()
        assert w4.device_status() == w4.OK
        assert torch.equal(Y.view(torch.int16), ref.view(torch.int16)), f"call {call}"


def test_noalloc_residual_channels():
    M, K, N, nS = 16, 1024, 256, 128
    S = w4.select_channels(dev(synth.calibration("qwen25_3b_aug", K, rows=512)), nS)
    Wq = w4.quantize_weight(dev(synth.weights("qwen25_3b_aug", N, K, seed=5)), w4.NVFP4, S=S)
    for call in range(2):
        X = dev(synth.activations("qwen25_3b_aug", M, K, seed=50 + call))
        ref = w4.linear(X, Wq, w4.SCALE_TOKEN, S=S)
        Y = w4.linear_noalloc(X, Wq, w4.SCALE_TOKEN, S=S)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), ref.view(torch.int16)), f"call {call}"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    M, K, N = 4096, 8192, 1024
    assert w4.linear_workspace(M, N, K, w4.NVFP4) > w4.NOALLOC_SCRATCH_BYTES
    Wq = w4.quantize_weight(dev(synth.weights("llama2_70b", N, K, seed=3)), w4.NVFP4)
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    Y = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4A4Error) as e:
        w4.linear_noalloc(X, Wq, w4.SCALE_TOKEN, Y=Y)
    assert e.value.status == w4.ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((Y == 3.0).all())          # nothing was launched


@pytest.mark.parametrize("model,M,K,N,fmt,mode", [
    ("llama2_70b", 1, 8192, 10240, w4.NVFP4, w4.SCALE_TOKEN),   # decode: split-K partials and tile counters
    ("llama2_70b", 16, 2048, 1024, w4.MXFP4, 0),
    ("llama2_70b", 300, 2048, 1024, w4.NVFP4, w4.SCALE_TOKEN),  # CTA-pair GEMM
])
def test_noalloc_back_to_back_calls_on_one_stream(model, M, K, N, fmt, mode):
    """Three no-alloc calls with different inputs issued on one stream with
    nothing between them (no synchronisation, no other launch), so each
    call's quantizer may start while the previous call's GEMM still runs;
    every output must equal the workspace path's, computed afterwards."""
    Wq = w4.quantize_weight(dev(synth.weights(model, N, K, seed=22)), fmt)
    Xs = [dev(synth.activations(model, M, K, seed=60 + c)) for c in range(3)]
    Ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    torch.cuda.synchronize()
    for X, Y in zip(Xs, Ys):
        w4.linear_noalloc(X, Wq, mode, Y=Y)
    torch.cuda.synchronize()
    assert w4.device_status() == w4.OK
    for c, (X, Y) in enumerate(zip(Xs, Ys)):
        ref = w4.linear(X, Wq, mode)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), ref.view(torch.int16)), f"call {c}"
