"""Seeded synthetic inputs shaped like the workloads the W4A4 pages describe.

This module holds random-number generation and nothing of the quantization
method: it is shared by the oracle-side and the GPU-side of every test and by
the benchmark, so that both sides see the same bits.  Every tensor is drawn
on the host with numpy's counter-based Philox generator keyed by
(seed, tensor id), rounded to bf16 (nearest even) and returned as uint16 bit
patterns.

Workloads (the model shapes named on the pages; values are synthetic, no
checkpoint or dataset is involved):
  * ``mxfp4_small``: 16x256 by 256x256, X ~ N(0,1), W ~ N(0,0.02), seed 0.
  * ``swiglu300m``: 300M-parameter SwiGLU decoder linears (d=1024,
    d_ff=2816) at 4096 tokens; X ~ N(0,1) with 8 fixed channels x50,
    W ~ N(0,0.02).  ("Depth Registers Unlock W4A4 on SwiGLU", abstract.)
  * ``llama2_70b``: Llama-2-70B linears (qkv 8192->10240, o 8192->8192,
    w1/w3 8192->28672, w2 28672->8192); X = 0.5 * Student-t(nu=4),
    W ~ N(0,0.01).  ("APEX4..." page, para 2 names LLaMA-2-70B.)
  * ``qwen25_7b_int4``: Qwen2.5-7B linears (qkv 3584->4608, w1/w3
    3584->18944, w2 18944->3584) at 2048 tokens; X ~ N(0,1) with 0.5% of
    channels x20; W ~ N(0,0.02).
  * ``qwen25_3b_aug``: Qwen2.5-3B linears (2048->2560, 2048->11008,
    11008->2048) at 8192 tokens; X ~ N(0,1) with 1% of channels x30;
    W ~ N(0,0.02); a 512-row calibration batch drawn with seed 1.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# (name, K, N) per linear of each model
SHAPES = {
    "mxfp4_small": [("gemm", 256, 256)],
    "swiglu300m": [("qkv", 1024, 3072), ("o", 1024, 1024), ("w1", 1024, 2816),
                   ("w3", 1024, 2816), ("w2", 2816, 1024)],
    "llama2_70b": [("qkv", 8192, 10240), ("o", 8192, 8192), ("w1", 8192, 28672),
                   ("w3", 8192, 28672), ("w2", 28672, 8192)],
    "qwen25_7b_int4": [("qkv", 3584, 4608), ("w1", 3584, 18944), ("w3", 3584, 18944),
                       ("w2", 18944, 3584)],
    "qwen25_3b_aug": [("up", 2048, 2560), ("gate_up", 2048, 11008), ("down", 11008, 2048)],
}

TOKENS = {"mxfp4_small": [16], "swiglu300m": [4096], "llama2_70b": [1, 16, 256, 4096, 16384],
          "qwen25_7b_int4": [2048], "qwen25_3b_aug": [8192]}


def _rng(seed: int, tensor_id: int, chunk: int = 0) -> np.random.Generator:
    key = [int(seed) & (2**64 - 1), ((int(tensor_id) << 32) + int(chunk)) & (2**64 - 1)]
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even) and return the bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


_CHUNK_ROWS = 256


def _draw_rows(shape, seed, tensor_id, draw, post=None, bf16=False):
    """Draw a [rows, cols] tensor in chunks of 256 rows, chunk c from the Philox
    stream keyed (seed, tensor_id, c); chunks run on a thread pool (numpy
    releases the GIL), the result does not depend on the thread count."""
    rows, cols = shape
    out = np.empty(shape, np.uint16 if bf16 else np.float32)

    def one(c):
        r0, r1 = c * _CHUNK_ROWS, min(rows, (c + 1) * _CHUNK_ROWS)
        x = draw(_rng(seed, tensor_id, c), (r1 - r0, cols))
        if post is not None:
            x = post(x)
        out[r0:r1] = f32_to_bf16_bits(x) if bf16 else x

    n = (rows + _CHUNK_ROWS - 1) // _CHUNK_ROWS
    if n <= 1:
        for c in range(n):
            one(c)
    else:
        with ThreadPoolExecutor(max_workers=min(n, os.cpu_count() or 1)) as ex:
            list(ex.map(one, range(n)))
    return out


def normal(shape, sigma: float, seed: int, tensor_id: int, bf16: bool = False) -> np.ndarray:
    def draw(g, sh):
        x = g.standard_normal(sh, dtype=np.float32)
        if sigma != 1.0:
            x *= np.float32(sigma)
        return x
    return _draw_rows(shape, seed, tensor_id, draw, bf16=bf16)


def student_t(shape, nu: float, scale: float, seed: int, tensor_id: int, bf16: bool = False) -> np.ndarray:
    def draw(g, sh):
        return (g.standard_t(nu, size=sh) * scale).astype(np.float32)
    return _draw_rows(shape, seed, tensor_id, draw, bf16=bf16)


def outlier_channels(K: int, count: int, seed: int) -> np.ndarray:
    """The first `count` entries of a seeded permutation of [0, K), ascending."""
    perm = _rng(seed, 0x0C4A, 0).permutation(K)
    return np.sort(perm[:count]).astype(np.int64)


def activations(model: str, M: int, K: int, seed: int = 0, tensor_id: int = 1) -> np.ndarray:
    """X [M, K] as bf16 bits for one of the workloads above."""
    if model == "llama2_70b":
        return student_t((M, K), 4.0, 0.5, seed, tensor_id, bf16=True)
    ch, f = outlier_spec(model, K)

    def draw(g, sh):
        x = g.standard_normal(sh, dtype=np.float32)
        if ch is not None:
            x[:, ch] *= np.float32(f)
        return x
    return _draw_rows((M, K), seed, tensor_id, draw, bf16=True)


def outlier_spec(model: str, K: int):
    """(outlier channel indices, multiplier) of a workload's activations, or (None, 1)."""
    if model == "swiglu300m":
        return outlier_channels(K, 8, 1234), 50.0
    if model == "qwen25_7b_int4":
        return outlier_channels(K, int(round(0.005 * K)), 1234), 20.0
    if model == "qwen25_3b_aug":
        return outlier_channels(K, int(round(0.01 * K)), 1234), 30.0
    return None, 1.0


def weights(model: str, N: int, K: int, seed: int = 0, tensor_id: int = 2) -> np.ndarray:
    """W [N, K] as bf16 bits."""
    sigma = 0.01 if model == "llama2_70b" else 0.02
    return normal((N, K), sigma, seed, tensor_id, bf16=True)


# Fused projection modules stacked along N: rows of each part and the spread of
# its weights relative to the model's weight sigma (synthetic; the parts of a
# fused module differ in magnitude, which is why each gets its own scale).
FUSED = {
    "llama2_70b": {"qkv": ((8192, 1024, 1024), (1.0, 4.0, 0.25)),
                   "w1w3": ((28672, 28672), (1.0, 0.5))},
}


def fused_weights(seg_rows, gains, K: int, model: str = "llama2_70b", seed: int = 0,
                  tensor_id: int = 2):
    """W [sum(seg_rows), K] as bf16 bits, part i drawn with sigma * gains[i];
    returns (bits, row boundaries [0, ..., N])."""
    sigma = 0.01 if model == "llama2_70b" else 0.02
    N = int(sum(seg_rows))
    w = normal((N, K), sigma, seed, tensor_id)
    bounds = np.concatenate([[0], np.cumsum(seg_rows)]).astype(np.int64)
    for i, gain in enumerate(gains):
        w[bounds[i]:bounds[i + 1]] *= np.float32(gain)
    return f32_to_bf16_bits(w), [int(b) for b in bounds]


def calibration(model: str, K: int, rows: int = 512) -> np.ndarray:
    """Calibration batch (seed 1) with the same outlier channels as the run data."""
    return activations(model, rows, K, seed=1, tensor_id=7)


def uniform_bf16(shape, lo: float, hi: float, seed: int, tensor_id: int) -> np.ndarray:
    return f32_to_bf16_bits(_rng(seed, tensor_id, 0).uniform(lo, hi, size=shape).astype(np.float32))


def e2m1_grid_values(shape, seed: int, tensor_id: int) -> np.ndarray:
    """Random values from the signed E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6}, as
    float32; the caller places a +-6 in every block when it needs one."""
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    r = _rng(seed, tensor_id, 0)
    v = grid[r.integers(0, 8, size=shape)]
    sgn = np.where(r.integers(0, 2, size=shape) == 1, -1.0, 1.0).astype(np.float32)
    return v * sgn
