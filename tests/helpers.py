"""Test-side helpers: layout decoding written independently of the library,
the GEMM tolerance of the pages' target, and torch/numpy conversions."""
import numpy as np


def pad128(x):
    return (x + 127) // 128 * 128


def sf_index(r, c, cols_blocks):
    """Byte index of scale (row r, block c) in the MMA layout: 512-byte atoms of
    128 rows x 4 blocks; inside an atom row r sits in line r%32, word (r%128)//32."""
    atom = (r // 128) * (cols_blocks // 4) + c // 4
    return atom * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (c % 4)


def unswizzle_scales(buf, rows, cols, group):
    """Row-major [rows][cols/group] view of an MMA-layout scale buffer (numpy uint8)."""
    nb = cols // group
    r = np.arange(rows)[:, None]
    c = np.arange(nb)[None, :]
    return np.asarray(buf)[sf_index(r, c, nb)]


def padding_scales(buf, rows, cols, group):
    """Scale bytes of the padding rows [rows, pad128(rows))."""
    nb = cols // group
    r = np.arange(rows, pad128(rows))[:, None]
    c = np.arange(nb)[None, :]
    return np.asarray(buf)[sf_index(r, c, nb)]


def int4_scales(buf_f32, rows, cols):
    """[rows][cols/128] view of the group-major INT4 scale buffer."""
    G = cols // 128
    return np.asarray(buf_f32)[: G * pad128(rows)].reshape(G, pad128(rows))[:, :rows].T


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def ulp_bf16(v):
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.exp2(e - 7)


def gemm_violations(y_gpu_bits, yref, absdot):
    """Elements outside |dY| <= 1 ulp_bf16(Y*) + 1e-5 * sum|a w| (the target tolerance)."""
    y = bf16_to_f64(y_gpu_bits)
    tol = ulp_bf16(yref) + 1e-5 * absdot
    bad = ~(np.abs(y - yref) <= tol)
    return bad


def to_np_u16(t):
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_dev_bf16(bits, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)
