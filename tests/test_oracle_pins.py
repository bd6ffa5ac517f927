"""Pins of the oracle to things other than itself: the format definitions
(golden table), library conversions (ml_dtypes, numpy), brute force, closed
forms, textbook special cases and invariants.  CPU only."""
import os

import ml_dtypes as md
import numpy as np
import pytest

from w4a4_quantized_gemm_token_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_e4m3_table.txt")
GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            rows.append(line.split())
    return rows


# ---- independent test-side helpers (library decoders, brute force) --------
def lib_e2m1(codes):
    """Decode E2M1 codes with ml_dtypes (float4_e2m1fn stores one code per byte)."""
    return np.asarray(codes, np.uint8).view(md.float4_e2m1fn).astype(np.float64)


def lib_e4m3(codes):
    return np.asarray(codes, np.uint8).view(md.float8_e4m3fn).astype(np.float64)


def unpack(codes):
    c = np.asarray(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 15
    out[..., 1::2] = c >> 4
    return out


def brute_e2m1(v):
    """Nearest grid magnitude, ties to the even code, saturating; sign bit kept."""
    m = min(abs(float(v)), 6.0)
    d = np.abs(GRID - m)
    best = np.flatnonzero(d == d.min())
    code = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
    return code | (8 if np.signbit(v) else 0)


def bf16(x):
    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


# ---- scalar encodings -------------------------------------------------------
def test_golden_table(orc):
    for row in _golden():
        if row[0] == "e2m1":
            assert orc.e2m1_decode(int(row[1])) == float(row[2])
            assert orc.e2m1_decode(int(row[1]) | 8) == -float(row[2])
        elif row[0] == "tie":
            assert orc.e2m1_encode(float(row[1])) == int(row[2])
            assert orc.e2m1_encode(-float(row[1])) == int(row[2]) | 8
        elif row[0] == "e4m3":
            assert orc.e4m3_decode(int(row[1], 16)) == float(row[2])


def test_e2m1_decode_vs_library(orc):
    got = np.array([orc.e2m1_decode(c) for c in range(16)])
    np.testing.assert_array_equal(got, lib_e2m1(np.arange(16)))
    # every decoded value is on the grid
    assert set(np.abs(got)) <= set(GRID)


def test_e2m1_encode_vs_brute_force_and_library(orc):
    r = np.random.default_rng(1)
    vals = np.concatenate([r.uniform(-8, 8, 4000), r.normal(0, 2, 4000),
                           GRID[1:] * 0.5 + GRID[:-1] * 0.5, -(GRID[1:] * 0.5 + GRID[:-1] * 0.5),
                           GRID, -GRID, [1e30, -1e30, 6.0001, -0.0, 1e-30, -1e-30]]).astype(np.float32)
    got = np.array([orc.e2m1_encode(v) for v in vals], np.uint8)
    ref = np.array([brute_e2m1(v) for v in vals], np.uint8)
    np.testing.assert_array_equal(got, ref)
    lib = vals.astype(md.float4_e2m1fn).view(np.uint8)
    np.testing.assert_array_equal(got, lib)


def test_e4m3_decode_vs_library(orc):
    for c in range(256):
        a, b = orc.e4m3_decode(c), lib_e4m3([c])[0]
        assert (np.isnan(a) and np.isnan(b)) or a == b, c


def test_e4m3_encode_vs_library(orc):
    r = np.random.default_rng(2)
    vals = np.concatenate([np.exp2(r.uniform(-12, 8.85, 20000)),
                           [2.0 ** -10, 2.0 ** -10 * 1.0001, 2.0 ** -9, 2.0 ** -6, 448.0, 464.0, 1.5 * 2 ** -10],
                           lib_e4m3(np.arange(0, 127))[1:]]).astype(np.float32)
    vals = vals[vals <= 464.0]
    got = np.array([orc.e4m3_encode(v) for v in vals], np.uint8)
    lib = vals.astype(md.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(got, lib)
    # saturation (the library's conversion overflows to NaN there instead)
    for v in [464.0001, 500.0, 1e6, np.inf]:
        assert orc.e4m3_encode(v) == 0x7E
    assert orc.e4m3_encode(0.0) == 0 and orc.e4m3_encode(2.0 ** -10) == 0


def test_floor_log2_vs_frexp(orc):
    r = np.random.default_rng(3)
    vals = np.concatenate([np.exp2(r.uniform(-148, 127, 3000)), [1.0, 2.0, 0.75, 2.0 ** -149, 3.4e38]])
    vals = vals.astype(np.float32)
    vals = vals[vals > 0]
    for v in vals:
        assert orc.floor_log2(v) == int(np.frexp(np.float64(v))[1]) - 1


def test_f64_to_bf16_is_nearest_even(orc):
    r = np.random.default_rng(4)
    vals = np.concatenate([r.normal(0, 1, 3000) * np.exp2(r.integers(-130, 120, 3000)),
                           [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, 2 ** -140]])
    for v in vals:
        b = orc.f64_to_bf16(v)
        got = float(np.array([b], np.uint16).view(md.bfloat16)[0])
        # neighbours (in magnitude, same sign) of the library's float-first conversion
        c = int(np.array([np.float32(v)]).astype(md.bfloat16).view(np.uint16)[0])
        sign, mag = c & 0x8000, c & 0x7FFF
        cands = []
        for d in (-1, 0, 1):
            if 0 <= mag + d < 0x7F80:
                w = sign | (mag + d)
                cands.append((abs(float(np.array([w], np.uint16).view(md.bfloat16)[0]) - v), w))
        best = min(x[0] for x in cands)
        ok = [w for (e, w) in cands if e == best]
        if len(ok) > 1:
            ok = [w for w in ok if w % 2 == 0]
        assert b in ok, (v, got)


# ---- NVFP4 ------------------------------------------------------------------
def test_nvfp4_s2_closed_form(orc):
    for a in [1.0, 3.0, 50.0, 1e-30, 1e-36, 0.0]:
        s2 = np.float32(a) / np.float32(2688.0)
        want = np.float32(1.0) if (a == 0 or s2 < np.finfo(np.float32).tiny) else s2
        assert orc.nvfp4_s2_from_amax(a) == want


def test_nvfp4_zero_and_single_outlier(orc):
    K = 64
    X = np.zeros((3, K), np.float32)
    X[1, 5] = 3.7
    X[2, 40] = -123.0
    c, s, s2 = orc.quant_nvfp4(bf16(X), mode=1)
    assert np.all(s[0] == 0) and np.all(c[0] == 0) and s2[0] == 1.0
    q = unpack(c)
    assert q[1, 5] == 0x7 and q[2, 40] == 0xF           # +6 and -6
    assert np.count_nonzero(q[1]) == 1 and np.count_nonzero(q[2]) == 1
    assert np.count_nonzero(s[1]) == 1 and lib_e4m3([s[1, 0]])[0] == 448.0


def test_nvfp4_textbook_identity_and_exact_gemm(orc):
    """E2M1-grid inputs with a +-6 in every block and static s2 = 1: every block
    scale is E4M3(1) and quantization is the identity; the GEMM is an exact
    integer matmul of the doubled values."""
    M, N, K = 8, 12, 64
    A = synth.e2m1_grid_values((M, K), 5, 1)
    B = synth.e2m1_grid_values((N, K), 5, 2)
    A[:, ::16] = 6.0
    B[:, 3::16] = -6.0
    one = np.ones(1, np.float32)
    ca, sa, s2a = orc.quant_nvfp4(bf16(A), mode=0, static_s2=one)
    cb, sb, s2b = orc.quant_nvfp4(bf16(B), mode=0, static_s2=one)
    assert np.all(sa == 0x38) and np.all(sb == 0x38) and s2a[0] == 1.0
    np.testing.assert_array_equal(lib_e2m1(unpack(ca)), A)
    Y, yref, _ = orc.gemm_nvfp4(ca, sa, s2a, 0, cb, sb, s2b)
    exact = (2 * A).astype(np.int64) @ (2 * B).astype(np.int64).T
    np.testing.assert_array_equal(yref, exact / 4.0)
    np.testing.assert_array_equal(Y, bf16(exact / 4.0))


def _nvfp4_lib_dequant(codes, scales, s2, mode):
    e = lib_e2m1(unpack(codes))
    sc = np.repeat(lib_e4m3(scales), 16, axis=1)
    s2 = np.asarray(s2, np.float64).reshape(-1, 1) if mode == 1 else np.float64(s2[0])
    return e * sc * s2


@pytest.mark.parametrize("mode", [0, 1])
def test_nvfp4_rule_against_library_steps(orc, mode):
    """Re-derive every block scale and code from X with library conversions."""
    M, K = 6, 96
    X = bf16(synth.normal((M, K), 1.0, 9, 1) * np.exp2(np.arange(M) - 3)[:, None])
    c, s, s2 = orc.quant_nvfp4(X, mode=mode)
    x = synth.bf16_bits_to_f32(X)
    amax = np.abs(x).max(axis=1) if mode == 1 else np.array([np.abs(x).max()])
    np.testing.assert_array_equal(s2, (amax / np.float32(2688)).astype(np.float32))
    for m in range(M):
        rs2 = np.float32(s2[m] if mode == 1 else s2[0])
        for b in range(K // 16):
            blk = x[m, 16 * b:16 * b + 16]
            t = (np.float32(np.abs(blk).max()) / np.float32(6)) / rs2
            sb = np.array([t], np.float32).astype(md.float8_e4m3fn).view(np.uint8)[0]
            assert s[m, b] == sb
            d = np.float32(lib_e4m3([sb])[0]) * rs2
            want = (blk / d).astype(np.float32).astype(md.float4_e2m1fn).view(np.uint8)
            np.testing.assert_array_equal(unpack(c)[m, 16 * b:16 * b + 16], want)


def test_nvfp4_idempotent_when_block_max_code_is_6(orc):
    """Blocks built so that amax/6 is an E4M3 normal (x s2 = 1): re-quantizing
    the dequantized tensor returns identical codes and scales."""
    M, K = 5, 128
    r = np.random.default_rng(11)
    normals = lib_e4m3(np.arange(0x08, 0x7F))
    sig = r.choice(normals[normals <= 8], size=(M, K // 16))
    X = r.uniform(-6, 6, (M, K)) * np.repeat(sig, 16, axis=1)
    X[:, ::16] = 6 * sig * np.sign(r.uniform(-1, 1, (M, K // 16)))
    one = np.ones(1, np.float32)
    c, s, s2 = orc.quant_nvfp4(bf16(X), mode=0, static_s2=one)
    xhat = orc.dequant_nvfp4(c, s, s2, 0)
    Xh = bf16(xhat)
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(Xh), xhat)   # representable
    c2, s2b, _ = orc.quant_nvfp4(Xh, mode=0, static_s2=one)
    np.testing.assert_array_equal(c, c2)
    np.testing.assert_array_equal(s, s2b)


def test_nvfp4_subnormal_scale_exception_documented(orc):
    """In the E4M3 subnormal range a block's largest code can fall below 6;
    re-quantization may then pick another scale (why the idempotence pin
    above keeps block scales normal)."""
    X = np.zeros((1, 16), np.float32)
    X[0, 0] = 5.0 * 2 ** -9 * 6 / 6 * 1.2   # amax/6 lands between E4M3 subnormals
    one = np.ones(1, np.float32)
    c, s, s2 = orc.quant_nvfp4(bf16(X), mode=0, static_s2=one)
    assert lib_e4m3(s)[0, 0] < 2.0 ** -6


# ---- MXFP4 ------------------------------------------------------------------
def test_mxfp4_rule_zero_outlier_idempotent(orc):
    M, K = 4, 128
    X = synth.normal((M, K), 1.0, 12, 1) * np.exp2(np.array([-20, 0, 7, 30]))[:, None]
    X[0, :32] = 0.0
    X[1, 32:64] = 0.0
    X[1, 40] = 4.9
    c, s = orc.quant_mxfp4(bf16(X))
    assert s[0, 0] == 0 and np.all(c[0, :16] == 0)
    assert s[1, 1] == 127 + 2 - 2 and unpack(c)[1, 40] == 0x6    # 4.9/2^0 -> 4 (code 6)
    x = synth.bf16_bits_to_f32(bf16(X)).astype(np.float64)
    for m in range(M):
        for b in range(K // 32):
            a = np.abs(x[m, 32 * b:32 * b + 32]).max()
            if a == 0:
                continue
            e = int(np.frexp(a)[1]) - 1
            assert s[m, b] == np.clip(e - 2 + 127, 0, 254)
    xhat = orc.dequant_mxfp4(c, s)
    c2, s2 = orc.quant_mxfp4(bf16(xhat))
    np.testing.assert_array_equal(c, c2)
    np.testing.assert_array_equal(s, s2)


def test_mxfp4_single_outlier_codes(orc):
    for v, code in [(4.0, 6), (4.9, 6), (5.0, 6), (5.1, 7), (7.9, 7), (-6.0, 0xF)]:
        X = np.zeros((1, 32), np.float32)
        X[0, 3] = v
        c, s = orc.quant_mxfp4(bf16(X))
        assert unpack(c)[0, 3] == code, v


# ---- INT4 -------------------------------------------------------------------
def test_int4_rule_zero_outlier_idempotent(orc):
    M, K = 3, 256
    X = synth.normal((M, K), 1.0, 13, 1)
    X[0, :128] = 0
    X[1, 128:] = 0
    X[1, 200] = -2.5
    c, s = orc.quant_int4(bf16(X))
    q = unpack(c).astype(np.int64)
    q = np.where(q >= 8, q - 16, q)
    assert s[0, 0] == 0 and np.all(q[0, :128] == 0)
    assert q[1, 200] == -7 and np.count_nonzero(q[1, 128:]) == 1
    x = synth.bf16_bits_to_f32(bf16(X))
    for m in range(M):
        for g in range(K // 128):
            blk = x[m, 128 * g:128 * g + 128]
            sc = np.float32(np.abs(blk).max()) / np.float32(7)
            assert s[m, g] == sc
            if sc:
                want = np.clip(np.rint((blk / sc).astype(np.float32)), -8, 7)
                np.testing.assert_array_equal(q[m, 128 * g:128 * g + 128], want)
    # idempotence on groups whose amax is 7 * 2^k (scale is a power of two)
    G = np.rint(synth.normal((2, 128), 2.0, 14, 1)).clip(-7, 7)
    G[:, 0] = 7
    G = G * np.array([[2.0 ** -3], [2.0 ** 5]])
    c1, s1 = orc.quant_int4(bf16(G))
    c2, s2 = orc.quant_int4(bf16(orc.dequant_int4(c1, s1)))
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)


# ---- GEMM brute force -------------------------------------------------------
def _bf16_nearest(v):
    return np.array([np.float32(x) for x in v.ravel()]).reshape(v.shape)


@pytest.mark.parametrize("K", [32, 128, 256])
def test_gemm_fp64_brute_force(orc, K):
    M, N = 17, 23
    Xa = bf16(synth.normal((M, K), 1.0, 20, 1))
    Xw = bf16(synth.normal((N, K), 0.02, 20, 2))
    # NVFP4 (token activations, tensor weights)
    ca, sa, s2a = orc.quant_nvfp4(Xa, mode=1)
    cw, sw, s2w = orc.quant_nvfp4(Xw, mode=0)
    A = _nvfp4_lib_dequant(ca, sa, s2a, 1)
    W = _nvfp4_lib_dequant(cw, sw, s2w, 0)
    Y, yref, absd = orc.gemm_nvfp4(ca, sa, s2a, 1, cw, sw, s2w)
    naive = A @ W.T
    assert np.all(np.abs(yref - naive) <= 1e-12 * (np.abs(A) @ np.abs(W).T))
    np.testing.assert_allclose(absd, np.abs(A) @ np.abs(W).T, rtol=1e-12)
    yb = synth.bf16_bits_to_f32(Y).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.abs(naive) + 1e-300)) - 7)
    assert np.all(np.abs(yb - naive) <= 0.5 * ulp * (1 + 1e-9))
    if K % 32 == 0:
        ca, sa = orc.quant_mxfp4(Xa)
        cw, sw = orc.quant_mxfp4(Xw)
        A = lib_e2m1(unpack(ca)) * np.repeat(np.exp2(sa.astype(np.float64) - 127), 32, axis=1)
        W = lib_e2m1(unpack(cw)) * np.repeat(np.exp2(sw.astype(np.float64) - 127), 32, axis=1)
        Y, yref, absd = orc.gemm_mxfp4(ca, sa, cw, sw)
        assert np.all(np.abs(yref - A @ W.T) <= 1e-12 * (np.abs(A) @ np.abs(W).T))
    if K % 128 == 0:
        ca, sa = orc.quant_int4(Xa)
        cw, sw = orc.quant_int4(Xw)
        qa = unpack(ca).astype(np.int64); qa = np.where(qa >= 8, qa - 16, qa)
        qw = unpack(cw).astype(np.int64); qw = np.where(qw >= 8, qw - 16, qw)
        A = qa * np.repeat(sa.astype(np.float64), 128, axis=1)
        W = qw * np.repeat(sw.astype(np.float64), 128, axis=1)
        Y, yref, absd = orc.gemm_int4(ca, sa, cw, sw)
        assert np.all(np.abs(yref - A @ W.T) <= 1e-12 * (np.abs(A) @ np.abs(W).T))


# ---- residual augmentation ----------------------------------------------------
@pytest.mark.parametrize("order", ["asc", "perm"])
def test_augment_invariants(orc, order):
    M, K, nS = 16, 512, 32
    X = bf16(synth.normal((M, K), 1.0, 30, 1) * np.where(np.arange(K) % 37 == 0, 30.0, 1.0))
    S = orc.select_channels(X, nS)
    if order == "perm":  # column K + j holds channel S[j], whatever the order
        S = S[np.random.default_rng(3).permutation(nS)]
    c, s, s2 = orc.quant_nvfp4(X, mode=1)
    rc, rs = orc.augment_nvfp4(X, S, c, s, s2, 1)
    x = synth.bf16_bits_to_f32(X).astype(np.float64)
    xhat = _nvfp4_lib_dequant(c, s, s2, 1).astype(np.float32).astype(np.float64)
    R = (x[:, S] - xhat[:, S]).astype(np.float32).astype(np.float64)
    Rh = _nvfp4_lib_dequant(rc, rs, s2, 1)
    assert np.all(np.abs(R - Rh) <= np.abs(R))                  # 0 is on the grid
    d2 = np.repeat(lib_e4m3(rs), 16, axis=1) * s2.reshape(-1, 1)
    assert np.all(np.abs(R - Rh) <= 1.0 * d2 + 1e-30)           # half the widest gap
    e1 = np.abs(x[:, S] - xhat[:, S]).sum()
    e2 = np.abs(x[:, S] - xhat[:, S] - Rh).sum()
    assert e2 < 0.5 * e1


def test_select_channels_vs_sort(orc):
    M, K = 40, 300
    X = synth.normal((M, K), 1.0, 31, 1)
    X[:, 10] = X[:, 11] = 9.0     # an exact tie: lower index first
    Xb = bf16(X)
    for nS in [0, 1, 16, 64, K]:
        S = orc.select_channels(Xb, nS)
        amax = np.abs(synth.bf16_bits_to_f32(Xb)).max(axis=0)
        order = np.lexsort((np.arange(K), -amax))
        np.testing.assert_array_equal(S, np.sort(order[:nS]))
    S = orc.select_channels(Xb, 1)
    assert list(S) == [10]


# ---- fused modules: per-segment weight scales ------------------------------------
def test_segments_single_segment_is_the_tensor_rule(orc):
    X = bf16(synth.normal((40, 64), 0.02, 40, 1))
    c, s, s2 = orc.quant_nvfp4_segments(X, [0, 40])
    c0, s0, t0 = orc.quant_nvfp4(X, mode=0)
    np.testing.assert_array_equal(c, c0)
    np.testing.assert_array_equal(s, s0)
    assert np.all(s2 == t0[0])


def test_segments_are_separate_tensors(orc):
    # rows of very different magnitude, as in fused q/k/v modules
    X = bf16(synth.normal((48, 64), 1.0, 41, 1) * np.repeat([1.0, 3000.0, 0.001], 16)[:, None])
    seg = [0, 16, 32, 48]
    c, s, s2 = orc.quant_nvfp4_segments(X, seg)
    for i in range(3):
        r0, r1 = seg[i], seg[i + 1]
        ci, si, ti = orc.quant_nvfp4(X[r0:r1], mode=0)
        np.testing.assert_array_equal(c[r0:r1], ci)
        np.testing.assert_array_equal(s[r0:r1], si)
        assert np.all(s2[r0:r1] == ti[0])
    # one scale for the whole fused tensor puts the small module's block scales below
    # E4M3's smallest subnormal: every code of it is 0, while its own scale keeps it
    ct, _, _ = orc.quant_nvfp4(X, mode=0)
    assert (unpack(ct[32:]) & 7 == 0).mean() == 1.0
    assert (unpack(c[32:]) & 7 == 0).mean() < 0.2


def test_gemm_per_row_weight_scale(orc):
    M, N, K = 9, 48, 128
    A = bf16(synth.normal((M, K), 1.0, 42, 1))
    W = bf16(synth.normal((N, K), 0.02, 42, 2) * np.repeat([1.0, 50.0, 0.02], 16)[:, None])
    ca, sa, s2a = orc.quant_nvfp4(A, mode=1)
    cw, sw, s2w = orc.quant_nvfp4_segments(W, [0, 16, 32, 48])
    Y, yref, absd = orc.gemm_nvfp4(ca, sa, s2a, 1, cw, sw, s2w)
    # brute force on the dequantized operands (library conversions, fp64)
    naive = _nvfp4_lib_dequant(ca, sa, s2a, 1) @ _nvfp4_lib_dequant(cw, sw, s2w, 1).T
    assert np.all(np.abs(yref - naive) <= 1e-12 * np.abs(naive) + 1e-300)
    # all rows sharing one scale reduces to the per-tensor form
    cw0, sw0, t0 = orc.quant_nvfp4(W, mode=0)
    Y1, y1, _ = orc.gemm_nvfp4(ca, sa, s2a, 1, cw0, sw0, np.full(N, t0[0], np.float32))
    Y0, y0, _ = orc.gemm_nvfp4(ca, sa, s2a, 1, cw0, sw0, t0)
    np.testing.assert_array_equal(Y1, Y0)
    np.testing.assert_array_equal(y1, y0)


# ---- multi-pass MXFP4 (MSD) -------------------------------------------------
def _mx_values(codes, scales, K):
    """Values of MXFP4 codes by the ml_dtypes decoder and 2^(c-127)."""
    return lib_e2m1(unpack(codes)) * np.repeat(np.exp2(scales.astype(np.float64) - 127), 32, axis=-1)[..., :K]


def _msd_inputs():
    X = np.concatenate([synth.normal((6, 256), 1.0, 51, 1),
                        synth.student_t((6, 256), 4.0, 0.5, 51, 2) * np.exp2(np.array([-30, -3, 0, 5, 20, 60]))[:, None]])
    X[0, :32] = 0.0                       # an all-zero block
    X[1, 32:64] = -0.0                    # negative zeros
    X[2, 64:96] = 1e-38                   # tiny values
    X[3, 100] = 3e38                      # near the top of the range
    return bf16(X)


def test_msd_one_pass_is_mxfp4(orc):
    Xb = _msd_inputs()
    c1, s1 = orc.quant_mxfp4_msd(Xb, passes=1)
    c, s = orc.quant_mxfp4(Xb)
    np.testing.assert_array_equal(c1, c)
    np.testing.assert_array_equal(s1, s)


def test_msd_exact_inputs_leave_no_residual(orc):
    """Blocks already on the MXFP4 grid (block maximum 4 or 6 times 2^e) are
    reproduced by the first pass; the second pass sees zeros only."""
    M, K = 4, 256
    V = synth.e2m1_grid_values((M, K), 52, 1)
    V[:, ::32] = 6.0
    V[1, ::32] = -4.0
    V *= np.exp2(np.arange(M) * 7 - 10)[:, None]
    c, s = orc.quant_mxfp4_msd(bf16(V), passes=2)
    np.testing.assert_array_equal(_mx_values(c[:, :K // 2], s[:, :K // 32], K), V)
    assert np.all(unpack(c[:, K // 2:]) & 7 == 0) and np.all(s[:, K // 32:] == 0)


@pytest.mark.parametrize("passes", [2, 3])
def test_msd_passes_follow_the_rule_on_the_residual(orc, passes):
    """Each later pass is the MXFP4 rule (restated here with frexp and the
    brute-force grid search) applied to the exact residual of the earlier
    passes; the residual is a bf16 value; every pass shrinks every element's
    error; a pass's error is at most twice its block unit (once without
    saturation)."""
    Xb = _msd_inputs()
    M, K = Xb.shape
    c, s = orc.quant_mxfp4_msd(Xb, passes=passes)
    x = synth.bf16_bits_to_f32(Xb).astype(np.float64)
    r = x.copy()
    prev = np.abs(r)
    for p in range(passes):
        cp, sp = c[:, p * K // 2:(p + 1) * K // 2], s[:, p * K // 32:(p + 1) * K // 32]
        # the rule on this pass's input r
        for m in range(M):
            for b in range(K // 32):
                blk = r[m, 32 * b:32 * b + 32]
                a = np.abs(blk).max()
                e = 0 if a == 0 else int(np.clip(np.frexp(a)[1] - 1 - 2 + 127, 0, 254))
                assert sp[m, b] == e, (p, m, b)
                want = [0] * 32 if a == 0 else [brute_e2m1(v * 2.0 ** (127 - e)) for v in blk]
                np.testing.assert_array_equal(unpack(cp)[m, 32 * b:32 * b + 32], want)
        v = _mx_values(cp, sp, K)
        unit = np.repeat(np.exp2(sp.astype(np.float64) - 127), 32, axis=-1)
        sat = np.abs(r) > 6 * unit
        r = r - v
        assert np.all(np.abs(r) <= np.where(sat, 2.0, 1.0) * unit)
        assert np.all(np.abs(r) <= prev)
        prev = np.abs(r)
        # the residual is exact in bf16
        np.testing.assert_array_equal(synth.bf16_bits_to_f32(bf16(r)).astype(np.float64), r)


def test_msd_two_passes_cut_the_error(orc):
    """On the Llama-like activations two passes cut the RMS error by more than
    4x (each pass has the resolution of one E2M1 grid under its own unit)."""
    Xb = synth.activations("llama2_70b", 64, 1024, seed=53)
    x = synth.bf16_bits_to_f32(Xb).astype(np.float64)
    c1, s1 = orc.quant_mxfp4(Xb)
    c2, s2 = orc.quant_mxfp4_msd(Xb, passes=2)
    e1 = x - _mx_values(c1, s1, 1024)
    e2 = x - _mx_values(c2[:, :512], s2[:, :32], 1024) - _mx_values(c2[:, 512:], s2[:, 32:], 1024)
    assert np.sqrt((e2 ** 2).mean()) < np.sqrt((e1 ** 2).mean()) / 4


# ---- block-local Walsh-Hadamard rotation ------------------------------------
def _sylvester(n):
    i = np.arange(n)
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i[:, None] & i[None, :])
    return np.where(pc % 2 == 0, 1.0, -1.0)


@pytest.mark.parametrize("n", [16, 32, 128])
def test_rotation_of_unit_vectors_is_sylvester_hadamard(orc, n):
    """Rows of the identity come out as the rows of H, H[i][j] = (-1)^popcount(i&j)
    (closed form); the activation side is H/n."""
    I = bf16(np.eye(n))
    np.testing.assert_array_equal(orc.rotate_blocks(I, n, act_side=False), _sylvester(n))
    np.testing.assert_array_equal(orc.rotate_blocks(I, n, act_side=True), _sylvester(n) / n)


@pytest.mark.parametrize("n", [16, 32, 128])
def test_rotation_exact_on_small_integers_and_cancels_in_the_product(orc, n):
    """Small integers keep every butterfly exact, so the transform equals the
    integer product X H (block by block), and (X H/n)(W H)^T = X W^T exactly."""
    K = 2 * n
    r = np.random.default_rng(61)
    X = r.integers(-8, 9, size=(5, K)).astype(np.float64)
    W = r.integers(-8, 9, size=(7, K)).astype(np.float64)
    Hb = np.kron(np.eye(K // n), _sylvester(n))
    Xa = orc.rotate_blocks(bf16(X), n, act_side=True).astype(np.float64)
    Wr = orc.rotate_blocks(bf16(W), n, act_side=False).astype(np.float64)
    np.testing.assert_array_equal(Xa, X @ Hb / n)
    np.testing.assert_array_equal(Wr, W @ Hb)
    np.testing.assert_array_equal(Xa @ Wr.T, X @ W.T)


@pytest.mark.parametrize("n", [16, 32, 128])
def test_rotation_rounding_within_the_butterfly_bound(orc, n):
    """On general bf16 data each of the log2(n) stages rounds once: the FP32
    result is within log2(n) * 2^-24 * (|X| |H|) of the exact product."""
    K = 4 * n
    spread = np.exp2(np.random.default_rng(62).integers(-14, 15, size=(8, K)))   # wide exponent range
    Xb = bf16(synth.normal((8, K), 1.0, 62, 1) * spread)
    x = synth.bf16_bits_to_f32(Xb).astype(np.float64)
    Hb = np.kron(np.eye(K // n), _sylvester(n))
    got = orc.rotate_blocks(Xb, n, act_side=False).astype(np.float64)
    bound = np.log2(n) * 2.0 ** -24 * (np.abs(x) @ np.abs(Hb))
    assert np.all(np.abs(got - x @ Hb) <= bound)
    assert np.any(got != x @ Hb)  # the data really exercises rounding


def test_fp32_quantizers_reduce_to_the_bf16_ones(orc):
    """On bf16-valued FP32 input the FP32-input quantizers equal the pinned ones."""
    Xb = synth.activations("llama2_70b", 9, 512, seed=63)
    xf = synth.bf16_bits_to_f32(Xb)
    for mode in (0, 1):
        a, b = orc.quant_nvfp4_f32(xf, mode), orc.quant_nvfp4(Xb, mode=mode)
        for u, v in zip(a, b):
            np.testing.assert_array_equal(u, v)
    for u, v in zip(orc.quant_mxfp4_f32(xf), orc.quant_mxfp4(Xb)):
        np.testing.assert_array_equal(u, v)
    for u, v in zip(orc.quant_int4_f32(xf), orc.quant_int4(Xb)):
        np.testing.assert_array_equal(u.view(np.uint8), v.view(np.uint8))


# ---- INT4 with coarser groups ------------------------------------------------
def test_int4_g128_is_the_base_rule(orc):
    Xb = synth.activations("qwen25_7b_int4", 7, 512, seed=71)
    for u, v in zip(orc.quant_int4_g(Xb, 128), orc.quant_int4(Xb)):
        np.testing.assert_array_equal(u.view(np.uint8), v.view(np.uint8))


@pytest.mark.parametrize("G", [256, 512, 1024])
def test_int4_groups_follow_the_rule(orc, G):
    """Each group of G: s = RN32(amax/7), q = clamp(rint(x/s), -8, 7) with IEEE
    FP32 division (numpy float32), ties to even; zero group -> s = 0, codes 0."""
    K = 2048
    Xb = synth.activations("qwen25_7b_int4", 5, K, seed=72)
    Xb[1, :G] = 0
    c, s = orc.quant_int4_g(Xb, G)
    x = synth.bf16_bits_to_f32(Xb)
    q = unpack(c).astype(np.int64)
    q = np.where(q >= 8, q - 16, q)
    for m in range(5):
        for g in range(K // G):
            blk = x[m, G * g:G * g + G]
            sc = np.float32(np.abs(blk).max()) / np.float32(7)
            assert s[m, g] == sc
            want = np.zeros(G, np.int64) if sc == 0 else np.clip(np.rint(blk / sc), -8, 7).astype(np.int64)
            np.testing.assert_array_equal(q[m, G * g:G * g + G], want)
    assert s[1, 0] == 0 and np.all(q[1, :G] == 0)


@pytest.mark.parametrize("G", [128, 512])
def test_int4_group_gemm_vs_fp64(orc, G):
    """The grouped product equals the fp64 product of the dequantized operands
    (codes times their group's scale, restated here)."""
    M, N, K = 6, 9, 1024
    Xa = synth.activations("qwen25_7b_int4", M, K, seed=73)
    Xw = synth.weights("qwen25_7b_int4", N, K, seed=73)
    ca, sa = orc.quant_int4_g(Xa, G)
    cw, sw = orc.quant_int4_g(Xw, G)

    def deq(c, s):
        q = unpack(c).astype(np.float64)
        q = np.where(q >= 8, q - 16, q)
        return q * np.repeat(s.astype(np.float64), G, axis=1)
    want = deq(ca, sa) @ deq(cw, sw).T
    _, yref, absd = orc.gemm_int4_g(ca, sa, cw, sw, G)
    np.testing.assert_allclose(yref, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert np.all(absd >= np.abs(yref) * (1 - 1e-12))
