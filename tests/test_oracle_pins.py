"""Pins of the float64 oracle against things other than itself.

Each test ties one part of ``oracle.c`` to a fixed outside fact: a printed
format table (tests/golden/), a library decoder (numpy, torch, ml_dtypes),
exact rational arithmetic on tiny shapes, or an invariant that the
mathematics of y = x . W^T fixes.  ``test_oracle_mutants.py`` checks that a
plausible slip anywhere in oracle.c trips at least one of these.
"""
from fractions import Fraction
import math

import numpy as np
import pytest
import torch

from conftest import read_golden

import oracle

ml_dtypes = pytest.importorskip("ml_dtypes")


# --------------------------------------------------------------------------
# Scalar decoders
# --------------------------------------------------------------------------

def test_e2m1_matches_printed_table(orc):
    rows = read_golden("e2m1_table.txt")
    assert len(rows) == 16
    for code_s, val_s in rows:
        code, want = int(code_s, 16), float(val_s)
        got = orc.e2m1(code)
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (code, got, want)


def test_e2m1_matches_ml_dtypes():
    import oracle

    orc = oracle.load()
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        assert orc.e2m1(c) == lib[c]


def test_e4m3_all_codes_match_torch_and_ml_dtypes(orc):
    b = np.arange(256, dtype=np.uint8)
    via_torch = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    via_mld = b.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for i in range(256):
        got = orc.e4m3(i)
        if math.isnan(via_torch[i]):
            assert math.isnan(got) and math.isnan(via_mld[i]), i
            assert i in (0x7F, 0xFF)
        else:
            assert got == via_torch[i] == via_mld[i], (i, got, via_torch[i])
            assert math.copysign(1.0, got) == math.copysign(1.0, via_torch[i])


def test_e4m3_matches_printed_special_values(orc):
    for byte_s, val_s in read_golden("e4m3_special.txt"):
        got = orc.e4m3(int(byte_s, 16))
        if val_s == "nan":
            assert math.isnan(got)
        else:
            want = float(val_s)
            assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), byte_s


def test_f16_all_bit_patterns_match_numpy(orc):
    bits = np.arange(65536, dtype=np.uint32)
    ref = bits.astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([orc.f16(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# --------------------------------------------------------------------------
# Independent exact decoders for the GEMM pins (built from the printed tables
# and from library casts, not from oracle.c)
# --------------------------------------------------------------------------

E2M1 = {int(c, 16): Fraction(float(v)) for c, v in read_golden("e2m1_table.txt")}


def e4m3_frac(byte):
    v = torch.tensor([byte], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).item()
    return Fraction(v)


def nvfp4_dense_exact(codes, scales, g):
    """W[n][k] as exact Fractions from the golden E2M1 table and torch's E4M3."""
    N, K2 = codes.shape
    K = 2 * K2
    W = [[None] * K for _ in range(N)]
    gf = Fraction(float(np.float32(g)))
    for n in range(N):
        for k in range(K):
            byte = int(codes[n, k // 2])
            code = byte & 0xF if k % 2 == 0 else byte >> 4
            W[n][k] = E2M1[code] * e4m3_frac(int(scales[n, k // 16])) * gf
    return W


def fp8_dense_exact(q, s):
    N, K = q.shape
    return [[e4m3_frac(int(q[n, k])) * Fraction(float(s[n])) for k in range(K)] for n in range(N)]


def exact_gemm(x, W):
    """Exact rational y = x . W^T and B = sum |w x|."""
    xf = [[Fraction(float(v)) for v in row] for row in x.astype(np.float64)]
    M, N, K = len(xf), len(W), len(W[0])
    y = [[sum(xf[m][k] * W[n][k] for k in range(K)) for n in range(N)] for m in range(M)]
    b = [[sum(abs(xf[m][k] * W[n][k]) for k in range(K)) for n in range(N)] for m in range(M)]
    return y, b


def assert_close_to_exact(y, b, y_ex, b_ex, K):
    """The oracle's only rounding is a K-term float64 sum of exact products:
    |fl(sum) - sum| <= (K-1) * 2^-53 * sum|p| (with slack for the same on B)."""
    M, N = y.shape
    for m in range(M):
        for n in range(N):
            bound = float(b_ex[m][n]) * K * 2.0 ** -52
            assert abs(Fraction(float(y[m, n])) - y_ex[m][n]) <= Fraction(bound), (m, n)
            assert abs(Fraction(float(b[m, n])) - b_ex[m][n]) <= Fraction(bound), (m, n)


def _tiny_nvfp4(rng, M, N, K):
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    # every scale byte class: subnormal, normal, large, zero
    scales = rng.choice(np.array([0x00, 0x01, 0x07, 0x08, 0x18, 0x38, 0x3F, 0x58, 0x7E], np.uint8),
                        size=(N, K // 16))
    x = (rng.standard_normal((M, K)) * 3).astype(np.float16)
    return x, codes, scales


@pytest.mark.parametrize("M,N,K,g", [(1, 3, 16, 0.5), (3, 4, 32, 3.0), (8, 2, 48, 1.0 / 448.0),
                                     (2, 1, 64, 1.0)])
def test_nvfp4_gemm_matches_exact_rationals(orc, M, N, K, g):
    rng = np.random.default_rng(1000 + M * 100 + N * 10 + K)
    x, codes, scales = _tiny_nvfp4(rng, M, N, K)
    y, b = orc.nvfp4_gemm(x, codes, scales, g, threads=2)
    y_ex, b_ex = exact_gemm(x, nvfp4_dense_exact(codes, scales, g))
    assert_close_to_exact(y, b, y_ex, b_ex, K)


@pytest.mark.parametrize("M,N,K", [(1, 3, 16), (4, 3, 40), (8, 2, 24)])
def test_fp8_gemm_matches_exact_rationals(orc, M, N, K):
    rng = np.random.default_rng(2000 + M * 100 + N * 10 + K)
    q = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x42  # no NaN codes
    s = (rng.random(N) * 0.01 + 1e-3).astype(np.float32)
    x = (rng.standard_normal((M, K)) * 2).astype(np.float16)
    y, b = orc.fp8_gemm(x, q, s, threads=3)
    y_ex, b_ex = exact_gemm(x, fp8_dense_exact(q, s))
    assert_close_to_exact(y, b, y_ex, b_ex, K)


def test_nvfp4_subnormal_x_is_honoured(orc):
    """x = smallest binary16 subnormal, w = 1 (code 2, scale 1.0): y = 2^-24."""
    K = 16
    x = np.zeros((1, K), np.uint16)
    x[0, 5] = 0x0001
    codes = np.zeros((1, K // 2), np.uint8)
    codes[0, 2] = 0x20  # element k=5 is the high nibble of byte 2 -> code 2 (1.0)
    scales = np.full((1, 1), 0x38, np.uint8)
    y, b = orc.nvfp4_gemm(x, codes, scales, 1.0, threads=1)
    assert y[0, 0] == 2.0 ** -24 and b[0, 0] == 2.0 ** -24


# --------------------------------------------------------------------------
# Invariants at sizes the brute force cannot reach
# --------------------------------------------------------------------------

def _nvfp4_case(seed, M=8, N=37, K=256):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = rng.integers(0x18, 0x59, size=(N, K // 16), dtype=np.uint8)
    x = rng.standard_normal((M, K)).astype(np.float16)
    return x, codes, scales


def _dense_library(codes, scales, g):
    """W decoded with library casts (ml_dtypes E2M1, torch E4M3), float64."""
    N, K2 = codes.shape
    lo = (codes & 0xF).astype(np.uint8)
    hi = (codes >> 4).astype(np.uint8)
    nib = np.stack([lo, hi], axis=-1).reshape(N, 2 * K2)
    e2 = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sc = torch.from_numpy(scales).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return e2 * np.repeat(sc, 16, axis=1) * float(np.float32(g))


def test_one_hot_extracts_each_weight(orc):
    x0, codes, scales = _nvfp4_case(7, M=1, N=19, K=64)
    W = _dense_library(codes, scales, 0.5)
    K = 64
    x = np.zeros((8, K), np.float16)
    ks = [0, 1, 15, 16, 17, 33, 62, 63]
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    y, _ = orc.nvfp4_gemm(x, codes, scales, 0.5, threads=2)
    for m, k in enumerate(ks):
        assert np.array_equal(y[m], W[:, k]), k


def test_second_implementation_numpy_matmul(orc):
    x, codes, scales = _nvfp4_case(11, M=8, N=53, K=512)
    g = 1.0 / 448.0
    y, b = orc.nvfp4_gemm(x, codes, scales, g, threads=4)
    ref = x.astype(np.float64) @ _dense_library(codes, scales, g).T
    assert np.all(np.abs(y - ref) <= 1e-12 * b + 1e-300)


def test_fp8_second_implementation(orc):
    rng = np.random.default_rng(5)
    N, K = 29, 320
    q = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x01
    s = rng.random(N).astype(np.float32) + np.float32(0.25)
    x = rng.standard_normal((4, K)).astype(np.float16)
    y, b = orc.fp8_gemm(x, q, s, threads=3)
    W = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy() * s.astype(np.float64)[:, None]
    ref = x.astype(np.float64) @ W.T
    assert np.all(np.abs(y - ref) <= 1e-12 * b)


def test_row_independence_is_bitwise(orc):
    x, codes, scales = _nvfp4_case(3)
    y8, _ = orc.nvfp4_gemm(x, codes, scales, 0.5, threads=4)
    for m in range(8):
        y1, _ = orc.nvfp4_gemm(x[m:m + 1], codes, scales, 0.5, threads=4)
        assert np.array_equal(y1[0], y8[m])


def test_power_of_two_scaling_is_exact(orc):
    x, codes, scales = _nvfp4_case(4, M=2)
    y, _ = orc.nvfp4_gemm(x, codes, scales, 0.5, threads=2)
    y4, _ = orc.nvfp4_gemm((x.astype(np.float32) * 4).astype(np.float16), codes, scales, 0.5, threads=2)
    assert np.array_equal(y4, 4 * y)
    yg, _ = orc.nvfp4_gemm(x, codes, scales, 2.0, threads=2)
    assert np.array_equal(yg, 4 * y)


def test_linearity_in_x(orc):
    rng = np.random.default_rng(9)
    _, codes, scales = _nvfp4_case(9, M=1)
    K = 256
    x1 = rng.integers(-8, 9, size=(3, K)).astype(np.float16)
    x2 = rng.integers(-8, 9, size=(3, K)).astype(np.float16)
    y1, b1 = orc.nvfp4_gemm(x1, codes, scales, 1.0)
    y2, b2 = orc.nvfp4_gemm(x2, codes, scales, 1.0)
    y12, _ = orc.nvfp4_gemm((x1.astype(np.float32) + x2).astype(np.float16), codes, scales, 1.0)
    assert np.all(np.abs(y12 - (y1 + y2)) <= 1e-13 * (b1 + b2))


def test_zero_scale_removes_block(orc):
    x, codes, scales = _nvfp4_case(12, M=2, N=5, K=64)
    s2 = scales.copy()
    s2[:, 1] = 0
    y, _ = orc.nvfp4_gemm(x, codes, s2, 1.0)
    xz = x.copy()
    xz[:, 16:32] = 0
    yz, _ = orc.nvfp4_gemm(xz, codes, scales, 1.0)
    assert np.array_equal(y, yz)


def test_block_permutation_of_k(orc):
    """Permuting whole 16-element K blocks in W (codes and scales) and in x
    together leaves y unchanged up to the order of the float64 sum."""
    x, codes, scales = _nvfp4_case(13, M=3, N=11, K=128)
    perm = np.random.default_rng(0).permutation(8)
    cp = codes.reshape(11, 8, 8)[:, perm].reshape(11, 64)
    sp = scales[:, perm]
    xp = x.reshape(3, 8, 16)[:, perm].reshape(3, 128)
    y, b = orc.nvfp4_gemm(x, codes, scales, 0.5)
    yp, _ = orc.nvfp4_gemm(xp, cp, sp, 0.5)
    assert np.all(np.abs(y - yp) <= 128 * 2.0 ** -52 * b)


def test_threads_do_not_change_result(orc):
    x, codes, scales = _nvfp4_case(14, M=4, N=101)
    y1, b1 = orc.nvfp4_gemm(x, codes, scales, 0.5, threads=1)
    y7, b7 = orc.nvfp4_gemm(x, codes, scales, 0.5, threads=7)
    assert np.array_equal(y1, y7) and np.array_equal(b1, b7)


def test_bad_arguments_raise(orc):
    x = np.zeros((1, 24), np.float16)
    with pytest.raises(ValueError):
        orc.nvfp4_gemm(x, np.zeros((1, 12), np.uint8), np.zeros((1, 1), np.uint8), 1.0)


# ---------------------------------------------------------------------------
# silu_mul: the gated-MLP activation on a gate+up output (fused SiLU*mul row)
# ---------------------------------------------------------------------------

def test_silu_mul_closed_forms():
    """sigmoid(ln 3) = 3/4 exactly, so silu(ln 3) * u = 0.75 ln 3 * u; silu(0) = 0;
    silu(z) -> z for large z and -> -0 for very negative z (no overflow NaN)."""
    import math

    z = np.array([[math.log(3.0), 0.0, 60.0, -800.0, 2.0, 2.0, 2.0, -3.0]])
    h = oracle.silu_mul(z)
    assert abs(h[0, 0] - 0.75 * math.log(3.0) * 2.0) < 1e-15
    assert h[0, 1] == 0.0
    assert abs(h[0, 2] - 60.0 * 2.0) < 1e-12
    assert h[0, 3] == 0.0 and not np.isnan(h[0, 3])


def test_silu_mul_identities():
    """silu(z) - silu(-z) = z (sigmoid(z) + sigmoid(-z) = 1); linear in u;
    gate and up are not interchangeable (a swapped operand fails)."""
    rng = np.random.default_rng(3)
    g = rng.normal(0, 4, size=(4, 64))
    one = np.ones_like(g)
    a = oracle.silu_mul(np.concatenate([g, one], axis=1))
    b = oracle.silu_mul(np.concatenate([-g, one], axis=1))
    assert np.allclose(a - b, g, rtol=0, atol=1e-12)
    u = rng.normal(0, 1, size=g.shape)
    h1 = oracle.silu_mul(np.concatenate([g, u], axis=1))
    h3 = oracle.silu_mul(np.concatenate([g, 3 * u], axis=1))
    assert np.allclose(h3, 3 * h1, rtol=1e-15, atol=0)
    swapped = oracle.silu_mul(np.concatenate([u, g], axis=1))
    assert not np.allclose(swapped, h1)


def test_silu_mul_matches_torch_silu():
    """A second implementation: torch.nn.functional.silu in float64."""
    import torch

    rng = np.random.default_rng(4)
    g = rng.normal(0, 6, size=(3, 128))
    u = rng.normal(0, 1, size=(3, 128))
    want = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    got = oracle.silu_mul(np.concatenate([g, u], axis=1))
    assert np.allclose(got, want, rtol=1e-14, atol=1e-300)
