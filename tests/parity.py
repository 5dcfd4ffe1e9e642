"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
binding and compare it with the float64 oracle on the same seeded bytes."""
import numpy as np

import oracle

# |y_gpu - y| <= REL_TOL * sum_k |w_k x_k|  (+ half an FP16 ulp for FP16 output)
REL_TOL = 1e-4


def ulp16(v):
    """Spacing of binary16 numbers at |v| (subnormal spacing 2^-24 below 2^-14)."""
    a = np.abs(np.asarray(v, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -14)
    return np.exp2(e - 10)


def assert_parity(y_gpu, y_ref, bound, out, what=""):
    """Elementwise parity check; out is "f32" or "f16"."""
    y_gpu = np.asarray(y_gpu, np.float64)
    assert y_gpu.shape == y_ref.shape, (y_gpu.shape, y_ref.shape)
    tol = REL_TOL * bound
    if out == "f16":
        big = np.abs(y_ref) >= 65520.0
        if big.any():
            assert np.all(np.isinf(y_gpu[big]) & (np.sign(y_gpu[big]) == np.sign(y_ref[big]))), what
        ok = ~big
        tol = tol + 0.5 * ulp16(np.maximum(np.abs(y_ref), np.abs(np.nan_to_num(y_gpu))))
    else:
        ok = np.ones_like(y_ref, bool)
    err = np.abs(y_gpu - y_ref)
    bad = ok & ~(err <= tol)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError("%s: %d of %d outside tolerance; first at %s: gpu=%r ref=%r tol=%r"
                             % (what, int(bad.sum()), bad.size, tuple(i), y_gpu[tuple(i)], y_ref[tuple(i)],
                                tol[tuple(i)]))
    return float(np.max(np.where(ok, err / np.maximum(bound, 1e-300), 0.0)))


def sample_rows(N, count, seed=0):
    """Row indices to check at full size: both ends, every tile seam nearby, random."""
    if N <= count:
        return np.arange(N)
    rng = np.random.default_rng(seed)
    fixed = np.concatenate([np.arange(min(16, N)), np.arange(max(0, N - 16), N),
                            np.arange(127, N, 128)[:64], np.arange(128, N, 128)[:64]])
    rest = rng.choice(N, size=max(0, count - fixed.size), replace=False)
    return np.unique(np.concatenate([fixed, rest]))


def oracle_nvfp4(x, codes, scales, g, rows=None):
    if rows is not None:
        codes, scales = codes[rows], scales[rows]
    return oracle.nvfp4_gemm(x, codes, scales, g)


def oracle_fp8(x, q, s, rows=None):
    if rows is not None:
        q, s = q[rows], s[rows]
    return oracle.fp8_gemm(x, q, s)
