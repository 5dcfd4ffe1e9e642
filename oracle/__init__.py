"""Float64 CPU oracle for the NVFP4 / FP8 weight-only skinny GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never imports it and it never imports the CUDA library.

The arithmetic lives in ``oracle.c`` (plain C, float64, one pthread per slice
of output rows).  This module compiles it with gcc on first use and wraps it
with ctypes so that numpy arrays can be passed in.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_default = None


def compile_library(src: str = SOURCE, out: str = LIBRARY, force: bool = False) -> str:
    """Compile an oracle source file into a shared library (gcc, -O2, strict FP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-Wall", "-Wextra", src, "-o", tmp, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it."""
    return compile_library(force=force)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _x_bits(x: np.ndarray) -> np.ndarray:
    if x.dtype == np.float16:
        x = x.view(np.uint16)
    if x.dtype != np.uint16 or x.ndim != 2:
        raise TypeError("x must be a 2-D float16 (or uint16 bit pattern) array")
    return np.ascontiguousarray(x)


class Oracle:
    """ctypes wrapper around one compiled copy of oracle.c."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        for name in ("oracle_e2m1", "oracle_e4m3", "oracle_f16"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_double
            fn.argtypes = [ctypes.c_uint]
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_nvfp4_gemm.restype = ctypes.c_int
        lib.oracle_nvfp4_gemm.argtypes = [p, i64, i64, p, p, ctypes.c_float, i64, p, p, ctypes.c_int]
        lib.oracle_fp8_gemm.restype = ctypes.c_int
        lib.oracle_fp8_gemm.argtypes = [p, i64, i64, p, p, i64, p, p, ctypes.c_int]
        self.lib = lib
        self.path = path

    def e2m1(self, code: int) -> float:
        return self.lib.oracle_e2m1(int(code))

    def e4m3(self, byte: int) -> float:
        return self.lib.oracle_e4m3(int(byte))

    def f16(self, bits: int) -> float:
        return self.lib.oracle_f16(int(bits))

    def nvfp4_gemm(self, x, codes, scales, global_scale, threads: int | None = None):
        """y, bound of the NVFP4 GEMM.

        x: [M, K] float16; codes: [N, K/2] uint8 (low nibble = even k);
        scales: [N, K/16] uint8 (UE4M3); global_scale: float32.
        Returns float64 y[M, N] and bound[M, N] = sum_k |w * x|.
        """
        xb = _x_bits(x)
        M, K = xb.shape
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        scales = np.ascontiguousarray(scales, dtype=np.uint8)
        N = codes.shape[0]
        if K % 16 or codes.shape != (N, K // 2) or scales.shape != (N, K // 16):
            raise ValueError("shape mismatch: codes %s scales %s K=%d" % (codes.shape, scales.shape, K))
        y = np.empty((M, N), np.float64)
        b = np.empty((M, N), np.float64)
        rc = self.lib.oracle_nvfp4_gemm(_ptr(xb), M, K, _ptr(codes), _ptr(scales),
                                        float(np.float32(global_scale)), N, _ptr(y), _ptr(b),
                                        threads or default_threads())
        if rc != 0:
            raise RuntimeError("oracle_nvfp4_gemm failed: %d" % rc)
        return y, b

    def fp8_gemm(self, x, q, channel_scale, threads: int | None = None):
        """y, bound of the FP8 (E4M3 + FP32 per-output-channel scale) GEMM.

        x: [M, K] float16; q: [N, K] uint8 (E4M3); channel_scale: [N] float32.
        """
        xb = _x_bits(x)
        M, K = xb.shape
        q = np.ascontiguousarray(q, dtype=np.uint8)
        s = np.ascontiguousarray(channel_scale, dtype=np.float32)
        N = q.shape[0]
        if q.shape != (N, K) or s.shape != (N,):
            raise ValueError("shape mismatch: q %s scale %s K=%d" % (q.shape, s.shape, K))
        y = np.empty((M, N), np.float64)
        b = np.empty((M, N), np.float64)
        rc = self.lib.oracle_fp8_gemm(_ptr(xb), M, K, _ptr(q), _ptr(s), N, _ptr(y), _ptr(b),
                                      threads or default_threads())
        if rc != 0:
            raise RuntimeError("oracle_fp8_gemm failed: %d" % rc)
        return y, b


def load() -> Oracle:
    """The oracle built from oracle.c (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def e2m1(code: int) -> float:
    return load().e2m1(code)


def e4m3(byte: int) -> float:
    return load().e4m3(byte)


def f16(bits: int) -> float:
    return load().f16(bits)


def nvfp4_gemm(x, codes, scales, global_scale, threads: int | None = None):
    return load().nvfp4_gemm(x, codes, scales, global_scale, threads)


def fp8_gemm(x, q, channel_scale, threads: int | None = None):
    return load().fp8_gemm(x, q, channel_scale, threads)


def silu_mul(y_gate_up: np.ndarray) -> np.ndarray:
    """The gated-MLP activation applied to a gate+up GEMM output, in float64.

    y_gate_up is [M][2F]: columns 0..F-1 are the gate pre-activations g, columns
    F..2F-1 the up projections u of the same outputs.  Returns [M][F] with
    silu(g) * u, where silu(z) = z * sigmoid(z) = z / (1 + e^-z) (the SiLU of
    the gated MLP that the gate+up projection feeds).  e^-z overflows to inf
    for very negative z, which gives the limit silu(z) -> -0."""
    y = np.asarray(y_gate_up, dtype=np.float64)
    F = y.shape[1] // 2
    g, u = y[:, :F], y[:, F:]
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * u
