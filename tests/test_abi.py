"""The C-ABI library loads and exports every function include/skinny.h declares;
argument checks that run before any CUDA call return the documented status."""
import ctypes
import os
import re

import numpy as np
import pytest

import fp8_weight_only_w4a16_b200 as sk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(skinny_\w+)\s*\(", text, flags=re.M)
    return names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    lib = ctypes.CDLL(sk.LIBRARY_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings():
    assert sk.status_string(0) == "SKINNY_OK"
    assert sk.status_string(-3) == "SKINNY_ERR_ALIGNMENT"
    assert sk.status_string(-99) == "SKINNY_ERR_UNKNOWN"
    assert sk.library().skinny_version() >= 100


ALIGNED = 1 << 20  # a fake, 16-byte aligned address: never dereferenced by these checks


@pytest.mark.parametrize("kw,status", [
    (dict(x=None), sk.ERR_INVALID_ARG),
    (dict(y=None), sk.ERR_INVALID_ARG),
    (dict(w=None), sk.ERR_INVALID_ARG),
    (dict(M=0), sk.ERR_UNSUPPORTED),
    (dict(M=17), sk.ERR_UNSUPPORTED),
    (dict(K=24), sk.ERR_INVALID_ARG),
    (dict(K=0), sk.ERR_INVALID_ARG),
    (dict(N=0), sk.ERR_INVALID_ARG),
    (dict(out=7), sk.ERR_INVALID_ARG),
    (dict(x=ALIGNED + 8), sk.ERR_ALIGNMENT),
    (dict(w=ALIGNED + 4), sk.ERR_ALIGNMENT),
    (dict(ws=ALIGNED + 8), sk.ERR_ALIGNMENT),
])
def test_nvfp4_argument_checks(kw, status):
    a = dict(x=ALIGNED, M=1, K=64, w=ALIGNED, N=32, y=ALIGNED, out=0, ws=None)
    a.update(kw)
    st = sk.library().skinny_nvfp4_gemm(a["x"], a["M"], a["K"], a["w"], 1.0, a["N"], a["y"], a["out"],
                                        a["ws"], 0, None)
    assert st == status


@pytest.mark.parametrize("kw,status", [
    (dict(scale=None), sk.ERR_INVALID_ARG),
    (dict(scale=ALIGNED + 2), sk.ERR_ALIGNMENT),
    (dict(M=17), sk.ERR_UNSUPPORTED),
])
def test_fp8_argument_checks(kw, status):
    a = dict(x=ALIGNED, M=2, K=64, w=ALIGNED, scale=ALIGNED, N=32, y=ALIGNED)
    a.update(kw)
    st = sk.library().skinny_fp8_gemm(a["x"], a["M"], a["K"], a["w"], a["scale"], a["N"], a["y"], 0, None, 0, None)
    assert st == status


def test_workspace_query_argument_checks():
    b = ctypes.c_size_t(0)
    lib = sk.library()
    assert lib.skinny_workspace_bytes(5, 1, 64, 64, ctypes.byref(b)) == sk.ERR_INVALID_ARG
    assert lib.skinny_workspace_bytes(0, 1, 64, 40, ctypes.byref(b)) == sk.ERR_INVALID_ARG
    assert lib.skinny_workspace_bytes(0, 17, 64, 64, ctypes.byref(b)) == sk.ERR_UNSUPPORTED
    assert lib.skinny_workspace_bytes(0, 1, 64, 64, None) == sk.ERR_INVALID_ARG


@pytest.mark.parametrize("kw,status", [
    (dict(idx=None), sk.ERR_INVALID_ARG),
    (dict(val=None), sk.ERR_INVALID_ARG),
    (dict(w=None), sk.ERR_INVALID_ARG),
    (dict(M=17), sk.ERR_UNSUPPORTED),
    (dict(K=40), sk.ERR_INVALID_ARG),
    (dict(idx=ALIGNED + 2), sk.ERR_ALIGNMENT),
    (dict(val=ALIGNED + 2), sk.ERR_ALIGNMENT),
    (dict(ws=None), sk.ERR_WORKSPACE),
])
def test_nvfp4_argmax_argument_checks(kw, status):
    a = dict(x=ALIGNED, M=1, K=64, w=ALIGNED, N=32, idx=ALIGNED, val=ALIGNED, ws=ALIGNED)
    a.update(kw)
    st = sk.library().skinny_nvfp4_gemm_argmax(a["x"], a["M"], a["K"], a["w"], 1.0, a["N"], a["idx"], a["val"],
                                               a["ws"], 1 << 20, None)
    assert st == status


@pytest.mark.parametrize("kw,status", [
    (dict(F=96), sk.ERR_INVALID_ARG),
    (dict(F=0), sk.ERR_INVALID_ARG),
    (dict(y=None), sk.ERR_INVALID_ARG),
    (dict(w=None), sk.ERR_INVALID_ARG),
    (dict(M=17), sk.ERR_UNSUPPORTED),
    (dict(out=5), sk.ERR_INVALID_ARG),
    (dict(w=ALIGNED + 4), sk.ERR_ALIGNMENT),
])
def test_nvfp4_silu_mul_argument_checks(kw, status):
    a = dict(x=ALIGNED, M=2, K=64, w=ALIGNED, F=64, y=ALIGNED, out=0)
    a.update(kw)
    st = sk.library().skinny_nvfp4_gemm_silu_mul(a["x"], a["M"], a["K"], a["w"], 1.0, a["F"], a["y"], a["out"],
                                                 None, 0, None)
    assert st == status


@pytest.mark.parametrize("fmt", ["nvfp4", "fp8"])
@pytest.mark.parametrize("kw,status", [
    (dict(res=None), sk.ERR_INVALID_ARG),
    (dict(res=ALIGNED + 2), sk.ERR_ALIGNMENT),
    (dict(y=None), sk.ERR_INVALID_ARG),
    (dict(M=17), sk.ERR_UNSUPPORTED),
])
def test_gemm_add_argument_checks(fmt, kw, status):
    a = dict(x=ALIGNED, M=2, K=64, w=ALIGNED, N=32, res=ALIGNED, y=ALIGNED)
    a.update(kw)
    lib = sk.library()
    if fmt == "nvfp4":
        st = lib.skinny_nvfp4_gemm_add(a["x"], a["M"], a["K"], a["w"], 1.0, a["N"], a["res"], a["y"], 0, None, 0, None)
    else:
        st = lib.skinny_fp8_gemm_add(a["x"], a["M"], a["K"], a["w"], ALIGNED, a["N"], a["res"], a["y"], 0, None, 0,
                                     None)
    assert st == status


def test_binding_rejects_bad_arguments_before_calling_the_library():
    """The Python binding's own checks (no GPU, no library call)."""
    import torch

    w = sk.PackedNVFP4(torch.zeros(36864, dtype=torch.uint8), 1.0, 128, 512)
    gu = sk.PackedGateUp(torch.zeros(36864, dtype=torch.uint8), 1.0, 64, 512)
    assert gu.N == 128 and gu.fmt == sk.FMT_NVFP4
    x32 = torch.zeros((2, 512), dtype=torch.float32)
    x16 = torch.zeros((2, 512), dtype=torch.float16)
    with pytest.raises(ValueError):
        sk.gemm_into(torch.zeros((2, 128), dtype=torch.float16), x32, w)
    with pytest.raises(ValueError):
        sk.gemm_into(torch.zeros((2, 64), dtype=torch.float16), x16, w)
    with pytest.raises(TypeError):
        sk.gemm_silu_mul_into(torch.zeros((2, 64), dtype=torch.float16), x16, w)
    with pytest.raises(ValueError):
        sk.gemm_argmax_into(torch.zeros(2, dtype=torch.int64), torch.zeros(2), x16, w, None)
    with pytest.raises(ValueError):
        sk.gemm_add_into(torch.zeros((2, 128), dtype=torch.float16), x16, w, torch.zeros((2, 128)))
    with pytest.raises(ValueError):
        sk.pack_nvfp4_gate_up(np.zeros((127, 256), np.uint8), np.zeros((127, 32), np.uint8))


def test_library_sources_allocate_no_device_memory():
    """The weights are never dequantised into a full copy: the library makes
    no device allocation at all (every buffer is the caller's, and the one
    static array is the documented split-K scratch of the allocation-free
    entry point)."""
    csrc = os.path.join(ROOT, "fp8_weight_only_w4a16_b200", "csrc")
    calls = re.compile(r"\b(cudaMalloc\w*|cudaMallocAsync|cudaMallocManaged|cudaMallocPitch|cuMemAlloc\w*|cuMemCreate|"
                       r"cudaHostAlloc|malloc|new\s+\w+\s*\[)\s*\(?")
    for name in sorted(os.listdir(csrc)):
        text = open(os.path.join(csrc, name)).read()
        code = re.sub(r"//[^\n]*|/\*.*?\*/", "", text, flags=re.S)
        assert not calls.search(code), (name, calls.search(code).group(0))
    skinny_cu = open(os.path.join(csrc, "skinny.cu")).read()
    assert len(re.findall(r"static __device__ __align__\(256\) unsigned char g_static_workspace", skinny_cu)) == 1


def _group(n, **kw):
    a = dict(x=ALIGNED, w=ALIGNED, g=1.0, N=256, y=ALIGNED)
    a.update(kw)
    arr = (sk.GroupMember * max(n, 1))()
    for i in range(n):
        arr[i] = sk.GroupMember(a["x"], a["w"], a["g"], a["N"], a["y"])
    return arr


@pytest.mark.parametrize("count,kw,status", [
    (0, {}, sk.ERR_INVALID_ARG),
    (9, {}, sk.ERR_UNSUPPORTED),
    (2, dict(x=None), sk.ERR_INVALID_ARG),
    (2, dict(w=None), sk.ERR_INVALID_ARG),
    (2, dict(y=None), sk.ERR_INVALID_ARG),
    (2, dict(N=0), sk.ERR_INVALID_ARG),
    (2, dict(x=ALIGNED + 8), sk.ERR_ALIGNMENT),
    (2, dict(w=ALIGNED + 4), sk.ERR_ALIGNMENT),
    (2, dict(y=ALIGNED + 2), sk.ERR_ALIGNMENT),
])
def test_grouped_argument_checks(count, kw, status):
    """Rejected before any CUDA call (the pointers are fake)."""
    arr = _group(count, **kw)
    st = sk.library().skinny_nvfp4_gemm_grouped(arr, count, 1, 512, sk.OUT_F32, None, 0, None)
    assert st == status, sk.status_string(st)


def test_grouped_rejects_bad_m_k_and_dtype():
    arr = _group(2)
    lib = sk.library()
    assert lib.skinny_nvfp4_gemm_grouped(arr, 2, 17, 512, sk.OUT_F32, None, 0, None) == sk.ERR_UNSUPPORTED
    assert lib.skinny_nvfp4_gemm_grouped(arr, 2, 1, 520, sk.OUT_F32, None, 0, None) == sk.ERR_INVALID_ARG
    assert lib.skinny_nvfp4_gemm_grouped(arr, 2, 1, 512, 3, None, 0, None) == sk.ERR_INVALID_ARG
    assert lib.skinny_nvfp4_gemm_grouped(None, 2, 1, 512, sk.OUT_F32, None, 0, None) == sk.ERR_INVALID_ARG


@pytest.mark.parametrize("buf, nbytes, method, status", [
    (None, 1 << 20, 0, "SKINNY_ERR_INVALID_ARG"),        # no buffer
    (ALIGNED, 8, 0, "SKINNY_ERR_INVALID_ARG"),           # fewer than 16 bytes
    (ALIGNED, 1 << 20, 2, "SKINNY_ERR_INVALID_ARG"),     # no such method
    (ALIGNED + 4, 1 << 20, 1, "SKINNY_ERR_ALIGNMENT"),   # not 16-byte aligned
])
def test_stream_read_argument_checks(buf, nbytes, method, status):
    """The read-only ceiling kernels validate their arguments before any CUDA call."""
    lib = sk.library()
    st = lib.skinny_stream_read(buf, nbytes, method, None, None)
    assert sk.status_string(st) == status
