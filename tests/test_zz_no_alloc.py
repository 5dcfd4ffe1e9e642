"""The allocation-free NVFP4 entry point (skinny_nvfp4_gemm_static_ws).

Some callers cannot call cudaMalloc: a serving engine that has handed all free
HBM to its own pool, a plugin inside a host framework that gives it no
allocator, or a latency-critical path that must not stall on cudaMalloc's
implicit synchronisation.  For them the library keeps its split-K scratch in a
static device array.

This test calls that entry point through the C ABI two times in a row, with
different shapes.  Between the calls it fills the whole static array with
non-zero bytes, so that the second call runs only if its own clear of the
scratch works: a stale "published" partial sum would otherwise be added into
its outputs.  Each result must equal, bit for bit, the ordinary entry point's
output with a caller-allocated workspace (same kernel, same split-K schedule,
same summation order), and must match the float64 oracle element by element
at the parity tolerance.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import synthetic_inputs as si
from parity import assert_parity, oracle_nvfp4

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _call_static(x, w, y):
    out = sk.OUT_F32 if y.dtype == torch.float32 else sk.OUT_F16
    st = sk.library().skinny_nvfp4_gemm_static_ws(
        x.data_ptr(), x.shape[0], w.K, w.data.data_ptr(), ctypes.c_float(w.global_scale), w.N, y.data_ptr(), out,
        torch.cuda.current_stream().cuda_stream)
    assert st == sk.OK, sk.status_string(st)


def _poison_static_array(byte: int):
    """Overwrite the whole static scratch array on the current device."""
    from cuda.bindings import runtime as cudart

    addr = ctypes.c_void_p(0)
    st = sk.library().skinny_debug_static_workspace_address(ctypes.byref(addr))
    assert st == sk.OK and addr.value, sk.status_string(st)
    torch.cuda.synchronize()
    (err,) = cudart.cudaMemset(addr.value, byte, sk.library().skinny_static_workspace_capacity())
    assert err == cudart.cudaError_t.cudaSuccess, err
    torch.cuda.synchronize()


@pytest.mark.parametrize("first,second", [((5120, 5120, 8, "f16"), (1000, 1040, 3, "f32"))])
def test_static_workspace_matches_oracle_and_allocating_entry_point(first, second):
    for call, (N, K, M, out) in enumerate((first, second)):
        codes, scales = si.nvfp4_weights(N, K, seed=call, cfg_id=70)
        x_np = si.activations(M, K, seed=call, cfg_id=70)
        w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
        x = torch.from_numpy(x_np).to(DEV)
        dt = torch.float32 if out == "f32" else torch.float16
        if call == 1:
            _poison_static_array(0x5A)
        y_static = torch.full((M, N), float("nan"), dtype=dt, device=DEV)
        _call_static(x, w, y_static)
        ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV)
        y_alloc = sk.gemm(x, w, dt, workspace=ws)
        torch.cuda.synchronize()
        a = y_static.double().cpu().numpy()
        b = y_alloc.double().cpu().numpy()
        assert np.array_equal(a, b), "call %d (%dx%d M=%d): static-scratch output differs from the " \
                                     "workspace entry point's" % (call, N, K, M)
        y_ref, bound = oracle_nvfp4(x_np, codes, scales, 0.5)
        assert_parity(a, y_ref, bound, out, "static scratch, call %d (%dx%d M=%d)" % (call, N, K, M))
    assert sk.device_error(clear=True) == 0


def test_static_workspace_rejects_oversized_shape():
    cap = sk.library().skinny_static_workspace_capacity()
    assert cap == 4 << 20
    # 2^23 row tiles x 2^21 K tiles: more tiles than the kernel's schedule can
    # index.  The call is refused before anything touches the (fake) pointers.
    big = 1 << 30
    st = sk.library().skinny_nvfp4_gemm_static_ws(1 << 20, 1, big, 1 << 20, ctypes.c_float(1.0), big, 1 << 20,
                                                  sk.OUT_F32, None)
    assert st == sk.ERR_UNSUPPORTED
