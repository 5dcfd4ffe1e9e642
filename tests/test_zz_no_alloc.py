"""The allocation-free NVFP4 entry point (skinny_nvfp4_gemm_static_ws).

Some callers cannot call cudaMalloc: a serving engine that has handed all free
HBM to its own pool, a plugin inside a host framework that gives it no
allocator, or a latency-critical path that must not stall on cudaMalloc's
implicit synchronisation.  For them the library keeps its split-K scratch in a
static device array.  This test calls that entry point through the C ABI two
times in a row (different shapes, so the second call finds the first call's
leftovers in the shared array) and checks each result against the ordinary
entry point with a caller-allocated workspace, within the parity tolerance.

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import synthetic_inputs as si
from parity import REL_TOL, oracle_nvfp4, ulp16

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _call_static(x, w, y):
    out = sk.OUT_F32 if y.dtype == torch.float32 else sk.OUT_F16
    st = sk.library().skinny_nvfp4_gemm_static_ws(
        x.data_ptr(), x.shape[0], w.K, w.data.data_ptr(), ctypes.c_float(w.global_scale), w.N, y.data_ptr(), out,
        torch.cuda.current_stream().cuda_stream)
    assert st == sk.OK, sk.status_string(st)


@pytest.mark.parametrize("first,second", [((5120, 5120, 8, "f16"), (1000, 1040, 3, "f32"))])
def test_static_workspace_matches_allocating_entry_point(first, second):
    for call, (N, K, M, out) in enumerate((first, second)):
        codes, scales = si.nvfp4_weights(N, K, seed=call, cfg_id=70)
        x_np = si.activations(M, K, seed=call, cfg_id=70)
        w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
        x = torch.from_numpy(x_np).to(DEV)
        dt = torch.float32 if out == "f32" else torch.float16
        y_static = torch.full((M, N), float("nan"), dtype=dt, device=DEV)
        _call_static(x, w, y_static)
        ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV)
        y_ref = sk.gemm(x, w, dt, workspace=ws)
        torch.cuda.synchronize()
        a = y_static.double().cpu().numpy()
        b = y_ref.double().cpu().numpy()
        _, bound = oracle_nvfp4(x_np, codes, scales, 0.5)
        tol = REL_TOL * bound
        if out == "f16":
            tol = tol + 0.5 * ulp16(np.maximum(np.abs(a), np.abs(b)))
        assert np.all(np.abs(a - b) <= tol), "call %d (%dx%d M=%d)" % (call, N, K, M)
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
