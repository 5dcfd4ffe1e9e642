"""Grouped NVFP4 GEMM (skinny_nvfp4_gemm_grouped): several independent GEMMs of
one K in one launch.  Every member's output is compared with the float64
oracle element by element at the parity tolerance; a group of one must equal
the single-GEMM entry point bit for bit (same schedule and summation order)."""
import ctypes

import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import synthetic_inputs as si
from parity import assert_parity, oracle_nvfp4

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert sk.device_error(clear=True) == 0


def _members(shapes, K, M, seed, shared_x=False, scale_dist="uniform"):
    """Logical weights, packed weights and activations of each member."""
    out = []
    x_shared = si.activations(M, K, seed=seed, cfg_id=80, tensor_id=500)
    for i, N in enumerate(shapes):
        codes, scales = si.nvfp4_weights(N, K, scale_dist=scale_dist, seed=seed, cfg_id=80, tensor_id=10 * i)
        g = [0.5, 0.25, 1.0, 2.0][i % 4]
        x = x_shared if shared_x else si.activations(M, K, seed=seed, cfg_id=80, tensor_id=100 + i)
        out.append((codes, scales, g, x, sk.PackedNVFP4.from_logical(codes, scales, g, DEV)))
    return out


def _run(mem, out, split):
    M, K = mem[0][3].shape
    dt = torch.float32 if out == "f32" else torch.float16
    xs = [torch.from_numpy(m[3]).to(DEV) for m in mem]
    ws = [m[4] for m in mem]
    ys = [torch.full((M, w.N), float("nan"), dtype=dt, device=DEV) for w in ws]
    wsp = sk.make_workspace(sk.FMT_NVFP4, M, max(w.N for w in ws), K, DEV) if split else None
    sk.gemm_grouped_into(ys, xs, ws, workspace=wsp)
    torch.cuda.synchronize()
    return [y.double().cpu().numpy() for y in ys]


@pytest.mark.parametrize("M", [1, 8])
def test_three_attention_projections_5120(M):
    """q, kv and o projections (5120 x 5120 each, own activations) in one launch."""
    mem = _members([5120, 5120, 5120], 5120, M, seed=0)
    ys = _run(mem, "f16", True)
    for i, ((codes, scales, g, x, _), y) in enumerate(zip(mem, ys)):
        yr, b = oracle_nvfp4(x, codes, scales, g)
        assert_parity(y, yr, b, "f16", "member %d M=%d" % (i, M))


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("M", [1, 3, 8])
def test_ragged_members(M, split):
    """Members of different N (ragged row tiles), one K with a ragged tail."""
    mem = _members([300, 1000, 17, 129], 1040, M, seed=M)
    for out in ("f32", "f16"):
        ys = _run(mem, out, split)
        for i, ((codes, scales, g, x, _), y) in enumerate(zip(mem, ys)):
            yr, b = oracle_nvfp4(x, codes, scales, g)
            assert_parity(y, yr, b, out, "member %d M=%d %s split=%s" % (i, M, out, split))


def test_shared_activations_and_max_group():
    """Eight members reading the same x (q/k/v style), loguniform scales."""
    mem = _members([128, 256, 64, 500, 5, 1024, 640, 200], 2048, 4, seed=9, shared_x=True,
                   scale_dist="loguniform")
    ys = _run(mem, "f32", True)
    for i, ((codes, scales, g, x, _), y) in enumerate(zip(mem, ys)):
        yr, b = oracle_nvfp4(x, codes, scales, g)
        assert_parity(y, yr, b, "f32", "member %d" % i)


@pytest.mark.parametrize("split", [True, False])
def test_group_of_one_is_the_single_gemm(split):
    mem = _members([5120], 5120, 8, seed=3)
    y_grouped = _run(mem, "f32", split)[0]
    codes, scales, g, x, w = mem[0]
    xt = torch.from_numpy(x).to(DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, 8, 5120, 5120, DEV) if split else None
    y_single = sk.gemm(xt, w, torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert np.array_equal(y_grouped, y_single.double().cpu().numpy())


def test_grouped_is_deterministic():
    mem = _members([5120, 3000, 5120], 5120, 8, seed=4)
    a = _run(mem, "f32", True)
    b = _run(mem, "f32", True)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))


def test_grouped_rejects_bad_groups():
    lib = sk.library()
    mem = _members([256], 512, 1, seed=5)
    x = torch.from_numpy(mem[0][3]).to(DEV)
    y = torch.empty((1, 256), dtype=torch.float32, device=DEV)
    arr = (sk.GroupMember * 9)(*[sk.GroupMember(x.data_ptr(), mem[0][4].data.data_ptr(), 1.0, 256, y.data_ptr())
                                 for _ in range(9)])
    st = torch.cuda.current_stream().cuda_stream
    assert lib.skinny_nvfp4_gemm_grouped(arr, 9, 1, 512, sk.OUT_F32, None, 0, st) == sk.ERR_UNSUPPORTED
    assert lib.skinny_nvfp4_gemm_grouped(arr, 0, 1, 512, sk.OUT_F32, None, 0, st) == sk.ERR_INVALID_ARG
    arr[1].x = x.data_ptr() + 2
    assert lib.skinny_nvfp4_gemm_grouped(arr, 2, 1, 512, sk.OUT_F32, None, 0, st) == sk.ERR_ALIGNMENT
    arr[1].x = None
    assert lib.skinny_nvfp4_gemm_grouped(arr, 2, 1, 512, sk.OUT_F32, None, 0, st) == sk.ERR_INVALID_ARG
    assert lib.skinny_nvfp4_gemm_grouped(ctypes.cast(None, ctypes.POINTER(sk.GroupMember)), 1, 1, 512,
                                         sk.OUT_F32, None, 0, st) == sk.ERR_INVALID_ARG
