"""GEMMs fused with a residual add (skinny_nvfp4_gemm_add / skinny_fp8_gemm_add)
against the float64 oracle: y = x . W^T + r.

The kernel adds r to the FP32 output value (the same value the plain GEMM
stores) in FP32 and rounds once to the output type, so with the GEMM parity
bound REL * B:
    |y_gpu - (y + r)| <= REL * B + 2^-23 |y + r|  (+ half an FP16 ulp of y + r).
"""
import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import synthetic_inputs as si
from parity import REL_TOL, oracle_fp8, oracle_nvfp4, sample_rows, ulp16

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert sk.device_error(clear=True) == 0


def residual_like(M, N, dt, seed):
    rng = np.random.default_rng(seed)
    r = rng.normal(0, 50, size=(M, N))
    return r.astype(np.float16 if dt == torch.float16 else np.float32)


def check(y_gpu, want, bound, dt, what):
    tol = REL_TOL * bound + 2.0 ** -23 * np.abs(want)
    if dt == torch.float16:
        tol = tol + 0.5 * ulp16(want)
    err = np.abs(y_gpu - want)
    assert np.all(err <= tol), "%s: max err/tol %g" % (what, float((err / tol).max()))


@pytest.mark.parametrize("M,dt", [(1, torch.float16), (8, torch.float16), (8, torch.float32)])
def test_nvfp4_add_attention_output_shape(M, dt):
    """5120 x 5120 NVFP4 (the attention output projection), FP16 residual stream."""
    N = K = 5120
    codes, scales = si.nvfp4_weights(N, K, seed=0, cfg_id=2)
    x = si.activations(M, K, seed=0, cfg_id=2)
    r = residual_like(M, N, dt, 1)
    w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV)
    y = torch.empty((M, N), dtype=dt, device=DEV)
    sk.gemm_add_into(y, torch.from_numpy(x).to(DEV), w, torch.from_numpy(r).to(DEV), workspace=ws)
    torch.cuda.synchronize()
    rows = sample_rows(N, 600, seed=M)
    yr, b = oracle_nvfp4(x, codes, scales, 0.5, rows)
    check(y.double().cpu().numpy()[:, rows], yr + r[:, rows].astype(np.float64), b, dt, "nvfp4 add M=%d" % M)


def test_fp8_add_in_place_down_projection_shape():
    """5120 x 17408 FP8 (the MLP down projection), residual updated in place."""
    N, K, M = 5120, 17408, 4
    q, s = si.fp8_weights(N, K, seed=0, cfg_id=4)
    x = si.activations(M, K, seed=0, cfg_id=4)
    r = residual_like(M, N, torch.float16, 2)
    w = sk.PackedFP8.from_logical(q, s, DEV)
    ws = sk.make_workspace(sk.FMT_FP8, M, N, K, DEV)
    y = torch.from_numpy(r.copy()).to(DEV)
    sk.gemm_add_into(y, torch.from_numpy(x).to(DEV), w, y, workspace=ws)
    torch.cuda.synchronize()
    rows = sample_rows(N, 600, seed=9)
    yr, b = oracle_fp8(x, q, s, rows)
    check(y.double().cpu().numpy()[:, rows], yr + r[:, rows].astype(np.float64), b, torch.float16, "fp8 add in place")


@pytest.mark.parametrize("split", [True, False])
def test_add_ragged_and_split(split):
    N, K, M = 257, 150016, 3
    codes, scales = si.nvfp4_weights(N, K, seed=14, cfg_id=68)
    x = si.activations(M, K, seed=14, cfg_id=68)
    r = residual_like(M, N, torch.float32, 3)
    w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV) if split else None
    y = torch.empty((M, N), dtype=torch.float32, device=DEV)
    sk.gemm_add_into(y, torch.from_numpy(x).to(DEV), w, torch.from_numpy(r).to(DEV), workspace=ws)
    torch.cuda.synchronize()
    yr, b = oracle_nvfp4(x, codes, scales, 0.5)
    check(y.double().cpu().numpy(), yr + r.astype(np.float64), b, torch.float32, "ragged split=%s" % split)


def test_add_equals_plain_gemm_plus_residual_in_fp32():
    """The fused add is the plain FP32 GEMM output plus r, rounded once."""
    N, K, M = 1000, 2048, 8
    codes, scales = si.nvfp4_weights(N, K, seed=15, cfg_id=69)
    xt = torch.from_numpy(si.activations(M, K, seed=15, cfg_id=69)).to(DEV)
    w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV)
    r = torch.from_numpy(residual_like(M, N, torch.float32, 4)).to(DEV)
    y_plain = sk.gemm(xt, w, torch.float32, workspace=ws)
    y = torch.empty_like(y_plain)
    sk.gemm_add_into(y, xt, w, r, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y_plain + r)


@pytest.mark.parametrize("fmt", ["nvfp4", "fp8"])
@pytest.mark.parametrize("M", [12, 16])
def test_add_with_two_token_blocks(fmt, M):
    """The residual-add kernels for 9 <= M <= 16 (two MMA token blocks), FP16
    in place, split K, ragged N and K."""
    N, K = 700, 1040
    x = si.activations(M, K, seed=M, cfg_id=66)
    r = residual_like(M, N, torch.float16, 30 + M)
    if fmt == "nvfp4":
        codes, scales = si.nvfp4_weights(N, K, seed=M, cfg_id=66)
        w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
        yr, b = oracle_nvfp4(x, codes, scales, 0.5)
        ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV)
    else:
        q, s = si.fp8_weights(N, K, seed=M, cfg_id=66)
        w = sk.PackedFP8.from_logical(q, s, DEV)
        yr, b = oracle_fp8(x, q, s)
        ws = sk.make_workspace(sk.FMT_FP8, M, N, K, DEV)
    y = torch.from_numpy(r.copy()).to(DEV)
    sk.gemm_add_into(y, torch.from_numpy(x).to(DEV), w, y, workspace=ws)
    torch.cuda.synchronize()
    check(y.double().cpu().numpy(), yr + r.astype(np.float64), b, torch.float16, "%s add M=%d" % (fmt, M))
