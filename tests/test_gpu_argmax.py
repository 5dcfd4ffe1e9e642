"""The NVFP4 GEMM fused with a per-token argmax (skinny_nvfp4_gemm_argmax).

Two references for every case:
  * the library's own FP32-output GEMM on the same inputs and workspace: the
    fused kernel runs the same schedule and summation order, so its (row,
    value) must equal the argmax of that y BITWISE (first row among ties,
    NaN counted as the largest, as torch.argmax);
  * the float64 oracle: the chosen row's oracle value must lie within the
    parity tolerance of the oracle's maximum (several rows can be correct
    when outputs are within rounding of each other), and the returned value
    must match the oracle's value of that row within tolerance.
"""
import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import synthetic_inputs as si
from parity import REL_TOL, oracle_nvfp4

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert sk.device_error(clear=True) == 0


def fused_and_plain(x_np, codes, scales, g, ws=None):
    w = sk.PackedNVFP4.from_logical(codes, scales, g, DEV)
    x = torch.from_numpy(x_np).to(DEV)
    if ws is None:
        ws = sk.make_workspace(sk.FMT_NVFP4, x.shape[0], w.N, w.K, DEV)
    idx, val = sk.gemm_argmax(x, w, ws)
    y = sk.gemm(x, w, torch.float32, workspace=ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy(), y, ws


def check_against_plain(idx, val, y):
    """(idx, val) equal the first-occurrence argmax of y (NaN the largest) and
    its value, bit for bit (a NaN as a NaN; -0.0 and +0.0 as equal)."""
    y = y.cpu().numpy()
    for m in range(y.shape[0]):
        row = y[m]
        nan = np.isnan(row)
        ref = int(np.argmax(nan)) if nan.any() else int(np.argmax(row))
        assert idx[m] == ref, (m, idx[m], ref)
        a, b = np.float32(val[m]), np.float32(row[ref])
        assert (a.view(np.uint32) == b.view(np.uint32)) or (np.isnan(a) and np.isnan(b)) or (a == 0 and b == 0), (m, a, b)


def check_against_oracle(idx, val, yr, bound):
    for m in range(yr.shape[0]):
        tol = REL_TOL * bound[m]
        assert yr[m, idx[m]] >= yr[m].max() - tol[idx[m]] - tol[np.argmax(yr[m])], m
        assert abs(float(val[m]) - yr[m, idx[m]]) <= tol[idx[m]], m


@pytest.mark.parametrize("M", [1, 8])
def test_lm_head_argmax(M):
    """The vocabulary projection 151936 x 5120 (uniform scales, g = 1)."""
    spec_codes, spec_scales = si.nvfp4_weights(151936, 5120, scale_dist="uniform", seed=0, cfg_id=5)
    x = si.activations(M, 5120, seed=0, cfg_id=5)
    idx, val, y, _ = fused_and_plain(x, spec_codes, spec_scales, 1.0)
    check_against_plain(idx, val, y)
    yr, bound = oracle_nvfp4(x, spec_codes, spec_scales, 1.0)
    check_against_oracle(idx, val, yr, bound)


@pytest.mark.parametrize("N,K,M", [(1000, 1040, 3), (130, 150016, 8), (256, 512, 1)])
def test_argmax_ragged_and_split(N, K, M):
    codes, scales = si.nvfp4_weights(N, K, seed=N, cfg_id=62)
    x = si.activations(M, K, seed=N, cfg_id=62)
    idx, val, y, ws = fused_and_plain(x, codes, scales, 0.5)
    check_against_plain(idx, val, y)
    yr, bound = oracle_nvfp4(x, codes, scales, 0.5)
    check_against_oracle(idx, val, yr, bound)
    assert int((ws != 0).sum()) == 0


def test_argmax_ties_take_the_first_row():
    """Rows 5, 130 and 250 are identical and hold the largest outputs."""
    N, K, M = 300, 512, 4
    codes, scales = si.nvfp4_weights(N, K, seed=11, cfg_id=63)
    scales[:] = 0x20                       # small block scales everywhere ...
    for r in (5, 130, 250):
        codes[r] = codes[250]
        scales[r] = 0x60                   # ... and large ones on the tied rows
    x = np.abs(si.activations(M, K, seed=11, cfg_id=63)).astype(np.float16)
    codes[250] = np.where((codes[250] & 0x8) != 0, codes[250] ^ 0x8, codes[250])  # positive codes, low nibble
    codes[250] = np.where((codes[250] & 0x80) != 0, codes[250] ^ 0x80, codes[250])  # and high nibble
    codes[5] = codes[250]
    codes[130] = codes[250]
    idx, val, y, _ = fused_and_plain(x, codes, scales, 1.0)
    check_against_plain(idx, val, y)
    assert np.all(idx == 5)


def test_argmax_nan_counts_as_largest():
    """An infinite activation turns the rows whose weight at that column is a
    zero into NaN outputs; the first such row is the argmax (as torch.argmax)."""
    N, K, M, k0 = 256, 1024, 2, 100
    codes, scales = si.nvfp4_weights(N, K, seed=12, cfg_id=64)
    x = si.activations(M, K, seed=12, cfg_id=64)
    x[0, k0] = np.float16(np.inf)
    nib = (codes[:, k0 // 2] >> (4 * (k0 % 2))) & 0xF
    wzero = ((nib & 7) == 0) | (scales[:, k0 // 16] == 0)
    assert wzero.any()
    idx, val, y, _ = fused_and_plain(x, codes, scales, 0.5)
    assert idx[0] == int(np.argmax(wzero)) and np.isnan(val[0])
    check_against_plain(idx, val, y)


def test_argmax_workspace_reused_across_calls():
    """Back-to-back fused calls of different shapes on one workspace, then a
    plain GEMM: every call finds the running maxima at zero and leaves them so."""
    ws = torch.zeros(sk.workspace_bytes(sk.FMT_NVFP4, 8, 5120, 5120), dtype=torch.uint8, device=DEV)
    for (N, K, M) in [(5120, 5120, 8), (700, 512, 2), (5120, 5120, 1)]:
        codes, scales = si.nvfp4_weights(N, K, seed=K + M, cfg_id=65)
        x = si.activations(M, K, seed=K + M, cfg_id=65)
        idx, val, y, _ = fused_and_plain(x, codes, scales, 0.5, ws=ws)
        check_against_plain(idx, val, y)
    assert int((ws != 0).sum()) == 0
