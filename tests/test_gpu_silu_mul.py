"""The NVFP4 gate+up GEMM fused with the SiLU*mul activation
(skinny_nvfp4_gemm_silu_mul), against the float64 oracle.

Tolerance.  The kernel forms g and u (the gate and up outputs) as FP32 sums,
each within the GEMM parity bound REL * B (B = sum_k |w x| of that row), then
evaluates silu(g) * u in FP32 (expf, one divide, two multiplies: a few FP32
ulps) and rounds once to the output type.  With |silu'| <= 1.1:
    |h_gpu - h| <= 1.1 REL B_g (|u| + REL B_u) + |silu(g)| REL B_u + 1e-6 |h|
                   (+ half an FP16 ulp of h for FP16 output).
A second check runs the library's plain FP32 GEMM on the same packed bytes
and workspace: its g and u are the fused kernel's, so the fused FP32 output
must equal silu(g) * u evaluated in FP32 to within a few ulps.
"""
import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import oracle
import synthetic_inputs as si
from parity import REL_TOL, oracle_nvfp4, sample_rows, ulp16

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert sk.device_error(clear=True) == 0


def reference(x, codes, scales, g, cols):
    """Oracle h[:, cols] and the tolerance, from the gate rows cols and up rows F + cols."""
    F = codes.shape[0] // 2
    rows = np.concatenate([cols, F + cols])
    y, b = oracle_nvfp4(x, codes, scales, g, rows)
    h = oracle.silu_mul(y)
    n = cols.size
    gate, up, bg, bu = y[:, :n], y[:, n:], b[:, :n], b[:, n:]
    silu = gate / (1.0 + np.exp(np.minimum(-gate, 700.0)))
    tol = 1.1 * REL_TOL * bg * (np.abs(up) + REL_TOL * bu) + np.abs(silu) * REL_TOL * bu + 1e-6 * np.abs(h)
    return h, tol


def run(x, codes, scales, g, out, split=True):
    w = sk.PackedGateUp.from_logical(codes, scales, g, DEV)
    xt = torch.from_numpy(x).to(DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, x.shape[0], 2 * w.F, w.K, DEV) if split else None
    h = sk.gemm_silu_mul(xt, w, torch.float32 if out == "f32" else torch.float16, workspace=ws)
    torch.cuda.synchronize()
    return h.double().cpu().numpy(), w, xt, ws


def check(h_gpu, h, tol, out, what):
    if out == "f16":
        tol = tol + 0.5 * ulp16(np.maximum(np.abs(h), np.abs(h_gpu)))
    err = np.abs(h_gpu - h)
    bad = ~(err <= tol)
    assert not bad.any(), "%s: %d outside; first %s gpu=%r ref=%r tol=%r" % (
        what, int(bad.sum()), tuple(np.argwhere(bad)[0]), h_gpu[tuple(np.argwhere(bad)[0])],
        h[tuple(np.argwhere(bad)[0])], tol[tuple(np.argwhere(bad)[0])])


@pytest.mark.parametrize("M,out", [(1, "f16"), (2, "f16"), (4, "f16"), (8, "f16"), (8, "f32")])
def test_gate_up_silu_mul_full_size(M, out):
    """34816 x 5120 gate+up (F = 17408), log-uniform block scales, g = 1/448."""
    codes, scales = si.nvfp4_weights(34816, 5120, scale_dist="loguniform", seed=0, cfg_id=3)
    x = si.activations(M, 5120, seed=0, cfg_id=3)
    h_gpu, *_ = run(x, codes, scales, 1.0 / 448, out)
    cols = sample_rows(17408, 700, seed=M)
    h, tol = reference(x, codes, scales, 1.0 / 448, cols)
    check(h_gpu[:, cols], h, tol, out, "gate_up M=%d" % M)


@pytest.mark.parametrize("split", [True, False])
@pytest.mark.parametrize("F,K,M", [(192, 1040, 3), (64, 150016, 8), (1024, 512, 1)])
def test_silu_mul_ragged_and_split(F, K, M, split):
    codes, scales = si.nvfp4_weights(2 * F, K, seed=F, cfg_id=66)
    x = si.activations(M, K, seed=F, cfg_id=66)
    h_gpu, *_ = run(x, codes, scales, 0.5, "f32", split)
    cols = np.arange(F)
    h, tol = reference(x, codes, scales, 0.5, cols)
    check(h_gpu, h, tol, "f32", "F=%d K=%d M=%d split=%s" % (F, K, M, split))


def test_silu_mul_pairs_each_output_with_its_own_gate_and_up_rows():
    """The plain FP32 GEMM of the same packed bytes (rows in packed order:
    64 gate rows, then their 64 up rows, per 128-row tile) gives the fused
    kernel's g and u; silu(g) * u in FP32 must match the fused output."""
    F, K, M = 256, 2048, 8
    codes, scales = si.nvfp4_weights(2 * F, K, seed=13, cfg_id=67)
    x = si.activations(M, K, seed=13, cfg_id=67)
    h_gpu, w, xt, ws = run(x, codes, scales, 0.5, "f32")
    plain = sk.PackedNVFP4(w.data, w.global_scale, 2 * F, K)
    y = sk.gemm(xt, plain, torch.float32, workspace=ws).cpu()
    torch.cuda.synchronize()
    y = y.view(M, F // 64, 2, 64)
    gate, up = y[:, :, 0, :].reshape(M, F), y[:, :, 1, :].reshape(M, F)
    want = (gate / (1.0 + torch.exp(-gate)) * up).double().numpy()
    assert np.allclose(h_gpu, want, rtol=2e-6, atol=1e-30)
    assert int((ws != 0).sum()) == 0
