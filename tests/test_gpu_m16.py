"""M = 9..16: two token blocks of the m16n8k16 MMA per decoded weight fragment
(a deeper speculative draft, or two requests' verify rounds in one call).

Every case is compared with the float64 oracle element by element at the
parity tolerance.  Two exact invariants pin the second token block as well:
the MMA computes every output column on its own and the split of K depends
only on the shape, so rows 0..7 of an M=16 call equal the M=8 call on those
rows bit for bit, and rows 8..15 equal the M=8 call on rows 8..15."""
import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import synthetic_inputs as si
from parity import assert_parity, oracle_fp8, oracle_nvfp4, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert sk.device_error(clear=True) == 0


def run(x, w, out="f32", split=True):
    xt = torch.from_numpy(x).to(DEV)
    ws = sk.make_workspace(w.fmt, x.shape[0], w.N, w.K, DEV) if split else None
    y = sk.gemm(xt, w, torch.float32 if out == "f32" else torch.float16, workspace=ws)
    torch.cuda.synchronize()
    return y.double().cpu().numpy()


@pytest.mark.parametrize("M", [9, 12, 16])
def test_attention_projection_5120(M):
    codes, scales = si.nvfp4_weights(5120, 5120, seed=0, cfg_id=2)
    x = si.activations(M, 5120, seed=0, cfg_id=2)
    w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
    y = run(x, w, "f16")
    yr, b = oracle_nvfp4(x, codes, scales, 0.5)
    assert_parity(y, yr, b, "f16", "5120x5120 M=%d" % M)


@pytest.mark.parametrize("M", [9, 16])
def test_gate_up_34816(M):
    codes, scales = si.nvfp4_weights(34816, 5120, scale_dist="loguniform", seed=0, cfg_id=3)
    x = si.activations(M, 5120, seed=0, cfg_id=3)
    w = sk.PackedNVFP4.from_logical(codes, scales, 1.0 / 448.0, DEV)
    y = run(x, w, "f16")
    rows = sample_rows(34816, 2000, seed=M)
    yr, b = oracle_nvfp4(x, codes, scales, 1.0 / 448.0, rows)
    assert_parity(y[:, rows], yr, b, "f16", "gate_up M=%d" % M)


@pytest.mark.parametrize("M", [12, 16])
def test_down_fp8_17408(M):
    q, s = si.fp8_weights(5120, 17408, seed=0, cfg_id=4)
    x = si.activations(M, 17408, seed=0, cfg_id=4)
    w = sk.PackedFP8.from_logical(q, s, DEV)
    y = run(x, w, "f16")
    rows = sample_rows(5120, 1200, seed=M)
    yr, b = oracle_fp8(x, q, s, rows)
    assert_parity(y[:, rows], yr, b, "f16", "down M=%d" % M)


@pytest.mark.parametrize("N,K", [(17, 48), (257, 144), (1000, 1040), (300, 4096)])
@pytest.mark.parametrize("M", [9, 13, 16])
@pytest.mark.parametrize("split", [True, False])
def test_ragged(N, K, M, split):
    codes, scales = si.nvfp4_weights(N, K, seed=N + K, cfg_id=62)
    q, s = si.fp8_weights(N, K, seed=N + K, cfg_id=62)
    x = si.activations(M, K, seed=N + K, cfg_id=62)
    wn = sk.PackedNVFP4.from_logical(codes, scales, 0.75, DEV)
    wf = sk.PackedFP8.from_logical(q, s, DEV)
    for out in ("f32", "f16"):
        yr, b = oracle_nvfp4(x, codes, scales, 0.75)
        assert_parity(run(x, wn, out, split), yr, b, out, "nvfp4 N=%d K=%d M=%d %s" % (N, K, M, out))
        yr, b = oracle_fp8(x, q, s)
        assert_parity(run(x, wf, out, split), yr, b, out, "fp8 N=%d K=%d M=%d %s" % (N, K, M, out))


@pytest.mark.parametrize("fmt", ["nvfp4", "fp8"])
@pytest.mark.parametrize("split", [True, False])
def test_token_blocks_match_the_eight_token_kernel_bitwise(fmt, split):
    N, K = 2048, 5120
    x = si.activations(16, K, seed=11, cfg_id=63)
    if fmt == "nvfp4":
        codes, scales = si.nvfp4_weights(N, K, seed=11, cfg_id=63)
        w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
    else:
        q, s = si.fp8_weights(N, K, seed=11, cfg_id=63)
        w = sk.PackedFP8.from_logical(q, s, DEV)
    y16 = run(x, w, "f32", split)
    assert np.array_equal(y16[:8], run(x[:8], w, "f32", split))
    assert np.array_equal(y16[8:], run(x[8:], w, "f32", split))


def test_one_hot_is_bitwise():
    N, K = 700, 640
    codes, scales = si.nvfp4_weights(N, K, seed=12, cfg_id=64)
    ks = [0, 1, 2, 3, 15, 16, 63, 64, 127, 128, 129, 255, 256, 511, 512, 639]
    x = np.zeros((16, K), np.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
    yr, _ = oracle_nvfp4(x, codes, scales, 0.5)
    assert np.array_equal(run(x, w, "f32"), yr)


def test_fused_epilogues_and_grouped_at_m16():
    """The fused argmax, SiLU*mul and residual add, the grouped launch and the
    allocation-free entry point at M = 16 (oracle-checked)."""
    M, K = 16, 1040
    x = si.activations(M, K, seed=13, cfg_id=65)
    xt = torch.from_numpy(x).to(DEV)
    # argmax
    N = 3000
    codes, scales = si.nvfp4_weights(N, K, seed=13, cfg_id=65)
    w = sk.PackedNVFP4.from_logical(codes, scales, 1.0, DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV)
    idx, val = sk.gemm_argmax(xt, w, ws)
    torch.cuda.synchronize()
    idx, val = idx.cpu().numpy(), val.cpu().numpy()
    yr, b = oracle_nvfp4(x, codes, scales, 1.0)
    tol = 1e-4 * b
    for m in range(M):
        assert yr[m, idx[m]] >= yr[m].max() - tol[m, idx[m]] - tol[m, np.argmax(yr[m])]
        assert abs(float(val[m]) - yr[m, idx[m]]) <= tol[m, idx[m]]
    # residual add in place (FP32)
    y = torch.from_numpy(np.linspace(-3, 3, M * N).reshape(M, N).astype(np.float32)).to(DEV)
    r0 = y.double().cpu().numpy()
    sk.gemm_add_into(y, xt, w, y, workspace=ws)
    torch.cuda.synchronize()
    assert_parity(y.double().cpu().numpy(), yr + r0, b, "f32", "residual M=16")
    # grouped (two members, own activations)
    x2 = si.activations(M, K, seed=14, cfg_id=65)
    c2, s2 = si.nvfp4_weights(700, K, seed=14, cfg_id=65)
    w2 = sk.PackedNVFP4.from_logical(c2, s2, 0.25, DEV)
    ya = torch.empty((M, N), dtype=torch.float32, device=DEV)
    yb = torch.empty((M, 700), dtype=torch.float32, device=DEV)
    sk.gemm_grouped_into([ya, yb], [xt, torch.from_numpy(x2).to(DEV)], [w, w2], workspace=ws)
    torch.cuda.synchronize()
    assert_parity(ya.double().cpu().numpy(), yr, b, "f32", "grouped member 0")
    yr2, b2 = oracle_nvfp4(x2, c2, s2, 0.25)
    assert_parity(yb.double().cpu().numpy(), yr2, b2, "f32", "grouped member 1")
    # SiLU*mul
    F = 256
    cg, sg = si.nvfp4_weights(2 * F, K, seed=15, cfg_id=65)
    wg = sk.PackedGateUp.from_logical(cg, sg, 0.5, DEV)
    h = sk.gemm_silu_mul(xt, wg, torch.float32, workspace=ws)
    torch.cuda.synchronize()
    yg, bg = oracle_nvfp4(x, cg, sg, 0.5)
    import oracle

    hr = oracle.silu_mul(yg)
    gate, up = yg[:, :F], yg[:, F:]
    silu = gate / (1.0 + np.exp(np.minimum(-gate, 700.0)))
    rel = 1e-4   # the SiLU*mul tolerance of the fused-activation tests, from the GEMM parity bound
    tol = 1.1 * rel * bg[:, :F] * (np.abs(up) + rel * bg[:, F:]) + np.abs(silu) * rel * bg[:, F:] + 1e-6 * np.abs(hr)
    assert np.all(np.abs(h.double().cpu().numpy() - hr) <= tol)
    # allocation-free entry point: bitwise the workspace entry point's output
    import ctypes

    y_static = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    st = sk.library().skinny_nvfp4_gemm_static_ws(xt.data_ptr(), M, K, w.data.data_ptr(), ctypes.c_float(1.0), N,
                                                  y_static.data_ptr(), sk.OUT_F32,
                                                  torch.cuda.current_stream().cuda_stream)
    assert st == sk.OK
    y_ws = sk.gemm(xt, w, torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y_static, y_ws)
    assert_parity(y_static.double().cpu().numpy(), yr, b, "f32", "static scratch M=16")
