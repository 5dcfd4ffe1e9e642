"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Every case draws seeded inputs from synthetic_inputs, packs them with the
library's host packer, runs the sm_100a kernel, and compares each checked
output with the oracle on the same bytes:
    |y_gpu - y| <= 1e-4 * sum_k |w_k x_k|        (FP32 output)
    ... + half an FP16 ulp                       (FP16 output)
Exactness cases (one-hot x) must match bit for bit.
"""
import numpy as np
import pytest
import torch

import fp8_weight_only_w4a16_b200 as sk
import synthetic_inputs as si
from parity import assert_parity, oracle_fp8, oracle_nvfp4, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_nvfp4(x, codes, scales, g, out="f16", split=True, M=None):
    w = sk.PackedNVFP4.from_logical(codes, scales, g, DEV)
    xt = torch.from_numpy(x).to(DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, x.shape[0], w.N, w.K, DEV) if split else None
    y = sk.gemm(xt, w, torch.float32 if out == "f32" else torch.float16, workspace=ws)
    torch.cuda.synchronize()
    return y.double().cpu().numpy()


def run_fp8(x, q, s, out="f16", split=True):
    w = sk.PackedFP8.from_logical(q, s, DEV)
    xt = torch.from_numpy(x).to(DEV)
    ws = sk.make_workspace(sk.FMT_FP8, x.shape[0], w.N, w.K, DEV) if split else None
    y = sk.gemm(xt, w, torch.float32 if out == "f32" else torch.float16, workspace=ws)
    torch.cuda.synchronize()
    return y.double().cpu().numpy()


@pytest.fixture(autouse=True)
def no_device_errors():
    yield
    assert sk.device_error(clear=True) == 0


# --------------------------------------------------------------------------
# The workloads at their own sizes
# --------------------------------------------------------------------------

@pytest.mark.parametrize("split", [True, False])
def test_config_small_gemv(split):
    """NVFP4 GEMV M=1, N=256, K=512, uniform codes, scales in [2^-4, 2^4], g=0.5, FP32 out."""
    codes, scales = si.nvfp4_weights(256, 512, scale_dist="uniform", seed=0, cfg_id=1)
    x = si.activations(1, 512, seed=0, cfg_id=1)
    y = run_nvfp4(x, codes, scales, 0.5, "f32", split)
    yr, b = oracle_nvfp4(x, codes, scales, 0.5)
    assert_parity(y, yr, b, "f32", "small gemv")


@pytest.mark.parametrize("M", [1, 8])
def test_attention_projection_5120(M):
    codes, scales = si.nvfp4_weights(5120, 5120, seed=0, cfg_id=2)
    x = si.activations(M, 5120, seed=0, cfg_id=2)
    y = run_nvfp4(x, codes, scales, 0.5, "f16")
    yr, b = oracle_nvfp4(x, codes, scales, 0.5)
    assert_parity(y, yr, b, "f16", "5120x5120 M=%d" % M)


@pytest.fixture(scope="module")
def gate_up():
    return si.nvfp4_weights(34816, 5120, scale_dist="loguniform", seed=0, cfg_id=3)


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_gate_up_34816(gate_up, M):
    codes, scales = gate_up
    x = si.activations(M, 5120, seed=0, cfg_id=3)
    y = run_nvfp4(x, codes, scales, 1.0 / 448.0, "f16")
    rows = sample_rows(34816, 3000, seed=M)
    yr, b = oracle_nvfp4(x, codes, scales, 1.0 / 448.0, rows)
    assert_parity(y[:, rows], yr, b, "f16", "gate_up M=%d" % M)


@pytest.fixture(scope="module")
def down_fp8():
    return si.fp8_weights(5120, 17408, seed=0, cfg_id=4)


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_down_fp8_17408(down_fp8, M):
    q, s = down_fp8
    x = si.activations(M, 17408, seed=0, cfg_id=4)
    y = run_fp8(x, q, s, "f16")
    rows = sample_rows(5120, 1500, seed=M)
    yr, b = oracle_fp8(x, q, s, rows)
    assert_parity(y[:, rows], yr, b, "f16", "down M=%d" % M)


@pytest.mark.parametrize("M", [1, 8])
def test_lm_head_151936(M):
    codes, scales = si.nvfp4_weights(151936, 5120, seed=0, cfg_id=5)
    x = si.activations(M, 5120, seed=0, cfg_id=5)
    y = run_nvfp4(x, codes, scales, 1.0, "f32")
    rows = sample_rows(151936, 3000, seed=M)
    yr, b = oracle_nvfp4(x, codes, scales, 1.0, rows)
    assert_parity(y[:, rows], yr, b, "f32", "lm_head M=%d" % M)


# --------------------------------------------------------------------------
# Edge cases: ragged shapes, every M, both schedules, both output types
# --------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 16), (17, 48), (255, 80), (257, 144), (1000, 1040), (300, 4096)])
@pytest.mark.parametrize("M", [1, 3, 5, 8])
@pytest.mark.parametrize("split", [True, False])
def test_nvfp4_ragged(N, K, M, split):
    codes, scales = si.nvfp4_weights(N, K, seed=N + K, cfg_id=50)
    x = si.activations(M, K, seed=N + K, cfg_id=50)
    for out in ("f32", "f16"):
        y = run_nvfp4(x, codes, scales, 0.75, out, split)
        yr, b = oracle_nvfp4(x, codes, scales, 0.75)
        assert_parity(y, yr, b, out, "nvfp4 N=%d K=%d M=%d %s" % (N, K, M, out))


@pytest.mark.parametrize("N,K", [(1, 16), (17, 48), (255, 80), (257, 144), (1000, 1040)])
@pytest.mark.parametrize("M", [1, 2, 6, 8])
@pytest.mark.parametrize("split", [True, False])
def test_fp8_ragged(N, K, M, split):
    q, s = si.fp8_weights(N, K, seed=N + K, cfg_id=51)
    x = si.activations(M, K, seed=N + K, cfg_id=51)
    for out in ("f32", "f16"):
        y = run_fp8(x, q, s, out, split)
        yr, b = oracle_fp8(x, q, s)
        assert_parity(y, yr, b, out, "fp8 N=%d K=%d M=%d %s" % (N, K, M, out))


def test_one_hot_is_bitwise_nvfp4():
    """x = e_k: y[., n] = W[n][k] exactly (one exact product, no rounding: with
    g = 0.5 the weight e2m1 * ue4m3 * g is exact in FP32)."""
    N, K = 700, 640
    codes, scales = si.nvfp4_weights(N, K, seed=3, cfg_id=52)
    ks = [0, 1, 2, 3, 15, 16, 63, 64, 127, 128, 129, 511, 639]
    for start in range(0, len(ks), 8):
        sel = ks[start:start + 8]
        x = np.zeros((len(sel), K), np.float16)
        for m, k in enumerate(sel):
            x[m, k] = 1.0
        y = run_nvfp4(x, codes, scales, 0.5, "f32")
        yr, _ = oracle_nvfp4(x, codes, scales, 0.5)
        assert np.array_equal(y, yr), sel


def test_one_hot_is_bitwise_fp8():
    N, K = 300, 192
    q, s = si.fp8_weights(N, K, seed=4, cfg_id=53)
    ks = [0, 1, 2, 3, 4, 17, 64, 191]
    x = np.zeros((len(ks), K), np.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    y = run_fp8(x, q, s, "f32")
    yr, _ = oracle_fp8(x, q, s)
    # y = e4m3(q) * s[n]: the exact product has up to 4 + 24 significant bits,
    # so the FP32 output is that exact value rounded once (RNE) to FP32.
    assert np.array_equal(y, yr.astype(np.float32).astype(np.float64))


def test_subnormal_activations():
    """FP16 subnormal x values are honoured (a flush to zero changes y)."""
    N, K = 64, 256
    codes, scales = si.nvfp4_weights(N, K, seed=5, cfg_id=54)
    rng = np.random.default_rng(0)
    bits = rng.integers(1, 0x400, size=(4, K)).astype(np.uint16)  # all subnormal, positive
    bits |= (rng.integers(0, 2, size=(4, K)) << 15).astype(np.uint16)
    x = bits.view(np.float16)
    y = run_nvfp4(x, codes, scales, 1.0, "f32")
    yr, b = oracle_nvfp4(x, codes, scales, 1.0)
    assert np.all(np.abs(yr) > 0)
    assert_parity(y, yr, b, "f32", "subnormal x")


def test_fp16_output_overflows_to_inf():
    N, K = 32, 64
    codes = np.full((N, K // 2), 0x77, np.uint8)   # every code 6.0
    scales = np.full((N, K // 16), 0x7E, np.uint8)  # 448
    x = np.full((1, K), 2.0, np.float16)
    y = run_nvfp4(x, codes, scales, 1.0, "f16")
    assert np.all(np.isposinf(y))


# --------------------------------------------------------------------------
# Properties of the schedule
# --------------------------------------------------------------------------

def test_bitwise_deterministic_and_slots_cleared():
    codes, scales = si.nvfp4_weights(5120, 5120, seed=1, cfg_id=2)
    w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
    xt = torch.from_numpy(si.activations(8, 5120, seed=1, cfg_id=2)).to(DEV)
    ws = sk.make_workspace(sk.FMT_NVFP4, 8, 5120, 5120, DEV)
    ys = [sk.gemm(xt, w, torch.float32, workspace=ws) for _ in range(5)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])
    # Every published partial sum was consumed and its slot zeroed again.
    assert int((ws != 0).sum()) == 0


def test_workspace_reused_across_shapes_and_formats():
    """One workspace (sized for the largest call) serves different shapes in turn."""
    big = max(sk.workspace_bytes(sk.FMT_NVFP4, 8, 34816, 5120), sk.workspace_bytes(sk.FMT_FP8, 8, 5120, 17408))
    ws = torch.zeros(big, dtype=torch.uint8, device=DEV)
    # Row-tile counts 40, 8, 272, 3, 40: each call must find every slot empty
    # (zero) and leave it so, whatever the previous shape was.
    for (N, K, fmt) in [(5120, 5120, "nvfp4"), (1000, 1040, "fp8"), (34816, 5120, "nvfp4"), (257, 144, "nvfp4"),
                        (5120, 1024, "fp8")]:
        x = si.activations(4, K, seed=K, cfg_id=55)
        if fmt == "nvfp4":
            codes, scales = si.nvfp4_weights(N, K, seed=K, cfg_id=55)
            w = sk.PackedNVFP4.from_logical(codes, scales, 0.5, DEV)
            yr, b = oracle_nvfp4(x, codes, scales, 0.5)
        else:
            q, s = si.fp8_weights(N, K, seed=K, cfg_id=55)
            w = sk.PackedFP8.from_logical(q, s, DEV)
            yr, b = oracle_fp8(x, q, s)
        y = sk.gemm(torch.from_numpy(x).to(DEV), w, torch.float32, workspace=ws)
        torch.cuda.synchronize()
        assert_parity(y.double().cpu().numpy(), yr, b, "f32", "reuse %s %dx%d" % (fmt, N, K))
    assert int((ws != 0).sum()) == 0


@pytest.mark.parametrize("fmt", ["nvfp4", "fp8"])
def test_row_tile_split_across_every_cta(fmt):
    """Two row tiles (the second ragged) whose K range is shared by all CTAs:
    each finisher gathers the partial sums of ~70 contributors in batches,
    most of them CTAs whose whole range lies inside the row tile."""
    N, K, M = 130, 150016, 8
    x = si.activations(M, K, seed=9, cfg_id=60)
    if fmt == "nvfp4":
        codes, scales = si.nvfp4_weights(N, K, seed=9, cfg_id=60)
        y = run_nvfp4(x, codes, scales, 0.5, "f32")
        yr, b = oracle_nvfp4(x, codes, scales, 0.5)
    else:
        q, s = si.fp8_weights(N, K, seed=9, cfg_id=60)
        y = run_fp8(x, q, s, "f32")
        yr, b = oracle_fp8(x, q, s)
    assert_parity(y, yr, b, "f32", "split across all CTAs")


def test_non_finite_partial_sums():
    """An infinite activation makes some partial sums +-inf or NaN; they must
    pass through the split-K combine like any other value.  Row tile 0 is
    split over ten CTAs, one K tile each."""
    N, K, M, k0 = 256, 5120, 3, 1000
    codes, scales = si.nvfp4_weights(N, K, seed=10, cfg_id=61)
    x = si.activations(M, K, seed=10, cfg_id=61)
    x[0, k0] = np.float16(np.inf)
    y = run_nvfp4(x, codes, scales, 0.5, "f32")
    # Token 0: NaN where w[n, k0] is a signed zero (inf * 0), else +-inf.
    nib = (codes[:, k0 // 2] >> (4 * (k0 % 2))) & 0xF
    wzero = ((nib & 7) == 0) | (scales[:, k0 // 16] == 0)
    wneg = (nib & 8) != 0
    assert np.all(np.isnan(y[0, wzero]))
    assert np.all(np.isposinf(y[0, ~wzero & ~wneg])) and np.all(np.isneginf(y[0, ~wzero & wneg]))
    yr, b = oracle_nvfp4(x[1:], codes, scales, 0.5)
    assert_parity(y[1:], yr, b, "f32", "finite tokens")


def test_split_and_whole_tile_schedules_agree():
    codes, scales = si.nvfp4_weights(2048, 5120, seed=2, cfg_id=56)
    x = si.activations(8, 5120, seed=2, cfg_id=56)
    a = run_nvfp4(x, codes, scales, 0.5, "f32", split=True)
    b = run_nvfp4(x, codes, scales, 0.5, "f32", split=False)
    yr, bound = oracle_nvfp4(x, codes, scales, 0.5)
    assert_parity(a, yr, bound, "f32", "split")
    assert_parity(b, yr, bound, "f32", "whole")


def test_row_independence():
    """Row i of an M=8 call agrees with the M=1 call on row i (within tolerance:
    the two calls split K differently)."""
    codes, scales = si.nvfp4_weights(1024, 2048, seed=6, cfg_id=57)
    x = si.activations(8, 2048, seed=6, cfg_id=57)
    y8 = run_nvfp4(x, codes, scales, 0.5, "f32")
    _, b = oracle_nvfp4(x, codes, scales, 0.5)
    for m in range(8):
        y1 = run_nvfp4(x[m:m + 1], codes, scales, 0.5, "f32")
        assert np.all(np.abs(y1[0] - y8[m]) <= 2e-4 * b[m])


def test_guard_bands_untouched():
    """Outputs are written inside y only: canary words around y survive."""
    N, K, M = 257, 144, 5
    codes, scales = si.nvfp4_weights(N, K, seed=7, cfg_id=58)
    w = sk.PackedNVFP4.from_logical(codes, scales, 1.0, DEV)
    x = torch.from_numpy(si.activations(M, K, seed=7, cfg_id=58)).to(DEV)
    guard = 4096
    buf = torch.full((2 * guard + M * N,), -12345.0, dtype=torch.float32, device=DEV)
    y = buf[guard:guard + M * N].view(M, N)
    ws = sk.make_workspace(sk.FMT_NVFP4, M, N, K, DEV)
    sk.gemm_into(y, x, w, workspace=ws)
    torch.cuda.synchronize()
    assert torch.all(buf[:guard] == -12345.0) and torch.all(buf[guard + M * N:] == -12345.0)
    yr, b = oracle_nvfp4(x.cpu().numpy(), codes, scales, 1.0)
    assert_parity(y.double().cpu().numpy(), yr, b, "f32", "guarded")


def test_workspace_too_small_is_rejected():
    codes, scales = si.nvfp4_weights(512, 256, seed=8, cfg_id=59)
    w = sk.PackedNVFP4.from_logical(codes, scales, 1.0, DEV)
    x = torch.from_numpy(si.activations(1, 256, seed=8, cfg_id=59)).to(DEV)
    need = sk.workspace_bytes(sk.FMT_NVFP4, 1, 512, 256)
    ws = torch.zeros(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(sk.SkinnyError) as e:
        sk.gemm(x, w, workspace=ws)
    assert e.value.status == sk.ERR_WORKSPACE


def test_mixed_layer_back_to_back():
    """One decoder layer's five GEMMs back to back on one stream, M = 1 and 8."""
    for M in (1, 8):
        outs, refs = [], []
        ws = torch.zeros(max(sk.workspace_bytes(sk.FMT_NVFP4, M, 34816, 5120),
                             sk.workspace_bytes(sk.FMT_FP8, M, 5120, 17408)), dtype=torch.uint8, device=DEV)
        for i, spec in enumerate(si.MIXED_LAYER):
            x = si.activations(M, spec.K, seed=0, cfg_id=si.MIXED_CFG_ID, tensor_id=100 + i)
            rows = sample_rows(spec.N, 600, seed=i)
            if spec.fmt == "nvfp4":
                codes, scales = si.weights_for(spec, cfg_id=si.MIXED_CFG_ID, tensor_id=10 * i)
                w = sk.PackedNVFP4.from_logical(codes, scales, spec.global_scale, DEV)
                refs.append(oracle_nvfp4(x, codes, scales, spec.global_scale, rows) + (rows, spec.out))
            else:
                q, s = si.weights_for(spec, cfg_id=si.MIXED_CFG_ID, tensor_id=10 * i)
                w = sk.PackedFP8.from_logical(q, s, DEV)
                refs.append(oracle_fp8(x, q, s, rows) + (rows, spec.out))
            outs.append(sk.gemm(torch.from_numpy(x).to(DEV), w, torch.float16, workspace=ws))
        torch.cuda.synchronize()
        for y, (yr, b, rows, out) in zip(outs, refs):
            assert_parity(y.double().cpu().numpy()[:, rows], yr, b, out, "mixed M=%d" % M)
