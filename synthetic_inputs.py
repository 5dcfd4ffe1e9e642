"""Seeded synthetic inputs for the weight-only skinny GEMM.

This module is the one piece that both sides of every parity check use: the
float64 oracle and the CUDA library get the same bytes from here.  It holds
none of the GEMM's arithmetic: it draws integer codes and scale bytes, draws
Gaussian activations and rounds them to binary16 with numpy, and (for the FP8
weights) quantises Gaussian weights with torch's own float8_e4m3fn cast.

Workloads are the decoder shapes of a 27B-class model (5120 hidden, 34816
fused gate+up, 17408 down, 151936 vocabulary), at M = 1..8 rows: one decode
token, or a k=7 speculative-verify round plus its base token.

Every draw is seeded with ``SeedSequence([seed, cfg_id, tensor_id])``.
"""
from __future__ import annotations

import dataclasses

import numpy as np

# UE4M3 bytes 0x18..0x58 are exactly the 65 E4M3 values 2^-4 .. 2^4 (positive
# E4M3 bytes are monotone in value).
_UNIFORM_SCALE_LO = 0x18
_UNIFORM_SCALE_HI = 0x58


def rng_for(seed: int, cfg_id: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(cfg_id), int(tensor_id)]))


def activations(M: int, K: int, *, seed: int = 0, cfg_id: int = 0, tensor_id: int = 100) -> np.ndarray:
    """x[M, K] ~ N(0, 1) drawn in float64, rounded to float16 (RNE)."""
    r = rng_for(seed, cfg_id, tensor_id)
    return r.standard_normal((M, K)).astype(np.float16)


def nvfp4_weights(N: int, K: int, *, scale_dist: str = "uniform", seed: int = 0, cfg_id: int = 0,
                  tensor_id: int = 0):
    """Logical NVFP4 tensor: codes[N, K/2] (low nibble = even k), scales[N, K/16] (UE4M3 bytes).

    Codes are uniform over all 16 E2M1 codes: a uniform byte has two independent
    uniform nibbles.  ``scale_dist``:
      "uniform"     -- uniform over the 65 E4M3 values in [2^-4, 2^4];
      "loguniform"  -- u ~ U(-6, 6), then 2^u rounded to E4M3 (RNE) by torch.
    """
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    r = rng_for(seed, cfg_id, tensor_id)
    codes = r.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    r2 = rng_for(seed, cfg_id, tensor_id + 1)
    if scale_dist == "uniform":
        scales = r2.integers(_UNIFORM_SCALE_LO, _UNIFORM_SCALE_HI + 1, size=(N, K // 16), dtype=np.uint8)
    elif scale_dist == "loguniform":
        import torch

        u = r2.uniform(-6.0, 6.0, size=(N, K // 16))
        scales = torch.from_numpy(np.exp2(u)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    else:
        raise ValueError(scale_dist)
    return codes, np.ascontiguousarray(scales)


def fp8_weights(N: int, K: int, *, sigma: float = 0.02, seed: int = 0, cfg_id: int = 0, tensor_id: int = 0):
    """FP8 E4M3 tensor with one FP32 scale per output channel.

    W_f ~ N(0, sigma) (float32), s[n] = max_k |W_f[n, k]| / 448 in float32,
    q = E4M3(W_f / s) rounded by torch's cast after clamping to +-448.
    Returns q[N, K] uint8 and s[N] float32.
    """
    import torch

    r = rng_for(seed, cfg_id, tensor_id)
    q = np.empty((N, K), np.uint8)
    s = np.empty((N,), np.float32)
    step = max(1, (1 << 24) // max(K, 1))
    for n0 in range(0, N, step):
        n1 = min(N, n0 + step)
        w = r.standard_normal((n1 - n0, K), dtype=np.float32) * np.float32(sigma)
        sc = (np.abs(w).max(axis=1) / np.float32(448.0)).astype(np.float32)
        sc[sc == 0] = np.float32(1.0)
        t = np.clip(w / sc[:, None], -448.0, 448.0).astype(np.float32)
        q[n0:n1] = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        s[n0:n1] = sc
    return q, s


@dataclasses.dataclass(frozen=True)
class GemmSpec:
    """One weight-only GEMM of a workload."""
    name: str
    fmt: str            # "nvfp4" or "fp8"
    N: int
    K: int
    scale_dist: str = "uniform"   # NVFP4 block-scale distribution
    global_scale: float = 1.0     # NVFP4 per-tensor scale
    out: str = "f16"              # "f16" or "f32"


# The workloads (shapes and value distributions of the decoder layers served
# at M = 1..8).  cfg ids are stable: they seed the draws.
CONFIGS = {
    1: dict(desc="NVFP4 GEMV N=256 K=512 (small correctness case)", Ms=(1,),
            gemms=(GemmSpec("tiny", "nvfp4", 256, 512, "uniform", 0.5, "f32"),)),
    2: dict(desc="NVFP4 attention projection N=5120 K=5120", Ms=(1, 8),
            gemms=(GemmSpec("attn_proj", "nvfp4", 5120, 5120, "uniform", 0.5, "f16"),)),
    3: dict(desc="NVFP4 fused gate+up N=34816 K=5120", Ms=(1, 2, 4, 8),
            gemms=(GemmSpec("gate_up", "nvfp4", 34816, 5120, "loguniform", 1.0 / 448.0, "f16"),)),
    4: dict(desc="FP8 down projection N=5120 K=17408", Ms=(1, 2, 4),
            gemms=(GemmSpec("down", "fp8", 5120, 17408, out="f16"),)),
    5: dict(desc="NVFP4 lm_head N=151936 K=5120", Ms=(1, 8),
            gemms=(GemmSpec("lm_head", "nvfp4", 151936, 5120, "uniform", 1.0, "f32"),)),
}

# One decoder layer's weight-only GEMMs back to back: three 5120x5120 NVFP4
# attention projections, the 34816x5120 NVFP4 gate+up and the 5120x17408 FP8
# down projection.  Results are not chained (no norm/activation in between).
MIXED_LAYER = (
    GemmSpec("q_proj", "nvfp4", 5120, 5120, "uniform", 0.5, "f16"),
    GemmSpec("kv_proj", "nvfp4", 5120, 5120, "uniform", 0.5, "f16"),
    GemmSpec("o_proj", "nvfp4", 5120, 5120, "uniform", 0.5, "f16"),
    GemmSpec("gate_up", "nvfp4", 34816, 5120, "loguniform", 1.0 / 448.0, "f16"),
    GemmSpec("down", "fp8", 5120, 17408, out="f16"),
)
MIXED_CFG_ID = 6


def weights_for(spec: GemmSpec, *, seed: int = 0, cfg_id: int = 0, tensor_id: int = 0):
    """Logical weights for a GemmSpec: (codes, scales) for NVFP4, (q, s) for FP8."""
    if spec.fmt == "nvfp4":
        return nvfp4_weights(spec.N, spec.K, scale_dist=spec.scale_dist, seed=seed, cfg_id=cfg_id,
                             tensor_id=tensor_id)
    return fp8_weights(spec.N, spec.K, seed=seed, cfg_id=cfg_id, tensor_id=tensor_id)
