"""The seeded input generator: determinism and the stated value distributions."""
import numpy as np
import torch

import synthetic_inputs as si


def test_seeded_draws_are_reproducible():
    a = si.nvfp4_weights(64, 128, seed=3, cfg_id=2)
    b = si.nvfp4_weights(64, 128, seed=3, cfg_id=2)
    c = si.nvfp4_weights(64, 128, seed=4, cfg_id=2)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert not np.array_equal(a[0], c[0])
    assert np.array_equal(si.activations(2, 64, seed=1), si.activations(2, 64, seed=1))


def test_uniform_scales_cover_the_65_values_in_range():
    _, s = si.nvfp4_weights(512, 1024, scale_dist="uniform")
    vals = torch.from_numpy(s).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert vals.min() == 2.0 ** -4 and vals.max() == 2.0 ** 4
    assert len(np.unique(s)) == 65


def test_loguniform_scales_are_e4m3_in_range():
    _, s = si.nvfp4_weights(256, 1024, scale_dist="loguniform")
    vals = torch.from_numpy(s).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert vals.min() >= 2.0 ** -6 and vals.max() <= 2.0 ** 6
    med = np.median(np.log2(vals))
    assert abs(med) < 0.25


def test_codes_are_uniform_nibbles():
    c, _ = si.nvfp4_weights(256, 1024)
    lo, hi = c & 0xF, c >> 4
    for nib in (lo, hi):
        counts = np.bincount(nib.ravel(), minlength=16)
        assert counts.min() > 0.9 * counts.mean()


def test_fp8_weights_scale_is_row_absmax_over_448():
    q, s = si.fp8_weights(32, 512)
    w = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.all(np.abs(w).max(axis=1) == 448.0)
    assert np.all(np.isfinite(w))
    assert np.all((s > 0.02 * 2 / 448) & (s < 0.02 * 8 / 448))


def test_activations_are_standard_normal_fp16():
    x = si.activations(8, 5120)
    assert x.dtype == np.float16
    assert abs(float(x.astype(np.float64).std()) - 1.0) < 0.02
