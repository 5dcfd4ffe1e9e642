"""Host-side packing (pure CPU): round trips, padding, validation, tile order."""
import numpy as np
import pytest

import fp8_weight_only_w4a16_b200 as sk


@pytest.mark.parametrize("N,K", [(1, 16), (17, 80), (256, 128), (300, 512), (513, 144)])
def test_nvfp4_roundtrip(N, K):
    rng = np.random.default_rng(N * 1000 + K)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(N, K // 16), dtype=np.uint8)
    pc, ps = sk.pack_nvfp4(codes, scales)
    Np, Kp = -(-N // 256) * 256, -(-K // 128) * 128
    assert pc.size == Np * Kp // 2 and ps.size == Np * Kp // 16
    c2, s2 = sk.unpack_nvfp4(pc, ps, N, K)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    # padding holds only zero codes / zero scales: the payload is all there is
    assert np.count_nonzero(pc) <= np.count_nonzero(codes & 0xF) + np.count_nonzero(codes >> 4)
    assert np.count_nonzero(ps) == np.count_nonzero(scales)


@pytest.mark.parametrize("N,K", [(1, 16), (17, 80), (256, 64), (300, 208)])
def test_fp8_roundtrip(N, K):
    rng = np.random.default_rng(N * 7 + K)
    q = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x11
    pc = sk.pack_fp8(q)
    assert pc.size == (-(-N // 256) * 256) * (-(-K // 64) * 64)
    assert np.array_equal(sk.unpack_fp8(pc, N, K), q)
    assert np.count_nonzero(pc) == np.count_nonzero(q)


def test_nvfp4_element_lands_in_its_tile():
    """A single nonzero code at (n, k) lands in tile (n // 256) * C + k // 128, in
    the strip of row n, and in the 16-byte word of lane 4*((n%16)%8) + (k%64)//16."""
    N, K = 600, 384
    C = K // 128
    rng = np.random.default_rng(0)
    for _ in range(200):
        n, k = int(rng.integers(N)), int(rng.integers(K))
        codes = np.zeros((N, K // 2), np.uint8)
        codes[n, k // 2] = 0x5 if k % 2 == 0 else 0x50
        pc, _ = sk.pack_nvfp4(codes, np.zeros((N, K // 16), np.uint8))
        (idx,) = np.nonzero(pc)
        assert idx.size == 1
        tile, off = divmod(int(idx[0]), 16384)
        assert tile == (n // 256) * C + k // 128
        strip, rem = divmod(off, 1024)
        assert strip == (n % 256) // 16
        chunk, rem = divmod(rem, 512)
        assert chunk == (k % 128) // 64
        lane = rem // 16
        assert lane == 4 * ((n % 16) % 8) + (k % 64) // 16


def test_pack_rejects_bad_scale_bytes():
    codes = np.zeros((4, 8), np.uint8)
    for bad in (0x7F, 0x80, 0xFF, 0xB8):
        scales = np.full((4, 1), 0x38, np.uint8)
        scales[2, 0] = bad
        with pytest.raises(sk.SkinnyError) as e:
            sk.pack_nvfp4(codes, scales)
        assert e.value.status == sk.ERR_INVALID_ARG


def test_pack_rejects_fp8_nan():
    q = np.zeros((2, 16), np.uint8)
    q[1, 3] = 0xFF
    with pytest.raises(sk.SkinnyError):
        sk.pack_fp8(q)


def test_packed_bytes_reject_bad_shapes():
    assert sk.nvfp4_packed_bytes(0, 16) == (0, 0)
    assert sk.nvfp4_packed_bytes(4, 24) == (0, 0)
    assert sk.fp8_packed_bytes(4, 8) == 0
    assert sk.nvfp4_packed_bytes(5120, 5120) == (5120 * 5120 // 2, 5120 * 5120 // 16)
