"""Host-side packing (pure CPU): round trips, padding, validation, tile order."""
import numpy as np
import pytest

import fp8_weight_only_w4a16_b200 as sk


@pytest.mark.parametrize("N,K", [(1, 16), (17, 80), (256, 128), (300, 512), (513, 144)])
def test_nvfp4_roundtrip(N, K):
    rng = np.random.default_rng(N * 1000 + K)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(N, K // 16), dtype=np.uint8)
    pc = sk.pack_nvfp4(codes, scales)
    Np, Kp = -(-N // 128) * 128, -(-K // 512) * 512
    assert pc.size == Np * Kp // 2 + Np * Kp // 16
    c2, s2 = sk.unpack_nvfp4(pc, N, K)
    assert np.array_equal(c2, codes) and np.array_equal(s2, scales)
    # each tile is 32768 code bytes then 4096 scale bytes; the scale bytes hold exactly the scales
    tiles = pc.reshape(-1, 36864)
    assert np.count_nonzero(tiles[:, 32768:]) == np.count_nonzero(scales)


@pytest.mark.parametrize("N,K", [(1, 16), (17, 80), (256, 64), (300, 208)])
def test_fp8_roundtrip(N, K):
    rng = np.random.default_rng(N * 7 + K)
    q = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x11
    pc = sk.pack_fp8(q)
    assert pc.size == (-(-N // 128) * 128) * (-(-K // 512) * 512)
    assert np.array_equal(sk.unpack_fp8(pc, N, K), q)
    assert np.count_nonzero(pc) == np.count_nonzero(q)


def test_nvfp4_element_lands_in_its_tile():
    """A single nonzero code at (n, k) lands in tile (n // 128) * C + k // 512, in
    the strip of row n, the 64-column chunk of k, and the 16-byte word of lane
    4*((n%16)%8) + (k%64)//16 (all its bits inside one 32-bit word)."""
    N, K = 300, 1536
    C = K // 512
    rng = np.random.default_rng(0)
    for _ in range(200):
        n, k = int(rng.integers(N)), int(rng.integers(K))
        codes = np.zeros((N, K // 2), np.uint8)
        codes[n, k // 2] = 0xD if k % 2 == 0 else 0xD0
        pc = sk.pack_nvfp4(codes, np.zeros((N, K // 16), np.uint8))
        idx = np.nonzero(pc)[0]
        assert idx.size >= 1 and idx[-1] // 4 == idx[0] // 4
        tile, off = divmod(int(idx[0]), 36864)
        assert tile == (n // 128) * C + k // 512
        strip, rem = divmod(off, 4096)
        assert strip == (n % 128) // 16
        chunk, rem = divmod(rem, 512)
        assert chunk == (k % 512) // 64
        assert rem // 16 == 4 * ((n % 16) % 8) + (k % 64) // 16


def _emulate_lane_decode(words):
    """The kernel's decode of one lane's four 32-bit words into the 16 f16x2 A
    registers (as 32 float64 values, register-major, low half first), block
    scale left out: byte r of word j is register r of MMA step j, low nibble
    first, each nibble an E2M1 code (decoded here with ml_dtypes)."""
    import ml_dtypes

    out = []
    for w in words:
        w = int(w)
        for r in range(4):
            byte = (w >> (8 * r)) & 0xFF
            for e in range(2):
                nib = np.array([(byte >> (4 * e)) & 0xF], np.uint8)
                out.append(float(nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)[0]))
    return out


def test_nvfp4_lane_words_decode_to_their_slots():
    """Emulate the kernel's decode of every lane of one tile and check each A
    register element against the E2M1 value of the logical element it must
    carry: row gid + 8*(r&1), column 16t + 4j + 2*(r>>1) + e; and each lane's
    16-bit scale word: row gid in the low byte, row gid+8 in the high byte."""
    import ml_dtypes

    N, K = 128, 512
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    pc = sk.pack_nvfp4(codes, np.zeros((N, K // 16), np.uint8))
    assert pc.size == 36864
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(N, K)
    val = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    words = pc.view(np.uint32)
    for strip in range(8):
        for chunk in range(8):
            for lane in range(32):
                gid, t = lane // 4, lane % 4
                base = (strip * 4096 + chunk * 512 + lane * 16) // 4
                dec = _emulate_lane_decode(words[base:base + 4])
                i = 0
                for j in range(4):
                    for r in range(4):
                        for e in range(2):
                            row = strip * 16 + gid + 8 * (r & 1)
                            col = chunk * 64 + 16 * t + 4 * j + 2 * (r >> 1) + e
                            want = val[row, col]
                            assert dec[i] == want and np.signbit(dec[i]) == np.signbit(want), (strip, lane, j, r, e)
                            i += 1


def test_nvfp4_lane_scale_words():
    N, K = 128, 512
    rng = np.random.default_rng(7)
    scales = rng.integers(0, 0x7F, size=(N, K // 16), dtype=np.uint8)
    pc = sk.pack_nvfp4(np.zeros((N, K // 2), np.uint8), scales)
    sc = pc[32768:]
    for strip in range(8):
        for chunk in range(8):
            for lane in range(32):
                gid, t = lane // 4, lane % 4
                off = strip * 512 + chunk * 64 + t * 16 + gid * 2
                assert sc[off] == scales[strip * 16 + gid, chunk * 4 + t]
                assert sc[off + 1] == scales[strip * 16 + gid + 8, chunk * 4 + t]


def test_fp8_lane_bytes_hold_their_slots():
    N, K = 128, 512
    rng = np.random.default_rng(6)
    q = rng.integers(0, 0x7F, size=(N, K), dtype=np.uint8)
    pc = sk.pack_fp8(q)
    for strip in range(8):
        for chunk in range(8):
            for lane in range(32):
                gid, t = lane // 4, lane % 4
                for j in range(4):
                    # two 16-byte halves per lane, 512 bytes apart (conflict-free loads)
                    base = strip * 8192 + chunk * 1024 + (j // 2) * 512 + lane * 16 + 8 * (j % 2)
                    for r in range(4):
                        for e in range(2):
                            row = strip * 16 + gid + 8 * (r & 1)
                            col = chunk * 64 + 16 * t + 4 * j + 2 * (r >> 1) + e
                            assert pc[base + 2 * r + e] == q[row, col]


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
    assert sk.nvfp4_packed_bytes(0, 16) == 0
    assert sk.nvfp4_packed_bytes(4, 24) == 0
    assert sk.fp8_packed_bytes(4, 8) == 0
    assert sk.nvfp4_packed_bytes(5120, 5120) == 5120 * 5120 // 2 + 5120 * 5120 // 16


@pytest.mark.parametrize("F,K", [(64, 512), (192, 1040)])
def test_gate_up_packing_interleaves_blocks_of_64_rows(F, K):
    """skinny_pack_nvfp4_gate_up equals the ordinary packing of the rows
    reordered as [gate 0..63, up 0..63, gate 64..127, up 64..127, ...]."""
    rng = np.random.default_rng(F + K)
    codes = rng.integers(0, 256, size=(2 * F, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(2 * F, K // 16), dtype=np.uint8)
    order = np.concatenate([np.r_[np.arange(64 * b, 64 * b + 64), F + np.arange(64 * b, 64 * b + 64)]
                            for b in range(F // 64)])
    want = sk.pack_nvfp4(codes[order], scales[order])
    got = sk.pack_nvfp4_gate_up(codes, scales)
    assert np.array_equal(got, want)


def test_gate_up_packing_rejects_bad_shapes():
    lib = sk.library()
    buf = np.zeros(1 << 16, np.uint8)
    c = np.zeros((128, 256), np.uint8)
    s = np.zeros((128, 32), np.uint8)
    assert lib.skinny_pack_nvfp4_gate_up(c.ctypes.data, s.ctypes.data, 96, 512, buf.ctypes.data) == sk.ERR_INVALID_ARG
    assert lib.skinny_pack_nvfp4_gate_up(c.ctypes.data, s.ctypes.data, 64, 40, buf.ctypes.data) == sk.ERR_INVALID_ARG
    assert lib.skinny_pack_nvfp4_gate_up(None, s.ctypes.data, 64, 512, buf.ctypes.data) == sk.ERR_INVALID_ARG
