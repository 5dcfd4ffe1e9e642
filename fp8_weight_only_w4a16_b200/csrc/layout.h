// layout.h -- the packed weight layout shared by the host packer and the
// sm_100a kernels (private to libskinny; the public ABI only sees byte counts).
//
// A weight matrix W[N][K] is cut into tiles of 256 output rows x TILE_K
// columns (TILE_K = 128 for NVFP4, 64 for FP8).  Tiles are stored in the
// order  tile(g, c) = g * C + c  (g = row tile, c = K tile), so one CTA that
// walks a contiguous range of tiles streams one contiguous byte range.  Every
// tile is exactly 16384 code bytes (plus 2048 scale bytes for NVFP4, in a
// separate buffer with the same tile order), i.e. one bulk copy each.
//
// Inside a tile, 16 "strips" of 16 rows follow each other; a strip's 64-K
// chunk is laid out for one warp-wide m16n8k16 tensor-core sequence: lane
// l = 4*gid + t owns rows {gid, gid+8} of the strip and the 16 logical K
// values [16t, 16t+16) of the chunk, spread over four k16 MMA steps j = 0..3.
// MMA k-slot {2t, 2t+1, 2t+8, 2t+9} of step j carries logical k
// 16t + 4j + {0, 1, 2, 3}; the activations are staged in the same order, so
// the dot product is unchanged and each lane reads its B operand for all four
// steps as 32 contiguous bytes.  Register r of the A fragment (r = 0..3)
// holds row gid + 8*(r&1) at logical k 16t + 4j + 2*(r>>1) + {0, 1}.
#pragma once
#include <stdint.h>

namespace skinny {

constexpr int kTileRows = 256;       // output rows per tile
constexpr int kStripRows = 16;       // rows per MMA strip (the m16 of m16n8k16)
constexpr int kStrips = kTileRows / kStripRows;
constexpr int kChunkK = 64;          // K per strip chunk (four k16 steps)
constexpr int kTileCodeBytes = 16384;

constexpr int kNvfp4TileK = 128;     // two chunks per NVFP4 tile
constexpr int kNvfp4TileScaleBytes = kTileRows * kNvfp4TileK / 16;  // 2048
constexpr int kFp8TileK = 64;        // one chunk per FP8 tile

static_assert(kTileRows * kNvfp4TileK / 2 == kTileCodeBytes, "nvfp4 tile size");
static_assert(kTileRows * kFp8TileK == kTileCodeBytes, "fp8 tile size");

// cvt.rn.f16x2.e2m1x2 turns the low nibble of its byte into the low half of
// the f16x2 result, and cvt.rn.f16x2.e4m3x2 turns the low byte of its 16-bit
// input into the low half.
constexpr bool kLowFirst = true;

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Byte offset, inside a 16384-byte NVFP4 code tile, of the byte that holds the
// element (row r in 0..255, column k in 0..127); *high = 1 if it is the high
// nibble.
inline int nvfp4_code_offset(int r, int k, int* high)
{
    const int strip = r / 16, rr = r % 16;
    const int gid = rr % 8, h = rr / 8;
    const int ch = k / 64, kk = k % 64;
    const int t = kk / 16, w = kk % 16;
    const int j = w / 4, o = w % 4;
    const int reg = h + 2 * (o / 2);
    const int lane = 4 * gid + t;
    *high = kLowFirst ? (o % 2) : 1 - (o % 2);
    return strip * 1024 + ch * 512 + lane * 16 + 4 * j + reg;
}

// Byte offset, inside a 2048-byte NVFP4 scale tile, of the UE4M3 scale of row
// r (0..255) and 16-column block b (0..7).  A lane reads its two scales (rows
// gid and gid+8 of its strip, block t of the chunk) as one 16-bit word.
inline int nvfp4_scale_offset(int r, int b)
{
    const int strip = r / 16, rr = r % 16;
    const int gid = rr % 8, h = rr / 8;
    const int ch = b / 4, t = b % 4;
    return strip * 128 + ch * 64 + t * 16 + gid * 2 + (kLowFirst ? h : 1 - h);
}

// Byte offset, inside a 16384-byte FP8 tile, of element (row r, column k in 0..63).
inline int fp8_code_offset(int r, int k)
{
    const int strip = r / 16, rr = r % 16;
    const int gid = rr % 8, h = rr / 8;
    const int t = k / 16, w = k % 16;
    const int j = w / 4, o = w % 4;
    const int reg = h + 2 * (o / 2);
    const int e = kLowFirst ? (o % 2) : 1 - (o % 2);
    const int lane = 4 * gid + t;
    return strip * 1024 + lane * 32 + 8 * j + 2 * reg + e;
}

}  // namespace skinny
