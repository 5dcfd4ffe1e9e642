// layout.h -- the packed weight layout shared by the host packer and the
// sm_100a kernels (private to libskinny; the public ABI only sees byte counts).
//
// Tiles.  W[N][K] is cut into tiles of 128 output rows x 512 columns, stored in
// the order tile(g, c) = g * C + c (g = row tile, c = K tile), so a CTA that
// walks a contiguous range of tiles streams one contiguous byte range, one
// bulk copy per tile.  An NVFP4 tile is 32768 code bytes followed by its 4096
// UE4M3 scale bytes (36864 bytes); an FP8 tile is 65536 bytes.
//
// Inside a tile: 8 strips of 16 rows; each strip has eight 64-column chunks.
// One chunk of one strip is laid out for a warp-wide sequence of four
// m16n8k16 tensor-core steps j = 0..3: lane l = 4*gid + t owns rows
// {gid, gid+8} of the strip and the 16 logical columns [16t, 16t+16) of the
// chunk.  MMA k-slot {2t, 2t+1, 2t+8, 2t+9} of step j carries logical column
// 16t + 4j + {0, 1, 2, 3}; the activations are staged in the same order, so
// the dot product is unchanged and a lane reads its B operand for all four
// steps as 32 contiguous bytes.  Register r of the A fragment (r = 0..3) holds
// row gid + 8*(r&1) at logical columns 16t + 4j + 2*(r>>1) + {0, 1} (element
// e = 0 in the low half of the f16x2 register, e = 1 in the high half).
//
// NVFP4 words.  A lane's 16 bytes are four 32-bit words, word j feeding MMA
// step j: byte r holds A register r, element e in nibble e (low nibble first)
// -- the input of Blackwell's exact cvt.rn.f16x2.e2m1x2.
#pragma once
#include <stdint.h>

namespace skinny {

constexpr int kTileRows = 128;       // output rows per tile
constexpr int kStripRows = 16;       // rows per MMA strip (the m16 of m16n8k16)
constexpr int kStrips = kTileRows / kStripRows;
constexpr int kChunkK = 64;          // K per strip chunk (four k16 steps)
constexpr int kTileK = 512;          // K per tile: eight chunks
constexpr int kChunks = kTileK / kChunkK;

constexpr int kNvfp4TileCodeBytes = kTileRows * kTileK / 2;       // 32768
constexpr int kNvfp4TileScaleBytes = kTileRows * kTileK / 16;     // 4096
constexpr int kNvfp4TileBytes = kNvfp4TileCodeBytes + kNvfp4TileScaleBytes;
constexpr int kFp8TileBytes = kTileRows * kTileK;                 // 65536
constexpr int kNvfp4StripCodeBytes = kChunks * 512;   // one strip: 8 chunks x 32 lanes x 16 bytes
constexpr int kNvfp4StripScaleBytes = kChunks * 64;   // one strip: 8 chunks x 64 scale bytes
constexpr int kFp8StripBytes = kChunks * 1024;        // one strip: 8 chunks x 2 halves x 32 lanes x 16 bytes

inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// Where element (row r in 0..127, column k in 0..511) of a tile lives.
struct Slot {
    int word;   // byte offset of its 32-bit word inside the tile's codes
    int j;      // MMA step (word index inside the lane's 16 / 32 bytes)
    int reg;    // A-fragment register
    int e;      // half of the f16x2 register (0 = low)
};

inline Slot tile_slot(int r, int k)
{
    const int strip = r / 16, rr = r % 16;
    const int gid = rr % 8, h = rr / 8;
    const int ch = k / 64, kk = k % 64;
    const int t = kk / 16, w = kk % 16;
    const int j = w / 4, o = w % 4;
    Slot s;
    s.j = j;
    s.reg = h + 2 * (o / 2);
    s.e = o % 2;
    s.word = strip * kNvfp4StripCodeBytes + ch * 512 + (4 * gid + t) * 16 + 4 * j;  // NVFP4 placement
    return s;
}

// NVFP4: set / read the nibble of slot s in its word.
inline uint32_t nvfp4_put(uint32_t word, const Slot& s, uint32_t code)
{
    return word | (code << (8 * s.reg + 4 * s.e));
}

inline uint32_t nvfp4_get(uint32_t word, const Slot& s) { return (word >> (8 * s.reg + 4 * s.e)) & 0xFu; }

// Byte offset, inside the 4096 scale bytes of an NVFP4 tile, of the UE4M3 scale of
// row r (0..127) and 16-column block b (0..31).  A lane reads its two scales (rows
// gid and gid+8 of its strip, block t of the chunk) as one 16-bit word: row
// gid in the low byte (cvt.rn.f16x2.e4m3x2 turns the low byte into the low
// half).
inline int nvfp4_scale_offset(int r, int b)
{
    const int strip = r / 16, rr = r % 16;
    const int gid = rr % 8, h = rr / 8;
    const int ch = b / 4, t = b % 4;
    return strip * kNvfp4StripScaleBytes + ch * 64 + t * 16 + gid * 2 + h;
}

// Byte offset, inside a 65536-byte FP8 tile, of element (row r, column k).
// A lane's 32 bytes per chunk are two 16-byte halves 512 bytes apart (steps
// j = 0, 1 in the first, j = 2, 3 in the second), so that each 16-byte
// shared-memory load of a warp reads 512 contiguous bytes (no bank
// conflicts).  Inside a half: step j in bytes 8(j%2)..8(j%2)+7, register r in
// bytes 2r, 2r+1, element e in byte e (cvt.rn.f16x2.e4m3x2 turns the low byte
// into the low half).
inline int fp8_offset(int r, int k)
{
    const Slot s = tile_slot(r, k);
    const int strip = r / 16, rr = r % 16;
    const int gid = rr % 8;
    const int ch = k / 64, t = (k % 64) / 16;
    return strip * kFp8StripBytes + ch * 1024 + (s.j / 2) * 512 + (4 * gid + t) * 16 + 8 * (s.j % 2) + 2 * s.reg +
           s.e;
}

}  // namespace skinny
