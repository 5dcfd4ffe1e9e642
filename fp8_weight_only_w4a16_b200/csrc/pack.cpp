// pack.cpp -- host-side packing of NVFP4 / FP8 weights into the kernels' tiled
// layout (see layout.h), and the inverse.  Pure CPU code, no CUDA calls.
#include <string.h>

#include "../../include/skinny.h"
#include "layout.h"

using namespace skinny;

namespace {

bool valid_shape(int64_t N, int64_t K)
{
    return N > 0 && K > 0 && K % 16 == 0 && N <= (int64_t(1) << 30) && K <= (int64_t(1) << 30);
}

// A UE4M3 block scale must be finite and non-negative: sign bit clear and not
// the NaN pattern S.1111.111.
bool valid_ue4m3(uint8_t b) { return b < 0x7F; }

bool valid_e4m3(uint8_t b) { return (b & 0x7F) != 0x7F; }

inline uint32_t load_word(const uint8_t* p)
{
    uint32_t v;
    memcpy(&v, p, 4);
    return v;
}

inline void store_word(uint8_t* p, uint32_t v) { memcpy(p, &v, 4); }

}  // namespace

extern "C" size_t skinny_nvfp4_packed_bytes(int64_t N, int64_t K)
{
    if (!valid_shape(N, K)) return 0;
    return (size_t)(round_up(N, kTileRows) / kTileRows * (round_up(K, kTileK) / kTileK)) * kNvfp4TileBytes;
}

extern "C" size_t skinny_fp8_packed_bytes(int64_t N, int64_t K)
{
    if (!valid_shape(N, K)) return 0;
    return (size_t)(round_up(N, kTileRows) * round_up(K, kTileK));
}

extern "C" int skinny_pack_nvfp4(const uint8_t* codes, const uint8_t* scales, int64_t N, int64_t K,
                                 void* w_packed)
{
    if (!codes || !scales || !w_packed || !valid_shape(N, K)) return SKINNY_ERR_INVALID_ARG;
    const int64_t nblk = K / 16;
    for (int64_t i = 0; i < N * nblk; ++i)
        if (!valid_ue4m3(scales[i])) return SKINNY_ERR_INVALID_ARG;

    uint8_t* out = (uint8_t*)w_packed;
    // padding rows / columns: code 0 (+0.0) and scale 0 (the block contributes 0)
    memset(out, 0, skinny_nvfp4_packed_bytes(N, K));

    const int64_t C = round_up(K, kTileK) / kTileK;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kTileK;
            const uint8_t byte = codes[n * (K / 2) + k / 2];
            const uint32_t code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
            const Slot s = tile_slot(r, (int)(k % kTileK));
            uint8_t* dst = out + (g * C + c) * kNvfp4TileBytes + s.word;
            store_word(dst, nvfp4_put(load_word(dst), s, code));
        }
        for (int64_t b = 0; b < nblk; ++b) {
            const int64_t c = (b * 16) / kTileK;
            const int bb = (int)(b % (kTileK / 16));
            out[(g * C + c) * kNvfp4TileBytes + kNvfp4TileCodeBytes + nvfp4_scale_offset(r, bb)] = scales[n * nblk + b];
        }
    }
    return SKINNY_OK;
}

// Gate+up weights [2F][K] (rows 0..F-1 gate, F..2F-1 up) packed so that
// packed row tile g holds gate rows 64g..64g+63 in its rows 0..63 and the
// matching up rows F+64g.. in its rows 64..127: each 128-row tile then
// carries both factors of its 64 outputs of silu(gate) * up.
extern "C" int skinny_pack_nvfp4_gate_up(const uint8_t* codes, const uint8_t* scales, int64_t F, int64_t K,
                                         void* w_packed)
{
    if (!codes || !scales || !w_packed || F <= 0 || F % 64 != 0 || !valid_shape(2 * F, K))
        return SKINNY_ERR_INVALID_ARG;
    const int64_t N = 2 * F;
    const int64_t nblk = K / 16;
    for (int64_t i = 0; i < N * nblk; ++i)
        if (!valid_ue4m3(scales[i])) return SKINNY_ERR_INVALID_ARG;
    uint8_t* out = (uint8_t*)w_packed;
    memset(out, 0, skinny_nvfp4_packed_bytes(N, K));
    const int64_t C = round_up(K, kTileK) / kTileK;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t j = n < F ? n : n - F;           // output column of silu(gate) * up
        const int64_t g = j / 64;
        const int r = (int)(j % 64) + (n < F ? 0 : 64);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kTileK;
            const uint8_t byte = codes[n * (K / 2) + k / 2];
            const uint32_t code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
            const Slot s = tile_slot(r, (int)(k % kTileK));
            uint8_t* dst = out + (g * C + c) * kNvfp4TileBytes + s.word;
            store_word(dst, nvfp4_put(load_word(dst), s, code));
        }
        for (int64_t b = 0; b < nblk; ++b) {
            const int64_t c = (b * 16) / kTileK;
            const int bb = (int)(b % (kTileK / 16));
            out[(g * C + c) * kNvfp4TileBytes + kNvfp4TileCodeBytes + nvfp4_scale_offset(r, bb)] = scales[n * nblk + b];
        }
    }
    return SKINNY_OK;
}

extern "C" int skinny_unpack_nvfp4(const void* w_packed, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales)
{
    if (!codes || !scales || !w_packed || !valid_shape(N, K)) return SKINNY_ERR_INVALID_ARG;
    const uint8_t* in = (const uint8_t*)w_packed;
    const int64_t C = round_up(K, kTileK) / kTileK;
    const int64_t nblk = K / 16;
    memset(codes, 0, (size_t)(N * (K / 2)));
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kTileK;
            const Slot s = tile_slot(r, (int)(k % kTileK));
            const uint32_t code = nvfp4_get(load_word(in + (g * C + c) * kNvfp4TileBytes + s.word), s);
            codes[n * (K / 2) + k / 2] |= (k % 2 == 0) ? (uint8_t)code : (uint8_t)(code << 4);
        }
        for (int64_t b = 0; b < nblk; ++b) {
            const int64_t c = (b * 16) / kTileK;
            scales[n * nblk + b] = in[(g * C + c) * kNvfp4TileBytes + kNvfp4TileCodeBytes +
                                      nvfp4_scale_offset(r, (int)(b % (kTileK / 16)))];
        }
    }
    return SKINNY_OK;
}

extern "C" int skinny_pack_fp8(const uint8_t* q, int64_t N, int64_t K, void* w_packed)
{
    if (!q || !w_packed || !valid_shape(N, K)) return SKINNY_ERR_INVALID_ARG;
    for (int64_t i = 0; i < N * K; ++i)
        if (!valid_e4m3(q[i])) return SKINNY_ERR_INVALID_ARG;
    uint8_t* out = (uint8_t*)w_packed;
    memset(out, 0, skinny_fp8_packed_bytes(N, K));
    const int64_t C = round_up(K, kTileK) / kTileK;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kTileK;
            out[(g * C + c) * kFp8TileBytes + fp8_offset(r, (int)(k % kTileK))] = q[n * K + k];
        }
    }
    return SKINNY_OK;
}

extern "C" int skinny_unpack_fp8(const void* w_packed, int64_t N, int64_t K, uint8_t* q)
{
    if (!q || !w_packed || !valid_shape(N, K)) return SKINNY_ERR_INVALID_ARG;
    const uint8_t* in = (const uint8_t*)w_packed;
    const int64_t C = round_up(K, kTileK) / kTileK;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kTileK;
            q[n * K + k] = in[(g * C + c) * kFp8TileBytes + fp8_offset(r, (int)(k % kTileK))];
        }
    }
    return SKINNY_OK;
}
