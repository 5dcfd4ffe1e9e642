// pack.cpp -- host-side packing of NVFP4 / FP8 weights into the kernels' tiled
// layout (see layout.h), and the inverse.  Pure CPU code, no CUDA calls.
#include <string.h>

#include <vector>

#include "../../include/skinny.h"
#include "layout.h"

using namespace skinny;

namespace {

bool valid_shape(int64_t N, int64_t K)
{
    return N > 0 && K > 0 && K % 16 == 0 && N <= (int64_t(1) << 31) && K <= (int64_t(1) << 30);
}

// A UE4M3 block scale must be finite and non-negative: sign bit clear and not
// the NaN pattern S.1111.111.
bool valid_ue4m3(uint8_t b) { return b < 0x7F; }

bool valid_e4m3(uint8_t b) { return (b & 0x7F) != 0x7F; }

}  // namespace

extern "C" size_t skinny_nvfp4_packed_bytes(int64_t N, int64_t K, size_t* scale_bytes)
{
    if (!valid_shape(N, K)) {
        if (scale_bytes) *scale_bytes = 0;
        return 0;
    }
    const int64_t Np = round_up(N, kTileRows), Kp = round_up(K, kNvfp4TileK);
    if (scale_bytes) *scale_bytes = (size_t)(Np * Kp / 16);
    return (size_t)(Np * Kp / 2);
}

extern "C" size_t skinny_fp8_packed_bytes(int64_t N, int64_t K)
{
    if (!valid_shape(N, K)) return 0;
    return (size_t)(round_up(N, kTileRows) * round_up(K, kFp8TileK));
}

extern "C" int skinny_pack_nvfp4(const uint8_t* codes, const uint8_t* scales, int64_t N, int64_t K,
                                 void* w_packed, void* w_scales)
{
    if (!codes || !scales || !w_packed || !w_scales || !valid_shape(N, K)) return SKINNY_ERR_INVALID_ARG;
    const int64_t nblk = K / 16;
    for (int64_t i = 0; i < N * nblk; ++i)
        if (!valid_ue4m3(scales[i])) return SKINNY_ERR_INVALID_ARG;

    size_t sbytes = 0;
    const size_t cbytes = skinny_nvfp4_packed_bytes(N, K, &sbytes);
    uint8_t* out = (uint8_t*)w_packed;
    uint8_t* sout = (uint8_t*)w_scales;
    memset(out, 0, cbytes);  // padding rows / columns: code 0 (+0.0)
    memset(sout, 0, sbytes); // padding scales: 0 (the block contributes 0)

    const int64_t C = round_up(K, kNvfp4TileK) / kNvfp4TileK;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kNvfp4TileK;
            const int kk = (int)(k % kNvfp4TileK);
            const uint8_t byte = codes[n * (K / 2) + k / 2];
            const uint8_t code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
            int high = 0;
            const int off = nvfp4_code_offset(r, kk, &high);
            uint8_t* dst = out + (g * C + c) * kTileCodeBytes + off;
            *dst |= high ? (uint8_t)(code << 4) : code;
        }
        for (int64_t b = 0; b < nblk; ++b) {
            const int64_t c = (b * 16) / kNvfp4TileK;
            const int bb = (int)(b % (kNvfp4TileK / 16));
            sout[(g * C + c) * kNvfp4TileScaleBytes + nvfp4_scale_offset(r, bb)] = scales[n * nblk + b];
        }
    }
    return SKINNY_OK;
}

extern "C" int skinny_unpack_nvfp4(const void* w_packed, const void* w_scales, int64_t N, int64_t K,
                                   uint8_t* codes, uint8_t* scales)
{
    if (!codes || !scales || !w_packed || !w_scales || !valid_shape(N, K)) return SKINNY_ERR_INVALID_ARG;
    const uint8_t* in = (const uint8_t*)w_packed;
    const uint8_t* sin = (const uint8_t*)w_scales;
    const int64_t C = round_up(K, kNvfp4TileK) / kNvfp4TileK;
    const int64_t nblk = K / 16;
    memset(codes, 0, (size_t)(N * (K / 2)));
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kNvfp4TileK;
            int high = 0;
            const int off = nvfp4_code_offset(r, (int)(k % kNvfp4TileK), &high);
            const uint8_t byte = in[(g * C + c) * kTileCodeBytes + off];
            const uint8_t code = high ? (byte >> 4) : (byte & 0x0F);
            codes[n * (K / 2) + k / 2] |= (k % 2 == 0) ? code : (uint8_t)(code << 4);
        }
        for (int64_t b = 0; b < nblk; ++b) {
            const int64_t c = (b * 16) / kNvfp4TileK;
            scales[n * nblk + b] =
                sin[(g * C + c) * kNvfp4TileScaleBytes + nvfp4_scale_offset(r, (int)(b % (kNvfp4TileK / 16)))];
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
    const int64_t C = round_up(K, kFp8TileK) / kFp8TileK;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kFp8TileK;
            out[(g * C + c) * kTileCodeBytes + fp8_code_offset(r, (int)(k % kFp8TileK))] = q[n * K + k];
        }
    }
    return SKINNY_OK;
}

extern "C" int skinny_unpack_fp8(const void* w_packed, int64_t N, int64_t K, uint8_t* q)
{
    if (!q || !w_packed || !valid_shape(N, K)) return SKINNY_ERR_INVALID_ARG;
    const uint8_t* in = (const uint8_t*)w_packed;
    const int64_t C = round_up(K, kFp8TileK) / kFp8TileK;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t g = n / kTileRows;
        const int r = (int)(n % kTileRows);
        for (int64_t k = 0; k < K; ++k) {
            const int64_t c = k / kFp8TileK;
            q[n * K + k] = in[(g * C + c) * kTileCodeBytes + fp8_code_offset(r, (int)(k % kFp8TileK))];
        }
    }
    return SKINNY_OK;
}
