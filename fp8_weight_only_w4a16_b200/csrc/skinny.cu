// skinny.cu -- sm_100a kernels and C ABI of the weight-only skinny GEMM
//   y[M,N] = x[M,K] . W^T,  M = 1..8,  W in NVFP4 (E2M1 + UE4M3/16 + FP32) or
//   FP8 E4M3 (+ FP32 per output channel), x FP16, FP32 accumulation.
//
// The operation is the decode-time weight-only GEMM of the v100-skinny pages
// (taozi.news article, section "自研 QPN 内核": weights stay compressed on
// their way out of HBM and become FP16 in registers for the tensor cores;
// M=8 is the k=7 speculative-verify round).  The design here is B200-first:
//
//  * One persistent CTA per SM: 8 consumer warps + 1 producer warp.  The
//    producer streams 16 KB weight tiles (plus their 2 KB of NVFP4 block
//    scales and the matching slice of x) with bulk copies (the TMA engine,
//    cp.async.bulk) into an 8-stage shared-memory ring guarded by mbarriers,
//    so >100 KB per SM is in flight without spending registers on it.
//  * Consumers decode with Blackwell's native FP4/FP8 converts
//    (cvt.rn.f16x2.e2m1x2 / .e4m3x2, exact), apply the UE4M3 block scale with
//    one f16x2 multiply (exact: e2m1 * ue4m3 has <= 6 significant bits and
//    lies in [2^-10, 2688]), and feed m16n8k16 tensor-core MMAs with FP32
//    accumulation.  The MMA's n = 8 columns are the M <= 8 tokens.  The
//    tensor rate this needs (16 flop per weight) is a small fraction of the
//    SM's, so the kernel stays bound by HBM at every M.
//  * Work is balanced by "stream-K": the grid's CTAs take equal contiguous
//    ranges of the tile sequence.  A 256-row tile whose K range is split
//    between CTAs is finished by the last CTA to arrive (an atomic ticket, no
//    spinning), which adds the FP32 partials in CTA order -- so results are
//    bitwise reproducible.  Without a workspace, CTAs take whole row tiles.
//  * Every wait is bounded (1 s of global time); a wait that gives up sets a
//    bit in g_device_error and its CTA winds down instead of hanging.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/skinny.h"
#include "layout.h"
#include "ptx.cuh"

namespace skinny {

constexpr int kConsumerWarps = 8;                  // each owns 2 strips (32 rows) of a tile
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 8;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
constexpr int kMaxDevices = 64;

static_assert(kConsumerWarps * 2 == kStrips, "two strips per consumer warp");

__device__ unsigned int g_device_error;

template <int FMT>
struct Tile;

template <>
struct Tile<SKINNY_FMT_NVFP4> {
    static constexpr int kK = kNvfp4TileK;
    static constexpr int kScaleBytes = kNvfp4TileScaleBytes;
};

template <>
struct Tile<SKINNY_FMT_FP8> {
    static constexpr int kK = kFp8TileK;
    static constexpr int kScaleBytes = 0;
};

// One ring stage: [codes 16384 | scales (NVFP4 only) | x: 8 rows of kK halfs].
// x rows are padded by 16 bytes so that the lanes of a warp reading their B
// fragments hit 32 distinct banks.
template <int FMT>
struct Stage {
    static constexpr int kK = Tile<FMT>::kK;
    static constexpr int kChunks = kK / kChunkK;
    static constexpr int kScalesOff = kTileCodeBytes;
    static constexpr int kXOff = kTileCodeBytes + Tile<FMT>::kScaleBytes;
    static constexpr int kXStride = kK * 2 + 16;
    static constexpr int kBytes = kXOff + SKINNY_MAX_M * kXStride;
    static constexpr int kSmem = kStages * kBytes + 2 * kStages * 8 + 16;
    static_assert(kBytes % 16 == 0, "stage alignment");
};

struct Params {
    const uint16_t* x;            // [M][K] fp16 bits
    const uint8_t* codes;         // packed tiles
    const uint8_t* scales;        // packed NVFP4 scale tiles
    const float* channel_scale;   // FP8 per-channel scale [N]
    void* y;                      // [M][N]
    int* counters;                // [G] arrival tickets (split-K only)
    float4* partials;             // [P][2][8 warps][2 strips][32 lanes] (split-K only)
    float global_scale;
    int M, K, N;
    int C;                        // K tiles per row tile
    int U;                        // tiles in total (G * C)
    int Q;                        // scheduling quantum: 1 (split K) or C (whole row tiles)
    int out_f32;
};

// CTA b of P takes quanta [b*UQ/P, (b+1)*UQ/P) of the UQ = U/Q quanta.
__host__ __device__ __forceinline__ int range_start(int b, int P, int UQ, int Q)
{
    return (int)(((int64_t)b * UQ) / P) * Q;
}

// The CTA whose range holds tile u (inverse of range_start).
__device__ __forceinline__ int owner_of(int u, int P, int UQ, int Q)
{
    return (int)((((int64_t)(u / Q) + 1) * P - 1) / UQ);
}

__device__ __forceinline__ int partial_index(int cta, int slot, int warp, int lane)
{
    return ((cta * 2 + slot) * kConsumerWarps + warp) * 64 + lane;  // + 32 for the warp's second strip
}

template <int FMT>
__device__ __forceinline__ void epilogue(const Params& p, const float (&v)[2][4], int g, int warp, int lane)
{
    const int gid = lane >> 2, t = lane & 3;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = g * kTileRows + (2 * warp + q) * kStripRows + gid + 8 * h;
            if (n >= p.N) continue;
            const float sc = (FMT == SKINNY_FMT_NVFP4) ? p.global_scale : p.channel_scale[n];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int m = 2 * t + e;
                if (m >= p.M) continue;
                const float val = v[q][2 * h + e] * sc;
                const size_t idx = (size_t)m * p.N + n;
                if (p.out_f32)
                    static_cast<float*>(p.y)[idx] = val;
                else
                    static_cast<__half*>(p.y)[idx] = __float2half_rn(val);
            }
        }
    }
}

// Finish the accumulators of row tile g.  If this CTA covered the whole K
// range of g, write y directly; otherwise publish the partial sums, take a
// ticket, and let the last contributor add all partials in CTA order.
template <int FMT>
__device__ void flush(const Params& p, const float (&acc)[2][4], int g, int slot, volatile int* last_flag,
                      int b, int P, int UQ, int warp, int lane)
{
    const int c_first = owner_of(g * p.C, P, UQ, p.Q);
    const int c_last = owner_of(g * p.C + p.C - 1, P, UQ, p.Q);
    if (c_first == c_last) {
        epilogue<FMT>(p, acc, g, warp, lane);
        return;
    }
    float4* mine = p.partials + partial_index(b, slot, warp, lane);
    mine[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
    mine[32] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
    __threadfence();
    ptx::named_barrier_sync(1, kConsumerWarps * 32);
    if (threadIdx.x == 0) {
        const int old = atomicAdd(&p.counters[g], 1);
        *last_flag = (old == c_last - c_first);
    }
    ptx::named_barrier_sync(1, kConsumerWarps * 32);
    if (*last_flag) {
        __threadfence();
        float tot[2][4] = {};
        for (int cc = c_first; cc <= c_last; ++cc) {
            float part[2][4];
            if (cc == b) {
#pragma unroll
                for (int q = 0; q < 2; ++q)
#pragma unroll
                    for (int r = 0; r < 4; ++r) part[q][r] = acc[q][r];
            } else {
                const int sl = (g == range_start(cc, P, UQ, p.Q) / p.C) ? 0 : 1;
                const float4* src = p.partials + partial_index(cc, sl, warp, lane);
                const float4 v0 = __ldcg(src), v1 = __ldcg(src + 32);
                part[0][0] = v0.x; part[0][1] = v0.y; part[0][2] = v0.z; part[0][3] = v0.w;
                part[1][0] = v1.x; part[1][1] = v1.y; part[1][2] = v1.z; part[1][3] = v1.w;
            }
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) tot[q][r] += part[q][r];
        }
        epilogue<FMT>(p, tot, g, warp, lane);
        if (threadIdx.x == 0) p.counters[g] = 0;  // ready for the next call
    }
}

template <int FMT>
__device__ void produce(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, int u_begin,
                        int n_units)
{
    using S = Stage<FMT>;
    const uint64_t pol_w = ptx::policy_evict_first();
    const uint64_t pol_x = ptx::policy_evict_last();
    int issued = 0;
    for (int i = 0; i < n_units; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !ptx::mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, kWaitLimitNs)) {
            atomicOr(&g_device_error, 2u);
            break;
        }
        const int u = u_begin + i;
        const int k0 = (u % p.C) * S::kK;
        const int xbytes = min(S::kK, p.K - k0) * 2;  // K % 16 == 0: a multiple of 32 bytes
        uint8_t* st = smem + s * S::kBytes;
        ptx::mbar_arrive_expect_tx(&full[s], kTileCodeBytes + Tile<FMT>::kScaleBytes + p.M * xbytes);
        ptx::bulk_g2s(st, p.codes + (size_t)u * kTileCodeBytes, kTileCodeBytes, &full[s], pol_w);
        if constexpr (FMT == SKINNY_FMT_NVFP4)
            ptx::bulk_g2s(st + S::kScalesOff, p.scales + (size_t)u * kNvfp4TileScaleBytes, kNvfp4TileScaleBytes,
                          &full[s], pol_w);
        for (int m = 0; m < p.M; ++m)
            ptx::bulk_g2s(st + S::kXOff + m * S::kXStride, p.x + (size_t)m * p.K + k0, (uint32_t)xbytes, &full[s],
                          pol_x);
        issued = i + 1;
    }
    // No bulk copy may still be landing in this CTA's shared memory at exit.
    for (int i = max(0, issued - kStages); i < issued; ++i)
        if (!ptx::mbar_wait(&full[i % kStages], (i / kStages) & 1, kWaitLimitNs)) atomicOr(&g_device_error, 4u);
}

template <int FMT>
__device__ void consume(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, volatile int* last_flag,
                        int u_begin, int n_units, int b, int P, int UQ, int warp, int lane)
{
    using S = Stage<FMT>;
    const int gid = lane >> 2, t = lane & 3;
    float acc[2][4] = {};
    bool ok = true;
    const int first_g = u_begin / p.C;
    int cur_g = first_g;
    for (int i = 0; i < n_units; ++i) {
        const int u = u_begin + i;
        const int g = u / p.C, c = u % p.C;
        if (g != cur_g) {
            flush<FMT>(p, acc, cur_g, cur_g == first_g ? 0 : 1, last_flag, b, P, UQ, warp, lane);
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[q][r] = 0.f;
            cur_g = g;
        }
        const int s = i % kStages;
        if (ok) {
            // All lanes agree on the outcome, so the warp stays converged.
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(&full[s], (i / kStages) & 1, kWaitLimitNs));
            if (!ok && lane == 0) atomicOr(&g_device_error, 1u);
        }
        if (!ok) continue;
        const uint8_t* st = smem + s * S::kBytes;
#pragma unroll
        for (int ch = 0; ch < S::kChunks; ++ch) {
            // B fragments: token gid, logical k [kb, kb+16) of this chunk.
            const int kb = c * S::kK + ch * kChunkK + 16 * t;
            uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
            if (gid < p.M && kb < p.K) {
                const uint4* xp = reinterpret_cast<const uint4*>(st + S::kXOff + gid * S::kXStride + ch * 128 + 32 * t);
                x0 = xp[0];
                x1 = xp[1];
            }
            const uint32_t bx[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int strip = 2 * warp + q;
                if constexpr (FMT == SKINNY_FMT_NVFP4) {
                    const uint4 cw = *reinterpret_cast<const uint4*>(st + strip * 1024 + ch * 512 + lane * 16);
                    const uint16_t sw = *reinterpret_cast<const uint16_t*>(st + S::kScalesOff + strip * 128 + ch * 64 +
                                                                           t * 16 + gid * 2);
                    const uint32_t sc = ptx::e4m3x2_to_f16x2(sw);
                    const uint32_t s_row0 = ptx::dup_lo(sc), s_row8 = ptx::dup_hi(sc);
                    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t h[4];
                        ptx::e2m1x8_to_f16x8(words[j], h);
                        const uint32_t a[4] = {ptx::hmul2(h[0], s_row0), ptx::hmul2(h[1], s_row8),
                                               ptx::hmul2(h[2], s_row0), ptx::hmul2(h[3], s_row8)};
                        ptx::mma_f16_16816(acc[q], a, bx[2 * j], bx[2 * j + 1]);
                    }
                } else {
                    const uint4* cp = reinterpret_cast<const uint4*>(st + strip * 1024 + lane * 32);
                    const uint4 c0 = cp[0], c1 = cp[1];
                    const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t a[4];
                        ptx::e4m3x4_to_f16x4(words[2 * j], a[0], a[1]);
                        ptx::e4m3x4_to_f16x4(words[2 * j + 1], a[2], a[3]);
                        ptx::mma_f16_16816(acc[q], a, bx[2 * j], bx[2 * j + 1]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&empty[s]);
    }
    if (n_units > 0) flush<FMT>(p, acc, cur_g, cur_g == first_g ? 0 : 1, last_flag, b, P, UQ, warp, lane);
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params p)
{
    using S = Stage<FMT>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * S::kBytes);
    uint64_t* empty = full + kStages;
    volatile int* last_flag = reinterpret_cast<volatile int*>(empty + kStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, b = blockIdx.x;
    const int UQ = p.U / p.Q;
    const int u_begin = range_start(b, P, UQ, p.Q);
    const int n_units = range_start(b + 1, P, UQ, p.Q) - u_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], kConsumerWarps);
        }
        ptx::fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        if (lane == 0) produce<FMT>(p, smem, full, empty, u_begin, n_units);
        return;
    }
    consume<FMT>(p, smem, full, empty, last_flag, u_begin, n_units, b, P, UQ, warp, lane);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

struct DeviceState {
    bool ready = false;
    int sms = 0;
};

static std::mutex g_mu;
static DeviceState g_dev[kMaxDevices];

// SM count of the current device; sets the kernels' shared-memory limit once.
static int current_device(int* sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SKINNY_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& d = g_dev[dev];
    if (!d.ready) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return SKINNY_ERR_CUDA;
        if (cudaFuncSetAttribute(gemm_kernel<SKINNY_FMT_NVFP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Stage<SKINNY_FMT_NVFP4>::kSmem) != cudaSuccess)
            return SKINNY_ERR_CUDA;
        if (cudaFuncSetAttribute(gemm_kernel<SKINNY_FMT_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Stage<SKINNY_FMT_FP8>::kSmem) != cudaSuccess)
            return SKINNY_ERR_CUDA;
        d.sms = n;
        d.ready = true;
    }
    *sms = d.sms;
    return SKINNY_OK;
}

// Workspace layout (identical for every shape on a device, so one workspace
// can serve calls of different shapes in turn): the partial-sum slots of up
// to one CTA per SM first, then one arrival counter per row tile.
struct Plan {
    int G, C, U, P;
    size_t partial_bytes, workspace_bytes;
};

static int tile_k(int fmt) { return fmt == SKINNY_FMT_NVFP4 ? kNvfp4TileK : kFp8TileK; }

static int make_plan(int fmt, int64_t N, int64_t K, int sms, bool split, Plan* pl)
{
    const int64_t G = (N + kTileRows - 1) / kTileRows;
    const int64_t C = (K + tile_k(fmt) - 1) / tile_k(fmt);
    if (G * C >= (int64_t(1) << 31)) return SKINNY_ERR_UNSUPPORTED;
    pl->G = (int)G;
    pl->C = (int)C;
    pl->U = (int)(G * C);
    const int UQ = split ? pl->U : pl->G;
    pl->P = UQ < sms ? UQ : sms;
    pl->partial_bytes = (size_t)sms * 2 * kConsumerWarps * 64 * sizeof(float4);
    pl->workspace_bytes = pl->partial_bytes + ((size_t)G * sizeof(int) + 255) / 256 * 256;
    return SKINNY_OK;
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

static int check_common(const void* x, int M, int64_t K, int64_t N, const void* y, int out_dtype,
                        const void* workspace)
{
    if (!x || !y) return SKINNY_ERR_INVALID_ARG;
    if (out_dtype != SKINNY_OUT_F16 && out_dtype != SKINNY_OUT_F32) return SKINNY_ERR_INVALID_ARG;
    if (K <= 0 || K % 16 != 0 || N <= 0) return SKINNY_ERR_INVALID_ARG;
    if (M < 1 || M > SKINNY_MAX_M) return SKINNY_ERR_UNSUPPORTED;
    if (K > (int64_t(1) << 30) || N > (int64_t(1) << 30)) return SKINNY_ERR_UNSUPPORTED;
    if (!aligned(x, 16) || !aligned(y, 4) || (workspace && !aligned(workspace, 16))) return SKINNY_ERR_ALIGNMENT;
    return SKINNY_OK;
}

template <int FMT>
static int launch(Params p, int64_t N, int64_t K, void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    int sms = 0;
    int rc = current_device(&sms);
    if (rc != SKINNY_OK) return rc;
    const bool split = workspace != nullptr;
    Plan pl;
    rc = make_plan(FMT, N, K, sms, split, &pl);
    if (rc != SKINNY_OK) return rc;
    if (split && workspace_bytes < pl.workspace_bytes) return SKINNY_ERR_WORKSPACE;
    p.C = pl.C;
    p.U = pl.U;
    p.Q = split ? 1 : pl.C;
    p.partials = split ? static_cast<float4*>(workspace) : nullptr;
    p.counters = split ? reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + pl.partial_bytes) : nullptr;
    gemm_kernel<FMT><<<pl.P, kThreads, Stage<FMT>::kSmem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? SKINNY_OK : SKINNY_ERR_CUDA;
}

}  // namespace skinny

using namespace skinny;

extern "C" const char* skinny_status_string(int status)
{
    switch (status) {
        case SKINNY_OK: return "SKINNY_OK";
        case SKINNY_ERR_INVALID_ARG: return "SKINNY_ERR_INVALID_ARG";
        case SKINNY_ERR_UNSUPPORTED: return "SKINNY_ERR_UNSUPPORTED";
        case SKINNY_ERR_ALIGNMENT: return "SKINNY_ERR_ALIGNMENT";
        case SKINNY_ERR_CUDA: return "SKINNY_ERR_CUDA";
        case SKINNY_ERR_WORKSPACE: return "SKINNY_ERR_WORKSPACE";
        default: return "SKINNY_ERR_UNKNOWN";
    }
}

extern "C" int skinny_version(void) { return 100; }

extern "C" int skinny_workspace_bytes(int fmt, int M, int64_t N, int64_t K, size_t* bytes)
{
    if (!bytes || (fmt != SKINNY_FMT_NVFP4 && fmt != SKINNY_FMT_FP8)) return SKINNY_ERR_INVALID_ARG;
    if (K <= 0 || K % 16 != 0 || N <= 0) return SKINNY_ERR_INVALID_ARG;
    if (M < 1 || M > SKINNY_MAX_M) return SKINNY_ERR_UNSUPPORTED;
    int sms = 0;
    int rc = current_device(&sms);
    if (rc != SKINNY_OK) return rc;
    Plan pl;
    rc = make_plan(fmt, N, K, sms, true, &pl);
    if (rc != SKINNY_OK) return rc;
    *bytes = pl.workspace_bytes;
    return SKINNY_OK;
}

extern "C" int skinny_nvfp4_gemm(const void* x, int M, int64_t K, const void* w_packed, const void* w_scales,
                                 float global_scale, int64_t N, void* y, int out_dtype, void* workspace,
                                 size_t workspace_bytes, void* stream)
{
    int rc = check_common(x, M, K, N, y, out_dtype, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed || !w_scales) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16) || !aligned(w_scales, 16)) return SKINNY_ERR_ALIGNMENT;
    Params p{};
    p.x = static_cast<const uint16_t*>(x);
    p.codes = static_cast<const uint8_t*>(w_packed);
    p.scales = static_cast<const uint8_t*>(w_scales);
    p.y = y;
    p.global_scale = global_scale;
    p.M = M;
    p.K = (int)K;
    p.N = (int)N;
    p.out_f32 = out_dtype == SKINNY_OUT_F32;
    return launch<SKINNY_FMT_NVFP4>(p, N, K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int skinny_fp8_gemm(const void* x, int M, int64_t K, const void* w_packed, const float* channel_scale,
                               int64_t N, void* y, int out_dtype, void* workspace, size_t workspace_bytes,
                               void* stream)
{
    int rc = check_common(x, M, K, N, y, out_dtype, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed || !channel_scale) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16) || !aligned(channel_scale, 4)) return SKINNY_ERR_ALIGNMENT;
    Params p{};
    p.x = static_cast<const uint16_t*>(x);
    p.codes = static_cast<const uint8_t*>(w_packed);
    p.channel_scale = channel_scale;
    p.y = y;
    p.global_scale = 1.0f;
    p.M = M;
    p.K = (int)K;
    p.N = (int)N;
    p.out_f32 = out_dtype == SKINNY_OUT_F32;
    return launch<SKINNY_FMT_FP8>(p, N, K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// NVFP4 GEMM with split-K scratch in a static device array, for callers that
// cannot allocate device memory.
// ---------------------------------------------------------------------------

namespace skinny {

// 4 MiB of split-K scratch per device, reserved when the library's device code
// is loaded on that device and held until the process exits.
constexpr size_t kStaticWorkspaceBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Device address of g_static_workspace on each device.  In host code the
// array's name only stands in for the symbol, so the address is looked up with
// cudaGetSymbolAddress, once per device, while that device is current.
static void* g_static_workspace_addr[kMaxDevices];

static int static_workspace_address(void** addr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SKINNY_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_static_workspace_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) return SKINNY_ERR_CUDA;
        g_static_workspace_addr[dev] = p;
    }
    *addr = g_static_workspace_addr[dev];
    return SKINNY_OK;
}

}  // namespace skinny

extern "C" size_t skinny_static_workspace_capacity(void) { return kStaticWorkspaceBytes; }

extern "C" int skinny_nvfp4_gemm_static_ws(const void* x, int M, int64_t K, const void* w_packed,
                                           const void* w_scales, float global_scale, int64_t N, void* y,
                                           int out_dtype, void* stream)
{
    int rc = check_common(x, M, K, N, y, out_dtype, nullptr);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed || !w_scales) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16) || !aligned(w_scales, 16)) return SKINNY_ERR_ALIGNMENT;
    int sms = 0;
    rc = current_device(&sms);
    if (rc != SKINNY_OK) return rc;
    Plan pl;
    rc = make_plan(SKINNY_FMT_NVFP4, N, K, sms, true, &pl);
    if (rc != SKINNY_OK) return rc;
    if (pl.workspace_bytes > kStaticWorkspaceBytes) return SKINNY_ERR_UNSUPPORTED;
    void* ws = nullptr;
    rc = static_workspace_address(&ws);
    if (rc != SKINNY_OK) return rc;
    // The array keeps whatever the previous call left; the arrival counters of
    // this call must start at zero, so clear them on the call's stream.
    const size_t counter_bytes = pl.workspace_bytes - pl.partial_bytes;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(static_cast<uint8_t*>(ws) + pl.partial_bytes, 0, counter_bytes, st) != cudaSuccess)
        return SKINNY_ERR_CUDA;
    return skinny_nvfp4_gemm(x, M, K, w_packed, w_scales, global_scale, N, y, out_dtype, ws, kStaticWorkspaceBytes,
                             stream);
}

extern "C" int skinny_device_error(int clear, unsigned* flags)
{
    if (!flags) return SKINNY_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return SKINNY_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return SKINNY_ERR_CUDA;
    *flags = v;
    if (clear) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return SKINNY_ERR_CUDA;
    }
    return SKINNY_OK;
}
