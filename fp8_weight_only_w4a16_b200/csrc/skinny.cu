// skinny.cu -- sm_100a kernels and C ABI of the weight-only skinny GEMM
//   y[M,N] = x[M,K] . W^T,  M = 1..8,  W in NVFP4 (E2M1 + UE4M3/16 + FP32) or
//   FP8 E4M3 (+ FP32 per output channel), x FP16, FP32 accumulation.
//
// The operation is the decode-time weight-only GEMM of the v100-skinny pages
// (taozi.news article, section "自研 QPN 内核": weights stay compressed on
// their way out of HBM and become FP16 in registers for the tensor cores;
// M=8 is the k=7 speculative-verify round).  The design here is B200-first:
//
//  * One persistent CTA per SM: 16 consumer warps + 1 producer warp.  The
//    producer streams 256-row x 128-column weight tiles (16 KB NVFP4 codes +
//    2 KB block scales, or 32 KB FP8) and the matching slice of x with bulk
//    copies (the TMA engine, cp.async.bulk) into a shared-memory ring of 8
//    (NVFP4) or 6 (FP8) stages guarded by mbarriers, so well over 100 KB per
//    SM is in flight without spending registers on it.
//  * Weights are decoded with Blackwell's native converts: one
//    cvt.rn.f16x2.e2m1x2 per two FP4 codes (exact), the UE4M3 block scale
//    with cvt.rn.f16x2.e4m3x2 and one f16x2 multiply (exact: e2m1 * ue4m3 has
//    <= 6 significant bits and lies in [2^-10, 2688]).  FP8 weights use the
//    exact cvt.rn.f16x2.e4m3x2.
//  * m16n8k16 tensor-core MMAs with FP32 accumulation; the MMA's n = 8
//    columns are the M <= 8 tokens.  The tensor rate this needs (16 flop per
//    weight) is a small fraction of the SM's, so tensor cores are never the
//    bound.  Warps w and w+8 take the two 64-column halves of a tile for the
//    same 32 rows and add their sums (in a fixed order) when a tile is done.
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

// 16 consumer warps + 1 producer warp.  Consumer warp w handles strips
// 2*(w%8) and 2*(w%8)+1 of every tile, in K chunk w/8; warps w and w+8 thus
// hold the two K halves of the same 32 rows and add them at flush time.
constexpr int kConsumerWarps = 16;
constexpr int kPairs = kConsumerWarps / 2;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
constexpr int kMaxDevices = 64;

static_assert(kPairs * 2 == kStrips, "two strips per consumer warp");

// Barrier ids: 0 = __syncthreads, 1 = the 16 consumer warps, 2 = warps 0..7.
constexpr uint32_t kBarConsumers = 1, kBarLow = 2;

__device__ unsigned int g_device_error;

template <int FMT>
struct Tile;

// One ring stage holds kUnits consecutive tiles, fetched by ONE bulk copy:
// every cp.async.bulk costs its issuing thread on the order of 150 ns on
// B200, so copies must be large (>= 32 KB) to stream HBM at full rate.
template <>
struct Tile<SKINNY_FMT_NVFP4> {
    static constexpr int kBytes = kNvfp4TileBytes;        // 16 KB codes + 2 KB scales
    static constexpr int kScalesOff = kNvfp4TileCodeBytes;
    static constexpr int kUnits = 2;
    static constexpr int kStages = 5;
};

template <>
struct Tile<SKINNY_FMT_FP8> {
    static constexpr int kBytes = kFp8TileBytes;
    static constexpr int kScalesOff = 0;
    static constexpr int kUnits = 2;
    static constexpr int kStages = 3;
};

// Shared memory: kStages ring stages of kUnits tiles, then the flush exchange
// buffer (two parities of 8 pairs x 2 strips x 32 lanes x float4), then the
// mbarriers.
template <int FMT>
struct Smem {
    static constexpr int kStages = Tile<FMT>::kStages;
    static constexpr int kStageBytes = Tile<FMT>::kUnits * Tile<FMT>::kBytes;
    static constexpr int kXchgOff = kStages * kStageBytes;
    static constexpr int kXchgBytes = 2 * kPairs * 2 * 32 * 16;
    static constexpr int kBarOff = kXchgOff + kXchgBytes;
    static constexpr int kBytes = kBarOff + 2 * kStages * 8 + 16;
    static_assert(kStageBytes % 16 == 0, "stage alignment");
    static_assert(kBytes <= 232448, "shared memory per CTA");
};

struct Params {
    const uint16_t* x;            // [M][K] fp16 bits
    const uint8_t* codes;         // packed tiles (NVFP4 tiles carry their block scales)
    const float* channel_scale;   // FP8 per-channel scale [N]
    void* y;                      // [M][N]
    int* counters;                // [G] arrival tickets (split-K only)
    float4* partials;             // [P][2][8 pairs][2 strips][32 lanes] (split-K only)
    float out_scale;              // NVFP4 per-tensor scale (FP8: unused, the channel scales apply)
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

__device__ __forceinline__ int partial_index(int cta, int slot, int pair, int lane)
{
    return ((cta * 2 + slot) * kPairs + pair) * 64 + lane;  // + 32 for the pair's second strip
}

template <int FMT>
__device__ __forceinline__ void epilogue(const Params& p, const float (&v)[2][4], int g, int pair, int lane)
{
    const int gid = lane >> 2, t = lane & 3;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int n = g * kTileRows + (2 * pair + q) * kStripRows + gid + 8 * h;
            if (n >= p.N) continue;
            const float sc = (FMT == SKINNY_FMT_NVFP4) ? p.out_scale : p.channel_scale[n];
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

// Finish row tile g.  Warps 8..15 hand their K half to warps 0..7 (which add
// chunk 0 + chunk 1, a fixed order).  If this CTA covered the whole K range
// of g, warps 0..7 write y; otherwise they publish the partial sums, take a
// ticket, and the last contributor adds all partials in CTA order.
template <int FMT>
__device__ void flush(const Params& p, const float (&acc)[2][4], int g, int slot, int parity, uint8_t* smem,
                      volatile int* last_flag, int b, int P, int UQ, int warp, int lane)
{
    float4* xchg = reinterpret_cast<float4*>(smem + Smem<FMT>::kXchgOff) + parity * (kPairs * 64);
    const int pair = warp & (kPairs - 1);
    if (warp >= kPairs) {
        xchg[pair * 64 + lane] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
        xchg[pair * 64 + 32 + lane] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
    }
    ptx::named_barrier_sync(kBarConsumers, kConsumerWarps * 32);
    if (warp >= kPairs) return;

    float tot[2][4];
    {
        const float4 h0 = xchg[pair * 64 + lane], h1 = xchg[pair * 64 + 32 + lane];
        tot[0][0] = acc[0][0] + h0.x; tot[0][1] = acc[0][1] + h0.y; tot[0][2] = acc[0][2] + h0.z; tot[0][3] = acc[0][3] + h0.w;
        tot[1][0] = acc[1][0] + h1.x; tot[1][1] = acc[1][1] + h1.y; tot[1][2] = acc[1][2] + h1.z; tot[1][3] = acc[1][3] + h1.w;
    }
    const int c_first = owner_of(g * p.C, P, UQ, p.Q);
    const int c_last = owner_of(g * p.C + p.C - 1, P, UQ, p.Q);
    if (c_first == c_last) {
        epilogue<FMT>(p, tot, g, pair, lane);
        return;
    }
    float4* mine = p.partials + partial_index(b, slot, pair, lane);
    mine[0] = make_float4(tot[0][0], tot[0][1], tot[0][2], tot[0][3]);
    mine[32] = make_float4(tot[1][0], tot[1][1], tot[1][2], tot[1][3]);
    ptx::named_barrier_sync(kBarLow, kPairs * 32);
    if (threadIdx.x == 0) {
        __threadfence();  // release: the CTA's partials (ordered before by the barrier)
        const int old = atomicAdd(&p.counters[g], 1);
        __threadfence();  // acquire: the other contributors' partials
        *last_flag = (old == c_last - c_first);
    }
    ptx::named_barrier_sync(kBarLow, kPairs * 32);
    if (*last_flag) {
        // Add the contributors' partials in CTA order; their loads are issued in
        // batches of kBatch so that the L2 round trips overlap.
        constexpr int kBatch = 2;
        float sum[2][4] = {};
        for (int c0 = c_first; c0 <= c_last; c0 += kBatch) {
            float4 v[kBatch][2];
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                const int cc = c0 + k;
                if (cc <= c_last && cc != b) {
                    const int sl = (g == range_start(cc, P, UQ, p.Q) / p.C) ? 0 : 1;
                    const float4* src = p.partials + partial_index(cc, sl, pair, lane);
                    v[k][0] = __ldcg(src);
                    v[k][1] = __ldcg(src + 32);
                } else {
                    v[k][0] = make_float4(tot[0][0], tot[0][1], tot[0][2], tot[0][3]);
                    v[k][1] = make_float4(tot[1][0], tot[1][1], tot[1][2], tot[1][3]);
                }
            }
#pragma unroll
            for (int k = 0; k < kBatch; ++k) {
                if (c0 + k > c_last) break;
                sum[0][0] += v[k][0].x; sum[0][1] += v[k][0].y; sum[0][2] += v[k][0].z; sum[0][3] += v[k][0].w;
                sum[1][0] += v[k][1].x; sum[1][1] += v[k][1].y; sum[1][2] += v[k][1].z; sum[1][3] += v[k][1].w;
            }
        }
        epilogue<FMT>(p, sum, g, pair, lane);
        if (threadIdx.x == 0) p.counters[g] = 0;  // ready for the next call
    }
}

template <int FMT>
__device__ void produce(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, int u_begin,
                        int n_units)
{
    using S = Smem<FMT>;
    constexpr int kStages = S::kStages, kUnits = Tile<FMT>::kUnits;
    const uint64_t pol_w = ptx::policy_evict_first();
    const int n_stages = (n_units + kUnits - 1) / kUnits;
    int issued = 0;
    for (int q = 0; q < n_stages; ++q) {
        const int s = q % kStages;
        if (q >= kStages && !ptx::mbar_wait(&empty[s], ((q / kStages) & 1) ^ 1, kWaitLimitNs)) {
            atomicOr(&g_device_error, 2u);
            break;
        }
        const int u0 = u_begin + q * kUnits;
        const uint32_t bytes = (uint32_t)min(kUnits, n_units - q * kUnits) * Tile<FMT>::kBytes;
        ptx::mbar_arrive_expect_tx(&full[s], bytes);
        ptx::bulk_g2s(smem + s * S::kStageBytes, p.codes + (size_t)u0 * Tile<FMT>::kBytes, bytes, &full[s], pol_w);
        issued = q + 1;
    }
    // No bulk copy may still be landing in this CTA's shared memory at exit.
    for (int q = max(0, issued - kStages); q < issued; ++q)
        if (!ptx::mbar_wait(&full[q % kStages], (q / kStages) & 1, kWaitLimitNs)) atomicOr(&g_device_error, 4u);
}

// The B fragments of one K tile for this lane: token gid (row xrow of x),
// logical columns [kb, kb+16), as 8 f16x2 words read straight from x
// (read-only, L1-cached).  Tokens >= M (valid = false) and columns >= K read
// as zero; K % 16 == 0, so the 16 columns are all in range or all out.
__device__ __forceinline__ void load_b(const uint16_t* xrow, bool valid, int kb, int K, uint32_t (&bx)[8])
{
    uint4 x0 = make_uint4(0, 0, 0, 0), x1 = make_uint4(0, 0, 0, 0);
    if (valid && kb < K) {
        const uint4* xp = reinterpret_cast<const uint4*>(xrow + kb);
        x0 = __ldg(xp);
        x1 = __ldg(xp + 1);
    }
    bx[0] = x0.x; bx[1] = x0.y; bx[2] = x0.z; bx[3] = x0.w;
    bx[4] = x1.x; bx[5] = x1.y; bx[6] = x1.z; bx[7] = x1.w;
}

// Per-warp state of the consumer loop.  A warp owns strips 2*pair and
// 2*pair+1 of every tile in K chunk ch, and keeps one accumulator per strip and
// per unit parity (the two tiles of a stage are processed together, so four
// independent MMA chains hide the tensor-core latency); the parities are added
// in a fixed order when a row tile is flushed.
template <int FMT>
struct Consumer {
    float acc[2][2][4];     // [unit parity][strip][fragment]
    uint32_t lane_codes;    // this lane's code bytes of strip 2*pair, chunk ch, inside a tile
    uint32_t lane_scale;    // this lane's scale word of strip 2*pair, chunk ch (NVFP4)
    const uint16_t* xrow;   // x row of token gid
    bool xvalid;            // gid < M
    int K;

    __device__ __forceinline__ void zero()
    {
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[u][q][r] = 0.f;
    }

    // The per-strip sums of both parities (fixed order).
    __device__ __forceinline__ void total(float (&tot)[2][4]) const
    {
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int r = 0; r < 4; ++r) tot[q][r] = acc[0][q][r] + acc[1][q][r];
    }

    // NU (1 or 2) consecutive units of one row tile, tiles at shared addresses
    // tile[u], activations bx[u]: all shared loads first, then the decode and
    // MMAs of the NU x 2 strip chunks interleaved step by step.
    template <int NU>
    __device__ __forceinline__ void compute(const uint32_t (&tile)[2], const uint32_t (&bx)[2][8])
    {
        if constexpr (FMT == SKINNY_FMT_NVFP4) {
            uint4 cw[NU][2];
            uint32_t s0[NU][2], s8[NU][2];
#pragma unroll
            for (int u = 0; u < NU; ++u)
#pragma unroll
                for (int q = 0; q < 2; ++q) cw[u][q] = ptx::lds128(tile[u] + lane_codes + q * 1024);
#pragma unroll
            for (int u = 0; u < NU; ++u)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const uint32_t sc = ptx::e4m3x2_to_f16x2(ptx::lds16(tile[u] + lane_scale + q * 128));
                    s0[u][q] = ptx::dup_lo(sc);   // scale of row gid
                    s8[u][q] = ptx::dup_hi(sc);   // scale of row gid+8
                }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int u = 0; u < NU; ++u)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint32_t w = j == 0 ? cw[u][q].x : j == 1 ? cw[u][q].y : j == 2 ? cw[u][q].z : cw[u][q].w;
                        uint32_t h[4];
                        ptx::e2m1x8_to_f16x8(w, h);
                        const uint32_t a[4] = {ptx::hmul2(h[0], s0[u][q]), ptx::hmul2(h[1], s8[u][q]),
                                               ptx::hmul2(h[2], s0[u][q]), ptx::hmul2(h[3], s8[u][q])};
                        ptx::mma_f16_16816(acc[u][q], a, bx[u][2 * j], bx[u][2 * j + 1]);
                    }
        } else {
            uint4 cw[NU][2][2];
#pragma unroll
            for (int u = 0; u < NU; ++u)
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    cw[u][q][0] = ptx::lds128(tile[u] + lane_codes + q * 2048);
                    cw[u][q][1] = ptx::lds128(tile[u] + lane_codes + q * 2048 + 16);
                }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int u = 0; u < NU; ++u)
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint4& v = cw[u][q][j >> 1];
                        const uint32_t w0 = (j & 1) ? v.z : v.x, w1 = (j & 1) ? v.w : v.y;
                        uint32_t a[4];
                        ptx::e4m3x4_to_f16x4(w0, a[0], a[1]);
                        ptx::e4m3x4_to_f16x4(w1, a[2], a[3]);
                        ptx::mma_f16_16816(acc[u][q], a, bx[u][2 * j], bx[u][2 * j + 1]);
                    }
        }
    }
};

// The unit coordinates (row tile g, K tile c) of unit u_begin + i.
struct Cursor {
    int g, c;
    __device__ __forceinline__ void next(int C)
    {
        if (++c == C) {
            c = 0;
            ++g;
        }
    }
};

template <int FMT>
__device__ void consume(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, volatile int* last_flag,
                        int u_begin, int n_units, int b, int P, int UQ, int warp, int lane)
{
    using S = Smem<FMT>;
    constexpr int kStages = S::kStages, kUnits = Tile<FMT>::kUnits;
    static_assert(kUnits == 2, "the consumer processes two tiles per stage");
    constexpr int kTileBytes = Tile<FMT>::kBytes;
    const int gid = lane >> 2, t = lane & 3;
    const int ch = warp / kPairs, pair = warp % kPairs;
    const int kb_lane = ch * kChunkK + 16 * t;

    Consumer<FMT> w;
    w.zero();
    if constexpr (FMT == SKINNY_FMT_NVFP4) {
        w.lane_codes = (2 * pair) * 1024 + ch * 512 + lane * 16;
        w.lane_scale = Tile<FMT>::kScalesOff + (2 * pair) * 128 + ch * 64 + t * 16 + gid * 2;
    } else {
        w.lane_codes = (2 * pair) * 2048 + ch * 1024 + lane * 32;
        w.lane_scale = 0;
    }
    w.xvalid = gid < p.M;
    w.xrow = p.x + (size_t)(w.xvalid ? gid : 0) * p.K;
    w.K = p.K;

    const int first_g = u_begin / p.C;
    int cur_g = first_g, parity = 0;
    Cursor cu{first_g, u_begin - first_g * p.C};   // first unit of the stage being processed
    const uint32_t smem32 = ptx::smem_addr(smem);
    const int n_stages = (n_units + kUnits - 1) / kUnits;

    bool ok = true;
    int s = 0;
    uint32_t phase = 0;
    for (int q = 0; q < n_stages; ++q) {
        const int n_here = min(kUnits, n_units - q * kUnits);
        Cursor c1 = cu;
        c1.next(p.C);
        // Activations of this stage's units (L1/L2 hits; in flight during the wait below).
        uint32_t bx[2][8];
        load_b(w.xrow, w.xvalid, cu.c * kTileK + kb_lane, p.K, bx[0]);
        if (n_here > 1) load_b(w.xrow, w.xvalid, c1.c * kTileK + kb_lane, p.K, bx[1]);

        if (ok) {
            // All lanes agree on the outcome, so the warp stays converged.
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(&full[s], phase, kWaitLimitNs));
            if (!ok && lane == 0) atomicOr(&g_device_error, 1u);
        }
        const uint32_t tiles[2] = {smem32 + s * S::kStageBytes, smem32 + s * S::kStageBytes + kTileBytes};
        // unit 0 of the stage
        if (cu.g != cur_g) {
            float tot[2][4];
            w.total(tot);
            flush<FMT>(p, tot, cur_g, cur_g == first_g ? 0 : 1, parity, smem, last_flag, b, P, UQ, warp, lane);
            parity ^= 1;
            w.zero();
            cur_g = cu.g;
        }
        if (n_here == 2 && c1.g == cur_g) {
            if (ok) w.template compute<2>(tiles, bx);                 // both units, one row tile
        } else {
            if (ok) w.template compute<1>(tiles, bx);                 // unit 0 alone
            if (n_here == 2) {                                        // unit 1 starts a new row tile
                float tot[2][4];
                w.total(tot);
                flush<FMT>(p, tot, cur_g, cur_g == first_g ? 0 : 1, parity, smem, last_flag, b, P, UQ, warp, lane);
                parity ^= 1;
                w.zero();
                cur_g = c1.g;
                const uint32_t t1[2] = {tiles[1], tiles[1]};
                uint32_t b1[2][8];
#pragma unroll
                for (int k = 0; k < 8; ++k) b1[0][k] = b1[1][k] = bx[1][k];
                if (ok) w.template compute<1>(t1, b1);
            }
        }
        cu = c1;
        cu.next(p.C);
        if (ok) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[s]);
        }
        if (++s == kStages) {
            s = 0;
            phase ^= 1;
        }
    }
    if (n_units > 0) {
        float tot[2][4];
        w.total(tot);
        flush<FMT>(p, tot, cur_g, cur_g == first_g ? 0 : 1, parity, smem, last_flag, b, P, UQ, warp, lane);
    }
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params p)
{
    using S = Smem<FMT>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
    uint64_t* empty = full + S::kStages;
    volatile int* last_flag = reinterpret_cast<volatile int*>(empty + S::kStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x, b = blockIdx.x;
    const int UQ = p.U / p.Q;
    const int u_begin = range_start(b, P, UQ, p.Q);
    const int n_units = range_start(b + 1, P, UQ, p.Q) - u_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S::kStages; ++s) {
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
                                 Smem<SKINNY_FMT_NVFP4>::kBytes) != cudaSuccess)
            return SKINNY_ERR_CUDA;
        if (cudaFuncSetAttribute(gemm_kernel<SKINNY_FMT_FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Smem<SKINNY_FMT_FP8>::kBytes) != cudaSuccess)
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

static int make_plan(int fmt, int64_t N, int64_t K, int sms, bool split, Plan* pl)
{
    const int64_t G = (N + kTileRows - 1) / kTileRows;
    (void)fmt;
    const int64_t C = (K + kTileK - 1) / kTileK;
    if (G * C >= (int64_t(1) << 31)) return SKINNY_ERR_UNSUPPORTED;
    pl->G = (int)G;
    pl->C = (int)C;
    pl->U = (int)(G * C);
    const int UQ = split ? pl->U : pl->G;
    pl->P = UQ < sms ? UQ : sms;
    pl->partial_bytes = (size_t)sms * 2 * kPairs * 64 * sizeof(float4);
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
    gemm_kernel<FMT><<<pl.P, kThreads, Smem<FMT>::kBytes, stream>>>(p);
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

extern "C" int skinny_nvfp4_gemm(const void* x, int M, int64_t K, const void* w_packed, float global_scale,
                                 int64_t N, void* y, int out_dtype, void* workspace, size_t workspace_bytes,
                                 void* stream)
{
    int rc = check_common(x, M, K, N, y, out_dtype, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16)) return SKINNY_ERR_ALIGNMENT;
    Params p{};
    p.x = static_cast<const uint16_t*>(x);
    p.codes = static_cast<const uint8_t*>(w_packed);
    p.y = y;
    p.out_scale = global_scale;
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
    p.out_scale = 1.0f;
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
                                           float global_scale, int64_t N, void* y, int out_dtype, void* stream)
{
    int rc = check_common(x, M, K, N, y, out_dtype, nullptr);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16)) return SKINNY_ERR_ALIGNMENT;
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
    return skinny_nvfp4_gemm(x, M, K, w_packed, global_scale, N, y, out_dtype, ws, kStaticWorkspaceBytes, stream);
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
