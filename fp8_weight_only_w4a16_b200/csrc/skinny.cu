// skinny.cu -- sm_100a kernels and C ABI of the weight-only skinny GEMM
//   y[M,N] = x[M,K] . W^T,  M = 1..16, W in NVFP4 (E2M1 + UE4M3/16 + FP32) or
//   FP8 E4M3 (+ FP32 per output channel), x FP16, FP32 accumulation.
//
// The operation is the decode-time weight-only GEMM of the v100-skinny pages
// (taozi.news article, section "自研 QPN 内核": weights stay compressed on
// their way out of HBM and become FP16 in registers for the tensor cores;
// M=8 is the k=7 speculative-verify round).  The design here is B200-first:
//
//  * One persistent CTA per SM: 8 consumer warps and a producer warpgroup.
//    Weights stream in 128-row x 512-column tiles (32 KB NVFP4 codes + 4 KB
//    block scales, or 64 KB FP8), one tile per ring stage, each stage ONE
//    bulk copy (the TMA engine, cp.async.bulk): a bulk copy costs its issuing
//    thread ~150 ns, so copies must be large.  Stages are guarded by
//    mbarriers.  One thread of the producer warpgroup refills a slot as soon
//    as every consumer warp has released it, off the consumers' critical
//    path; the warpgroup gives its registers to the consumers (setmaxnreg).
//  * Programmatic dependent launch: a CTA starts streaming its first tiles
//    while the previous kernel in the stream is still finishing, and touches
//    x, y and the workspace only after that kernel has completed.
//  * Activations are read by each lane straight from x (L1-cached), one tile
//    ahead of use in ping-pong registers; they are tiny and shared by all CTAs.
//  * Weights are decoded with Blackwell's native converts: one
//    cvt.rn.f16x2.e2m1x2 per two FP4 codes (exact), the UE4M3 block scale
//    with cvt.rn.f16x2.e4m3x2 and one f16x2 multiply (exact: e2m1 * ue4m3 has
//    <= 6 significant bits and lies in [2^-10, 2688]).  FP8 weights use the
//    exact cvt.rn.f16x2.e4m3x2.
//  * m16n8k16 tensor-core MMAs with FP32 accumulation; the MMA's n = 8
//    columns are the M <= 8 tokens.  The tensor rate this needs (16 flop per
//    weight) is a small fraction of the SM's, so tensor cores are never the
//    bound.
//  * Work is balanced by "stream-K": the grid's CTAs take equal contiguous
//    ranges of the tile sequence and walk them BACKWARDS.  A row tile whose
//    K range is split between CTAs is then finished by its highest-numbered
//    contributor, which reaches it at the end of its range, while every other
//    contributor reached it at the start of its own (or holds nothing else).
//    Contributors publish their FP32 partial sums with plain stores, encoded
//    so that an all-zero word means "not written yet"; the finisher polls for
//    them (bounded), adds them in CTA order -- results are bitwise
//    reproducible -- and zeroes the slots again.  No atomics, no fences, and
//    each CTA publishes at most once.  Without a workspace, CTAs take whole
//    row tiles.
//  * Fused epilogues on the finished FP32 outputs: a per-token argmax (the
//    greedy pick of a vocabulary projection, no logits written) and the
//    SiLU*mul of a gated MLP (gate and up rows packed into the same tile).
//  * Every wait is bounded (1 s of global time); a wait that gives up sets a
//    bit in g_device_error and its CTA winds down instead of hanging.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>
#include <type_traits>

#include "../../include/skinny.h"
#include "layout.h"
#include "ptx.cuh"

namespace skinny {

// Consumer warp w handles kStripsPerWarp consecutive strips (strip group
// sg = w % kStripGroups) and the chunk pair kq = w / kStripGroups (chunks
// 2kq, 2kq+1) of every tile, so the kChunkPairs warps of a strip group hold
// the four K quarters of the same rows and add them at flush time.  Thread 0
// issues the first ring stages; the later ones are issued by a producer
// warpgroup (below), or, built without it, by the consumer warp that is last
// to release the ring slot it refills.
#ifndef SKINNY_STRIPS_PER_WARP
#define SKINNY_STRIPS_PER_WARP 4
#endif
constexpr int kStripsPerWarp = SKINNY_STRIPS_PER_WARP;          // 4: 8 consumer warps, 2: 16
constexpr int kStripGroups = kStrips / kStripsPerWarp;
constexpr int kChunkPairs = kChunks / 2;                        // 4
constexpr int kConsumerWarps = kStripGroups * kChunkPairs;
constexpr int kConsumerThreads = kConsumerWarps * 32;
// With a producer warpgroup (4 warps after the consumers) one thread of it
// refills the ring slots; the consumers only wait, compute and release.  The
// warpgroup hands its registers to the consumers (setmaxnreg).
#ifndef SKINNY_PRODUCER
#define SKINNY_PRODUCER 1
#endif
constexpr bool kProducer = SKINNY_PRODUCER != 0;
constexpr int kProducerWarps = kProducer ? 4 : 0;
constexpr int kThreads = kConsumerThreads + kProducerWarps * 32;
// Registers per thread: at launch (65536 / kThreads, rounded down to 8), then
// after the warpgroups re-balance (producer 24, consumers the rest).
constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;
constexpr int kProducerRegs = 24;
constexpr int kConsumerRegs = kProducer ? ((kLaunchRegs * kThreads - kProducerRegs * kProducerWarps * 32) /
                                           kConsumerThreads) / 8 * 8 > 240 ? 240 :
                                          ((kLaunchRegs * kThreads - kProducerRegs * kProducerWarps * 32) /
                                           kConsumerThreads) / 8 * 8
                                        : kLaunchRegs;
static_assert(!kProducer || kConsumerRegs * kConsumerThreads + kProducerRegs * kProducerWarps * 32 <=
                                kLaunchRegs * kThreads, "register split exceeds the launch total");
// (strip, row half) pairs of a strip group finished by each of its warps.
constexpr int kFinishPerWarp = kStripsPerWarp / 2;
// With the producer warpgroup, an NVFP4 ring slot is released by every lane
// of the consumer warps (empty barrier count kConsumerThreads); FP8 releases
// once per warp after a warp barrier (measured faster each way).
template <int FMT>
constexpr bool kLaneRelease = FMT == SKINNY_FMT_NVFP4;
static_assert(kStripsPerWarp == 2 || kStripsPerWarp == 4, "2 or 4 strips per warp");

// The f-th (strip, row half) pair that warp (sg, kq) finishes: strip
// kStripsPerWarp * sg + pi / 2, rows gid + 8 * (pi % 2), pi = kq * kFinishPerWarp + f.
__host__ __device__ __forceinline__ int finish_strip(int sg, int kq, int f)
{
    return kStripsPerWarp * sg + (kq * kFinishPerWarp + f) / 2;
}
__host__ __device__ __forceinline__ int finish_half(int kq, int f) { return (kq * kFinishPerWarp + f) % 2; }
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
constexpr int kMaxDevices = 64;



// Named barrier id of the consumer warps (0 is __syncthreads).
constexpr uint32_t kBarConsumers = 1;

// Bits of g_device_error: which bounded wait gave up.
constexpr unsigned kErrFullWait = 1u;      // a warp waiting for a tile
constexpr unsigned kErrEmptyWait = 2u;     // the refilling warp waiting for a slot
constexpr unsigned kErrDrainWait = 4u;     // draining copies in flight after an abort
constexpr unsigned kErrPartialWait = 8u;   // a finisher waiting for a partial sum

// What the finished outputs of a row tile turn into.  Each kind is its own
// kernel instance, so a launch carries only its own epilogue's code: the
// runtime switch between them cost the plain GEMMs 3-10%.
// The FP8 kernels, which wait on HBM, load a fused add's residual as they
// begin a row tile; the issue-bound NVFP4 kernels load it in the flush
// (each measured faster than the other way).
template <int FMT>
constexpr bool kEarlyResidual = FMT == SKINNY_FMT_FP8;

enum : int {
    kEpStore = 0,     // y = scale * acc
    kEpAdd = 1,       // y = scale * acc + residual
    kEpSiluMul = 2,   // y = silu(gate) * up (NVFP4, gate+up packing, one GEMM)
    kEpArgmax = 3,    // per-token (row, value) of the maximum (NVFP4, one GEMM)
};

__device__ unsigned int g_device_error;

// Fused argmax: this CTA's best key per token, folded into the global maxima
// once, at the end of the kernel.
__shared__ unsigned long long s_argmax_best[SKINNY_MAX_M];

// Tokens are the n = 8 columns of the m16n8k16 MMA: a launch with M <= 8
// runs one token block (NB = 1), one with 9 <= M <= 16 runs two (NB = 2),
// each decoded weight fragment feeding NB MMAs.
constexpr int kBlockTokens = 8;
static_assert(SKINNY_MAX_M == 2 * kBlockTokens, "at most two token blocks");

template <int FMT>
struct Tile;

// One ring stage holds one 128 x 512 tile, fetched by ONE bulk copy (36 KB
// NVFP4, 64 KB FP8): every cp.async.bulk costs its issuing thread on the
// order of 150 ns on B200, so copies must be large to stream HBM at full rate.
template <>
struct Tile<SKINNY_FMT_NVFP4> {
    static constexpr int kBytes = kNvfp4TileBytes;        // 32 KB codes + 4 KB scales
    static constexpr int kScalesOff = kNvfp4TileCodeBytes;
    // Three slots, like FP8: on B200 deeper NVFP4 rings streamed slower
    // (34816 x 5120: 21.7 us with 3 slots, 22.0 with 4, 22.5 with 5, 23.1 with 6).
    static constexpr int kStages = 3;
};

template <>
struct Tile<SKINNY_FMT_FP8> {
    static constexpr int kBytes = kFp8TileBytes;
    static constexpr int kScalesOff = 0;
    static constexpr int kStages = 3;
};

// Shared memory: kStages ring stages (one tile each), then the flush exchange
// buffer (two parities of kConsumerWarps x kStripsPerWarp strips x NB token
// blocks x 32 lanes x float4), then the mbarriers and the per-slot release counters, then (NVFP4)
// the buffer of the fused SiLU*mul epilogue.  With two token blocks the FP8
// ring has two slots (three do not fit next to the doubled exchange buffer).
template <int FMT, int NB>
struct Smem {
    static constexpr int kStages = (FMT == SKINNY_FMT_FP8 && NB == 2) ? 2 : Tile<FMT>::kStages;
    static constexpr int kStageBytes = Tile<FMT>::kBytes;
    static constexpr int kXchgOff = kStages * kStageBytes;
    static constexpr int kXchgFloat4 = kConsumerWarps * kStripsPerWarp * NB * 32;   // one parity
    static constexpr int kXchgBytes = 2 * kXchgFloat4 * 16;
    static constexpr int kBarOff = kXchgOff + kXchgBytes;
    static constexpr int kCountOff = kBarOff + 2 * kStages * 8;   // int released[kStages]
    // Fused SiLU*mul epilogue (NVFP4 only): a finished row tile's outputs, [128 rows][8 NB tokens] FP32.
    static constexpr int kActOff = (kCountOff + kStages * 4 + 15) / 16 * 16;
    static constexpr int kActBytes = FMT == SKINNY_FMT_NVFP4 ? kTileRows * kBlockTokens * NB * 4 : 0;
    static constexpr int kBytes = kActOff + kActBytes;
    static_assert(kStageBytes % 16 == 0, "stage alignment");
    // 227 KB per CTA; the static shared variables (fused argmax) take 128 B more.
    static_assert(kBytes <= 232448, "shared memory per CTA");
};

// One GEMM of a launch.  A launch runs one GEMM, or a group of independent
// GEMMs of the same K (and M, format and output type) whose row tiles are
// concatenated into one tile sequence: member m owns row tiles
// [g_begin, next member's g_begin).
struct Member {
    const uint16_t* x;            // [M][K] fp16 bits
    const uint8_t* codes;         // packed tiles (NVFP4 tiles carry their block scales)
    const float* channel_scale;   // FP8 per-output-channel scale [N]
    void* y;                      // [M][N]
    const void* residual;         // [M][N], y's dtype, added before the output rounding (or null; may alias y)
    float out_scale;              // NVFP4 per-tensor scale (FP8: unused, the channel scales apply)
    int N;
    int g_begin;                  // first row tile of this GEMM in the launch's tile sequence
    int u_begin;                  // its first tile (g_begin * C)
};

struct Params {
    Member mem[SKINNY_MAX_GROUP];
    int n_members;
    uint2* partials;              // [P][consumer warps][32 lanes][kFinishPerWarp * NB] encoded float pairs (split K)
    int M, K;
    int C;                        // K tiles per row tile
    int U;                        // tiles in total (G * C)
    int Q;                        // scheduling quantum: 1 (split K) or C (whole row tiles)
    int out_f32;
    // Fused SiLU*mul (instead of storing y): W packed by skinny_pack_nvfp4_gate_up,
    // y is [M][N/2] with y[m][j] = silu(gate[m][j]) * up[m][j].
    int silu_mul;
    // Fused argmax (instead of storing y): each token's largest output and its row.
    int argmax;
    unsigned long long* amax_key; // [SKINNY_MAX_M] running maxima, zero between calls
    int* amax_done;               // CTAs that have finished, zero between calls
    int* out_idx;                 // [M]
    float* out_val;               // [M]
};

// The GEMM of the launch that owns row tile g (member_of_row) or tile u
// (member_of_tile).  A launch of one GEMM (GR = false) has member 0 only,
// resolved at compile time, so its kernels carry no lookup at all.
template <bool GR>
__device__ __forceinline__ int member_of_row(const Params& p, int g)
{
    if constexpr (!GR) {
        return 0;
    } else {
        int m = p.n_members - 1;
        while (m > 0 && g < p.mem[m].g_begin) --m;
        return m;
    }
}

template <bool GR>
__device__ __forceinline__ int member_of_tile(const Params& p, int u)
{
    if constexpr (!GR) {
        return 0;
    } else {
        int m = p.n_members - 1;
        while (m > 0 && u < p.mem[m].u_begin) --m;
        return m;
    }
}

// CTA b of P takes quanta [range_start(b), range_start(b+1)) of the UQ = U/Q
// quanta: with q = UQ / P and r = UQ % P, the first r CTAs take q + 1 quanta
// and the others q.  CTAs are dispatched roughly in blockIdx order as SMs
// free up, so the CTAs that start last get the shorter ranges.  32-bit
// arithmetic only: b * q <= UQ < 2^31.
__host__ __device__ __forceinline__ int range_start(int b, int q, int r, int Q)
{
    return (b * q + (b < r ? b : r)) * Q;
}

// The CTA whose range holds tile u (inverse of range_start).
__host__ __device__ __forceinline__ int owner_of(int u, int q, int r, int Q)
{
    const int uq = u / Q, edge = r * (q + 1);
    return uq < edge ? uq / (q + 1) : r + (uq - edge) / q;
}

// This CTA's range and the contributors of the row tiles at its two ends
// (every row tile strictly inside the range is this CTA's alone).
struct Sched {
    int b;
    int u_last;       // last tile of the range (processed first)
    int n_units;
    int first_g, last_g;
    int first_owner;  // lowest contributor of row tile first_g
    int last_owner;   // highest contributor of row tile last_g
};

__host__ __device__ __forceinline__ Sched make_sched(const Params& p, int b, int P)
{
    const int UQ = p.U / p.Q;
    const int q = UQ / P, r = UQ % P;   // P <= UQ, so q >= 1
    Sched s;
    s.b = b;
    const int u_begin = range_start(b, q, r, p.Q);
    s.n_units = range_start(b + 1, q, r, p.Q) - u_begin;
    s.u_last = u_begin + s.n_units - 1;
    s.first_g = u_begin / p.C;
    s.last_g = s.u_last / p.C;
    s.first_owner = owner_of(s.first_g * p.C, q, r, p.Q);
    s.last_owner = owner_of(s.last_g * p.C + p.C - 1, q, r, p.Q);
    return s;
}

// A published partial sum never encodes to zero: NaNs are made canonical
// (0x7FC00000), so the one float pattern whose complement is zero
// (0xFFFFFFFF, a NaN) never occurs.  A zeroed slot therefore reads "empty".
__device__ __forceinline__ uint32_t encode_partial(float v)
{
    return ~(v == v ? __float_as_uint(v) : 0x7FC00000u);
}

__device__ __forceinline__ float decode_partial(uint32_t e) { return __uint_as_float(~e); }

// Argmax keys: 64 bits that order (value, row) pairs as "larger value first,
// then smaller row".  The value's bits are mapped to an unsigned integer in
// the order of the floats (NaN, made canonical, above +inf; -0 made +0); the
// row is stored complemented.  Every real key is above zero, so a zero key
// means "no candidate yet".
__device__ __forceinline__ unsigned long long argmax_key(float v, int n)
{
    if (v != v) v = __uint_as_float(0x7FC00000u);
    if (v == 0.f) v = 0.f;
    const uint32_t b = __float_as_uint(v);
    const uint32_t u = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (uint32_t)n);
}

__device__ __forceinline__ float argmax_key_value(unsigned long long key)
{
    const uint32_t u = (uint32_t)(key >> 32);
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

__device__ __forceinline__ int argmax_key_row(unsigned long long key) { return (int)(0xFFFFFFFFu - (uint32_t)key); }

// One warp's slice of a finished row tile: strip `strip`, rows gid + 8h,
// tokens tok0 + 2t and tok0 + 2t + 1 of this lane (v[0], v[1]; res[0],
// res[1] the residual of those outputs when the GEMM adds one).  Called by
// all 32 lanes.  With the fused argmax the outputs only update this lane's
// running best keys (best[0], best[1]); they are reduced across the CTA once,
// at the end of the kernel.
template <int FMT, bool GR, int EP>
__device__ __forceinline__ void epilogue(const Params& p, const float (&v)[2], const float (&res)[2], int g,
                                         int strip, int h, int lane, int tok0, unsigned long long (&best)[2])
{
    const int gid = lane >> 2, t = lane & 3;
    const Member& mb = p.mem[member_of_row<GR>(p, g)];
    const int n = (g - mb.g_begin) * kTileRows + strip * kStripRows + gid + 8 * h;
    const float sc = (FMT == SKINNY_FMT_NVFP4) ? mb.out_scale : (n < mb.N ? mb.channel_scale[n] : 0.f);
    if constexpr (EP == kEpArgmax) {
        // The value is the one the FP32-output GEMM would store.
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int m = tok0 + 2 * t + e;
            const unsigned long long key = (n < mb.N && m < p.M) ? argmax_key(v[e] * sc, n) : 0ull;
            best[e] = key > best[e] ? key : best[e];
        }
        return;
    }
    if (n >= mb.N) return;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int m = tok0 + 2 * t + e;
        if (m >= p.M) continue;
        const size_t idx = (size_t)m * mb.N + n;
        // Rounded FP32 product, never contracted with the add below, so the
        // fused add sees exactly the value the plain GEMM stores.
        float val = __fmul_rn(v[e], sc);
        // Fused residual add: one FP32 add, then the single output rounding.
        // Each element is read (early, by load_residual) and written by this
        // thread only, so the residual may be y itself.
        if constexpr (EP == kEpAdd) val = __fadd_rn(val, res[e]);
        if (p.out_f32)
            static_cast<float*>(mb.y)[idx] = val;
        else
            static_cast<__half*>(mb.y)[idx] = __float2half_rn(val);
    }
}

// Fused SiLU*mul epilogue of row tile g (all consumer warps of the CTA): rows
// 0..63 of the tile are gate rows 64g.., rows 64..127 the matching up rows,
// so the tile yields outputs j = 64g + 0..63 of every token:
// y[m][j] = silu(gate) * up, silu(z) = z / (1 + e^-z), in FP32.
template <int FMT, int NB>
__device__ void silu_mul_epilogue(const Params& p, const float (&v)[kFinishPerWarp][NB][2], int g, int sg, int kq,
                                  int lane, uint8_t* smem)
{
    constexpr int kTok = kBlockTokens * NB;
    float* act = reinterpret_cast<float*>(smem + Smem<FMT, NB>::kActOff);   // [128 rows][kTok tokens]
    const int gid = lane >> 2, t = lane & 3;
    const Member& mb = p.mem[0];   // the fused SiLU*mul runs one GEMM per launch
    ptx::named_barrier_sync(kBarConsumers, kConsumerThreads);   // earlier readers of act are done
#pragma unroll
    for (int f = 0; f < kFinishPerWarp; ++f) {
        const int r = finish_strip(sg, kq, f) * kStripRows + gid + 8 * finish_half(kq, f);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            act[r * kTok + kBlockTokens * nb + 2 * t] = v[f][nb][0] * mb.out_scale;
            act[r * kTok + kBlockTokens * nb + 2 * t + 1] = v[f][nb][1] * mb.out_scale;
        }
    }
    ptx::named_barrier_sync(kBarConsumers, kConsumerThreads);
    const int jl = threadIdx.x % 64;                     // 64 outputs x kConsumerThreads/64 tokens per pass
    const int F = mb.N / 2, j = g * 64 + jl;
#pragma unroll
    for (int pass = 0; pass < kTok / (kConsumerThreads / 64); ++pass) {
        const int m = threadIdx.x / 64 + (kConsumerThreads / 64) * pass;
        if (m < p.M && j < F) {
            const float gate = act[jl * kTok + m], up = act[(64 + jl) * kTok + m];
            const float val = gate / (1.f + expf(-gate)) * up;
            const size_t idx = (size_t)m * F + j;
            if (p.out_f32)
                static_cast<float*>(mb.y)[idx] = val;
            else
                static_cast<__half*>(mb.y)[idx] = __float2half_rn(val);
        }
    }
}

// The residual of this lane's outputs of row tile g (strip `strip`, rows
// gid + 8h, tokens 8nb + 2t + e), loaded ahead of the epilogue: by the FP8
// kernels when the CTA begins a row tile it finishes, by the NVFP4 kernels in
// the flush, before its barrier.  Zero where there is none.
template <int NB, bool GR>
__device__ __forceinline__ void load_residual(const Params& p, int g, int strip, int h, int lane,
                                              float (&res)[NB][2])
{
    const int gid = lane >> 2, t = lane & 3;
    const Member& mb = p.mem[member_of_row<GR>(p, g)];
    const int n = (g - mb.g_begin) * kTileRows + strip * kStripRows + gid + 8 * h;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int m = kBlockTokens * nb + 2 * t + e;
            res[nb][e] = 0.f;
            if (mb.residual && n < mb.N && m < p.M) {
                const size_t idx = (size_t)m * mb.N + n;
                res[nb][e] = p.out_f32 ? static_cast<const float*>(mb.residual)[idx]
                                       : __half2float(static_cast<const __half*>(mb.residual)[idx]);
            }
        }
}

// The finished outputs of row tile g (this warp's slice) go to y, to the
// fused argmax, or through the fused SiLU*mul.  Called by every warp of the
// CTA together.
template <int FMT, int NB, bool GR, int EP>
__device__ __forceinline__ void finish(const Params& p, const float (&v)[kFinishPerWarp][NB][2],
                                       const float (&res)[kFinishPerWarp][NB][2], int g, int sg, int kq, int lane,
                                       uint8_t* smem, unsigned long long (&best)[NB][2])
{
    if constexpr (EP == kEpSiluMul) {
        silu_mul_epilogue<FMT, NB>(p, v, g, sg, kq, lane, smem);
    } else {
#pragma unroll
        for (int f = 0; f < kFinishPerWarp; ++f)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                epilogue<FMT, GR, EP>(p, v[f][nb], res[f][nb], g, finish_strip(sg, kq, f), finish_half(kq, f), lane,
                                  kBlockTokens * nb, best[nb]);
    }
}

// Finish (or contribute to) row tile g, whose K range CTAs c_first..c_last
// share.  The kChunkPairs warps of a strip group (sg, kq = 0..3) hold the four
// K quarters of its strips; through shared memory each of them takes
// kFinishPerWarp (strip, row half) pairs of the group's outputs and adds the
// four K quarters in order (a fixed order).
//  * c_first == c_last: this CTA covered all of K; finish the outputs
//    (store y, or the fused argmax / SiLU*mul).
//  * this CTA is not c_last: publish the partial sums in this CTA's slot.
//  * this CTA is c_last (the finisher): wait for the slots of c_first ..
//    c_last-1, add them in CTA order and then its own sums, finish the
//    outputs, and zero the slots for the next call.
// Which case applies is the same for every warp of the CTA, so the barriers
// of the exchange and of the fused epilogues are reached by all of them.
// With two token blocks every lane carries both blocks' sums (NB pairs).
template <int FMT, int NB, bool GR, int EP>
__device__ void flush(const Params& p, const float (&acc)[kStripsPerWarp][NB][4], int g, int c_first, int c_last,
                      int parity, uint8_t* smem, int b, int warp, int lane, unsigned long long (&best)[NB][2],
                      const float (&res_early)[kFinishPerWarp][NB][2])
{
    using S = Smem<FMT, NB>;
    constexpr int F = kFinishPerWarp;
    float4* xchg = reinterpret_cast<float4*>(smem + S::kXchgOff) + parity * S::kXchgFloat4;
    const int sg = warp % kStripGroups, kq = warp / kStripGroups;
#pragma unroll
    for (int q = 0; q < kStripsPerWarp; ++q)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
            xchg[((warp * kStripsPerWarp + q) * NB + nb) * 32 + lane] =
                make_float4(acc[q][nb][0], acc[q][nb][1], acc[q][nb][2], acc[q][nb][3]);
    float res[F][NB][2];
    if constexpr (EP == kEpAdd) {
        if constexpr (kEarlyResidual<FMT>) {
#pragma unroll
            for (int f = 0; f < F; ++f)
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) res[f][nb][0] = res_early[f][nb][0], res[f][nb][1] = res_early[f][nb][1];
        } else if (c_first == c_last || b == c_last) {
#pragma unroll
            for (int f = 0; f < F; ++f)
                load_residual<NB, GR>(p, g, finish_strip(sg, kq, f), finish_half(kq, f), lane, res[f]);
        }
    }
    ptx::named_barrier_sync(kBarConsumers, kConsumerThreads);
    float tot[F][NB][2];
#pragma unroll
    for (int f = 0; f < F; ++f)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) tot[f][nb][0] = tot[f][nb][1] = 0.f;
#pragma unroll
    for (int k = 0; k < kChunkPairs; ++k)
#pragma unroll
        for (int f = 0; f < F; ++f)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int q = finish_strip(sg, kq, f) - kStripsPerWarp * sg;
                const float4 v = xchg[(((k * kStripGroups + sg) * kStripsPerWarp + q) * NB + nb) * 32 + lane];
                const bool hi = finish_half(kq, f) != 0;
                tot[f][nb][0] += hi ? v.z : v.x;
                tot[f][nb][1] += hi ? v.w : v.y;
            }
    if (c_first == c_last) {
        finish<FMT, NB, GR, EP>(p, tot, res, g, sg, kq, lane, smem, best);
        return;
    }
    constexpr int kSlot = F * NB;   // uint2 per lane
    uint2* const mine = p.partials + ((b * kConsumerWarps + warp) * 32 + lane) * kSlot;
    if (b != c_last) {
#pragma unroll
        for (int f = 0; f < F; ++f)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                ptx::st_volatile_v2(mine + f * NB + nb,
                                    make_uint2(encode_partial(tot[f][nb][0]), encode_partial(tot[f][nb][1])));
        return;
    }
    // Finisher.  The other contributors are lower-numbered CTAs; all but the
    // middle ones (whose whole range lies in g) published long ago.
    constexpr int kBatch = 8 / kSlot;
    float sum[F][NB][2];
#pragma unroll
    for (int f = 0; f < F; ++f)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) sum[f][nb][0] = sum[f][nb][1] = 0.f;
    bool timed_out = false;
    uint64_t t0 = 0;
    for (int c0 = c_first; c0 < c_last; c0 += kBatch) {
        uint2 v[kBatch][kSlot];
        auto slot = [&](int k) { return p.partials + (((c0 + k) * kConsumerWarps + warp) * 32 + lane) * kSlot; };
#pragma unroll
        for (int k = 0; k < kBatch; ++k)
#pragma unroll
            for (int e = 0; e < kSlot; ++e)
                v[k][e] = (c0 + k < c_last) ? ptx::ld_volatile_v2(slot(k) + e) : make_uint2(1u, 1u);
        for (uint32_t it = 0;; ++it) {
            bool missing = false;
#pragma unroll
            for (int k = 0; k < kBatch; ++k)
#pragma unroll
                for (int e = 0; e < kSlot; ++e) {
                    if (v[k][e].x == 0u || v[k][e].y == 0u) {
                        missing = true;
                        v[k][e] = ptx::ld_volatile_v2(slot(k) + e);
                    }
                }
            if (!missing || timed_out) break;
            if (it == 0) t0 = ptx::globaltimer_ns();
            else if ((it & 15u) == 0 && ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
                timed_out = true;
                atomicOr(&g_device_error, kErrPartialWait);
            }
        }
#pragma unroll
        for (int k = 0; k < kBatch; ++k) {
            if (c0 + k < c_last) {
#pragma unroll
                for (int f = 0; f < F; ++f)
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) {
                        sum[f][nb][0] += decode_partial(v[k][f * NB + nb].x);
                        sum[f][nb][1] += decode_partial(v[k][f * NB + nb].y);
                    }
#pragma unroll
                for (int e = 0; e < kSlot; ++e) ptx::st_volatile_v2(slot(k) + e, make_uint2(0u, 0u));
            }
        }
    }
#pragma unroll
    for (int f = 0; f < F; ++f)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            sum[f][nb][0] += tot[f][nb][0];
            sum[f][nb][1] += tot[f][nb][1];
        }
    finish<FMT, NB, GR, EP>(p, sum, res, g, sg, kq, lane, smem, best);
}

// Put tile `u` into ring slot s with one bulk copy.
template <int FMT, int NB, bool GR>
__device__ __forceinline__ void issue_stage(const Params& p, uint8_t* smem, uint64_t* full, int s, int u)
{
    const Member& mb = p.mem[member_of_tile<GR>(p, u)];
    const uint8_t* src = mb.codes + (size_t)(GR ? u - mb.u_begin : u) * Tile<FMT>::kBytes;
    ptx::mbar_arrive_expect_tx(&full[s], Tile<FMT>::kBytes);
    ptx::bulk_g2s(smem + s * Smem<FMT, NB>::kStageBytes, src, Tile<FMT>::kBytes, &full[s],
                  ptx::policy_evict_first());
}

// The B fragments of one K tile for this lane: one token (row xrow of x),
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

// Per-warp state of the consumer loop.  A warp owns strips
// kStripsPerWarp * sg .. + kStripsPerWarp - 1 and K chunks 2kq, 2kq+1 of every
// tile: 2 * kStripsPerWarp strip chunks, each with its own accumulator chain
// per token block (hiding the tensor-core latency); the two chunk
// accumulators of a strip are added in a fixed order when a row tile is
// flushed.
template <int FMT, int NB>
struct Consumer {
    static constexpr int Q = kStripsPerWarp;
    float acc[2][Q][NB][4];   // [chunk parity][strip][token block][fragment]
    uint32_t lane_codes;      // this lane's code bytes of its first strip, chunk 2kq, inside a tile
    uint32_t lane_scale;      // this lane's scale word of its first strip, chunk 2kq (NVFP4)

    __device__ __forceinline__ void zero()
    {
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int q = 0; q < Q; ++q)
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int r = 0; r < 4; ++r) acc[u][q][nb][r] = 0.f;
    }

    // The per-strip sums of both chunks (fixed order).
    __device__ __forceinline__ void total(float (&tot)[Q][NB][4]) const
    {
#pragma unroll
        for (int q = 0; q < Q; ++q)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int r = 0; r < 4; ++r) tot[q][nb][r] = acc[0][q][nb][r] + acc[1][q][nb][r];
    }

    // The warp's strip chunks of the tile at shared address `tile`;
    // bx[u][nb] holds the activations of chunk 2kq + u for token block nb.
    // All shared loads are issued first, then the decode and MMA steps of the
    // chains interleave; each decoded fragment feeds one MMA per token block.
    // NVFP4 calls `mid` half-way through the MMAs (the caller loads the next
    // tile's activations there).
    template <class Mid>
    __device__ __forceinline__ void compute(uint32_t tile, const uint32_t (&bx)[2][NB][8], Mid&& mid)
    {
        if constexpr (FMT == SKINNY_FMT_NVFP4) {
            uint4 cw[2][Q];
            uint32_t s0[2][Q], s8[2][Q];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int q = 0; q < Q; ++q)
                    cw[u][q] = ptx::lds128(tile + lane_codes + q * kNvfp4StripCodeBytes + u * 512);
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    const uint32_t sc =
                        ptx::e4m3x2_to_f16x2(ptx::lds16(tile + lane_scale + q * kNvfp4StripScaleBytes + u * 64));
                    s0[u][q] = ptx::dup_lo(sc);   // scale of row gid
                    s8[u][q] = ptx::dup_hi(sc);   // scale of row gid+8
                }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j == 2) mid();
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int q = 0; q < Q; ++q) {
                        const uint32_t w = j == 0 ? cw[u][q].x : j == 1 ? cw[u][q].y : j == 2 ? cw[u][q].z : cw[u][q].w;
                        uint32_t h[4];
                        ptx::e2m1x8_to_f16x8(w, h);
                        const uint32_t a[4] = {ptx::hmul2(h[0], s0[u][q]), ptx::hmul2(h[1], s8[u][q]),
                                               ptx::hmul2(h[2], s0[u][q]), ptx::hmul2(h[3], s8[u][q])};
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
                            ptx::mma_f16_16816(acc[u][q][nb], a, bx[u][nb][2 * j], bx[u][nb][2 * j + 1]);
                    }
            }
        } else {
            uint4 cw[2][Q][2];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int q = 0; q < Q; ++q) {
                    const uint32_t base = tile + lane_codes + q * kFp8StripBytes + u * 1024;
                    cw[u][q][0] = ptx::lds128(base);
                    cw[u][q][1] = ptx::lds128(base + 512);
                }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int q = 0; q < Q; ++q) {
                        const uint4& v = cw[u][q][j >> 1];
                        const uint32_t w0 = (j & 1) ? v.z : v.x, w1 = (j & 1) ? v.w : v.y;
                        uint32_t a[4];
                        ptx::e4m3x4_to_f16x4(w0, a[0], a[1]);
                        ptx::e4m3x4_to_f16x4(w1, a[2], a[3]);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
                            ptx::mma_f16_16816(acc[u][q][nb], a, bx[u][nb][2 * j], bx[u][nb][2 * j + 1]);
                    }
        }
    }
};

// The consumer loop of one warp over the CTA's range of tiles.  The
// activations of the next tile are fetched one tile ahead into ping-pong
// registers where the registers allow (always with the producer warpgroup's
// registers); otherwise each tile's activations are fetched as the tile
// begins (before its wait) and the next tile's lines are pulled into L1.
template <int FMT, int NB, bool GR, int EP>
__device__ void consume(const Params& p, uint8_t* smem, uint64_t* full, uint64_t* empty, const Sched& sc, int warp,
                        int lane)
{
    using S = Smem<FMT, NB>;
    constexpr int kStages = S::kStages;
    // Activations one tile ahead in ping-pong registers, where the registers allow.
    constexpr bool kAhead = NB == 1 || kConsumerRegs >= 200;
    const int gid = lane >> 2, t = lane & 3;
    const int sg = warp % kStripGroups, kq = warp / kStripGroups;
    const int n_units = sc.n_units;

    Consumer<FMT, NB> w;
    w.zero();
    const int strip0 = kStripsPerWarp * sg;
    if constexpr (FMT == SKINNY_FMT_NVFP4) {
        w.lane_codes = strip0 * kNvfp4StripCodeBytes + (2 * kq) * 512 + lane * 16;
        w.lane_scale = Tile<FMT>::kScalesOff + strip0 * kNvfp4StripScaleBytes + (2 * kq) * 64 + t * 16 + gid * 2;
    } else {
        w.lane_codes = strip0 * kFp8StripBytes + (2 * kq) * 1024 + lane * 16;
        w.lane_scale = 0;
    }
    // Activations: tokens gid + 8nb, columns c*512 + (2kq + u)*64 + [16t, 16t+16),
    // from the x of the GEMM that owns the tile.
    bool xvalid[NB];
    size_t xoff[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        xvalid[nb] = gid + kBlockTokens * nb < p.M;
        xoff[nb] = (size_t)(xvalid[nb] ? gid + kBlockTokens * nb : 0) * p.K;
    }
    const int kb_lane = 2 * kq * kChunkK + 16 * t;

    // The range is walked from its last tile down to its first.
    int cur_g = sc.last_g, parity = 0;
    int g = sc.last_g, c = sc.u_last - sc.last_g * p.C;   // tile being processed
    int nc = c;                                            // K tile whose activations are fetched next
    int ng = g;                                            // ... and its row tile
    int nm = member_of_row<GR>(p, ng);                     // ... and its GEMM
    const uint16_t* xbase = p.mem[nm].x;
    const uint32_t smem32 = ptx::smem_addr(smem);
    int* released = reinterpret_cast<int*>(smem + S::kCountOff);
    // Fused argmax: this lane's best key per token it holds (tokens 8nb + 2t + e).
    unsigned long long best[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) best[nb][0] = best[nb][1] = 0ull;
    // Contributors of a row tile: only the two at the ends of the range are shared.
    // Fused residual add (FP8): the residual of a row tile this CTA finishes
    // is loaded as the CTA begins the row tile, so the loads are long done
    // when the epilogue needs them.  NVFP4 loads it in the flush instead.
    float res[kFinishPerWarp][NB][2];
    auto load_res = [&](int rg) {
        if constexpr (EP == kEpAdd && kEarlyResidual<FMT>) {
            const int c_first = rg == sc.first_g ? sc.first_owner : sc.b;
            const int c_last = rg == sc.last_g ? sc.last_owner : sc.b;
            if (c_first == c_last || sc.b == c_last) {
                const int sg = warp % kStripGroups, kq = warp / kStripGroups;
#pragma unroll
                for (int f = 0; f < kFinishPerWarp; ++f)
                    load_residual<NB, GR>(p, rg, finish_strip(sg, kq, f), finish_half(kq, f), lane, res[f]);
            }
        }
    };
    auto flush_g = [&](int fg) {
        float tot[kStripsPerWarp][NB][4];
        w.total(tot);
        const int c_first = fg == sc.first_g ? sc.first_owner : sc.b;
        const int c_last = fg == sc.last_g ? sc.last_owner : sc.b;
        flush<FMT, NB, GR, EP>(p, tot, fg, c_first, c_last, parity, smem, sc.b, warp, lane, best, res);
        parity ^= 1;
    };
    auto fetch = [&](uint32_t (&dst)[2][NB][8]) {
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                load_b(xbase + xoff[nb], xvalid[nb], nc * kTileK + kb_lane + u * kChunkK, p.K, dst[u][nb]);
    };
    auto prefetch_l1 = [&]() {   // the lines `fetch` will read at the cursor
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int kb = nc * kTileK + kb_lane + u * kChunkK;
                if (xvalid[nb] && kb < p.K) ptx::prefetch_l1(xbase + xoff[nb] + kb);
            }
    };
    auto advance = [&]() {   // the fetch cursor moves one tile down the range
        if (nc == 0) {
            nc = p.C;
            if constexpr (GR) {
                if (--ng < p.mem[nm].g_begin && nm > 0) xbase = p.mem[--nm].x;
            }
        }
        --nc;
    };

    bool ok = true;
    int s = 0;
    uint32_t phase = 0;
    // Flush the finished row tile when tile i starts a new one.
    auto new_row_tile = [&]() {
        if (g != cur_g) {
            flush_g(cur_g);
            w.zero();
            cur_g = g;
            load_res(cur_g);
        }
    };
    // One tile: wait for its slot, flush the previous row tile if this one
    // starts a new one (here, unless the caller did before), decode and
    // multiply, release the slot.
    auto body = [&](int i, const uint32_t (&cur)[2][NB][8], auto&& mid, auto flush_here) {
        if (ok) {
            // All lanes agree on the outcome, so the warp stays converged.
            ok = __all_sync(0xffffffffu, ptx::mbar_wait(&full[s], phase, kWaitLimitNs));
            if (!ok && lane == 0) atomicOr(&g_device_error, kErrFullWait);
        }
        if constexpr (decltype(flush_here)::value) new_row_tile();
        if (ok) {
            w.compute(smem32 + s * S::kStageBytes, cur, mid);
            if (kProducer && kLaneRelease<FMT>) {
                // Every lane releases its own reads of the slot: no warp
                // barrier before the release (measured faster for NVFP4).
                ptx::mbar_arrive(&empty[s]);
            } else {
                __syncwarp();
                if (kProducer) {
                    if (lane == 0) ptx::mbar_arrive(&empty[s]);   // the producer refills the slot
                } else if (lane == 0) {
                    // Release the slot; the last of the consumer warps to do so refills it.
                    ptx::mbar_arrive(&empty[s]);
                    if (atomicAdd(&released[s], 1) == kConsumerWarps - 1) {
                        released[s] = 0;
                        if (i + kStages < n_units) {
                            if (ptx::mbar_wait(&empty[s], phase, kWaitLimitNs))
                                issue_stage<FMT, NB, GR>(p, smem, full, s, sc.u_last - (i + kStages));
                            else
                                atomicOr(&g_device_error, kErrEmptyWait);
                        }
                    }
                }
            }
        }
        if (++s == kStages) {
            s = 0;
            phase ^= 1;
        }
        if (c == 0) {
            c = p.C;
            --g;
        }
        --c;
    };

    if (n_units > 0) load_res(cur_g);
    if constexpr (kAhead) {
        uint32_t bx[2][2][NB][8];   // ping-pong: [buffer][chunk][token block][words]
        fetch(bx[0]);
        // The loop is unrolled by two so the ping-pong buffers stay in registers.
        // An MMA reads its register operands when it executes, so loading
        // into `nxt` right after the previous tile's MMAs were issued stalls
        // until they have.  NVFP4 loads half-way through this tile's MMAs
        // instead (measured faster); FP8 loads before the tile.
        // With one token block the loop runs tile pairs (three inlined copies
        // of the tile, with the flush after the wait).  The larger NVFP4
        // two-block tile is inlined twice and the flush once, before the wait:
        // instruction fetch then stalls less (measured: gate+up at M=16 28.9 ->
        // 26.9 us; slower at M <= 8 and for FP8).
        constexpr bool kOneSite = NB == 2 && FMT == SKINNY_FMT_NVFP4;
        auto step = [&](int i, uint32_t (&cur)[2][NB][8], uint32_t (&nxt)[2][NB][8]) {
            advance();
            if constexpr (FMT == SKINNY_FMT_NVFP4) {
                body(i, cur, [&] {
                    if (i + 1 < n_units) fetch(nxt);
                }, std::integral_constant<bool, !kOneSite>{});
            } else {
                if (i + 1 < n_units) fetch(nxt);   // next tile's activations, one tile ahead
                body(i, cur, [] {}, std::integral_constant<bool, !kOneSite>{});
            }
        };
        if constexpr (kOneSite) {
            for (int i = 0; i < n_units; ++i) {
                new_row_tile();
                if (i & 1)
                    step(i, bx[1], bx[0]);
                else
                    step(i, bx[0], bx[1]);
            }
        } else {
            int i = 0;
            for (; i + 1 < n_units; i += 2) {
                step(i, bx[0], bx[1]);
                step(i + 1, bx[1], bx[0]);
            }
            if (i < n_units) step(i, bx[0], bx[1]);
        }
    } else {
        // No room for a second set of activation registers: fetch each tile's
        // activations as the tile begins, and pull the next tile's lines into
        // L1 meanwhile so that fetch hits L1.
        uint32_t bx[2][NB][8];
        for (int i = 0; i < n_units; ++i) {
            fetch(bx);
            advance();
            if (i + 1 < n_units) prefetch_l1();
            body(i, bx, [] {}, std::true_type{});
        }
    }

    if (n_units > 0) flush_g(cur_g);
    if constexpr (EP == kEpArgmax) {
        // The lanes with the same t hold the same tokens for different rows:
        // reduce over them, then one shared-memory atomic per token per warp.
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                unsigned long long key = best[nb][e];
#pragma unroll
                for (int d = 4; d < 32; d <<= 1) {
                    const unsigned long long o = __shfl_xor_sync(0xffffffffu, key, d);
                    key = o > key ? o : key;
                }
                if (gid == 0 && key != 0ull) atomicMax(&s_argmax_best[kBlockTokens * nb + 2 * t + e], key);
            }
    }
    if (!ok && threadIdx.x == 0) {
        // After a wait gave up, tiles may still be landing in shared memory:
        // wait (bounded) for the last ring's worth before the CTA exits.
        for (int q = max(0, n_units - kStages); q < n_units; ++q)
            if (!ptx::mbar_wait(&full[q % kStages], (q / kStages) & 1, kWaitLimitNs))
                atomicOr(&g_device_error, kErrDrainWait);
    }
}

template <int FMT, int NB, bool GR, int EP>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ Params p)
{
    using S = Smem<FMT, NB>;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
    uint64_t* empty = full + S::kStages;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Sched sc = make_sched(p, blockIdx.x, gridDim.x);

    if (threadIdx.x < SKINNY_MAX_M) s_argmax_best[threadIdx.x] = 0ull;
    if (threadIdx.x == 0) {
        ptx::pdl_launch_dependents();
        for (int s = 0; s < S::kStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], kLaneRelease<FMT> && kProducer ? kConsumerThreads : kConsumerWarps);
            reinterpret_cast<int*>(smem + S::kCountOff)[s] = 0;
        }
        ptx::fence_mbar_init();
        // The packed weights are read-only parameters: start streaming them
        // before the previous kernel in the stream has finished.
        for (int q = 0; q < S::kStages && q < sc.n_units; ++q)
            issue_stage<FMT, NB, GR>(p, smem, full, q, sc.u_last - q);
    }
    __syncthreads();
    if constexpr (kProducer) {
        if (warp >= kConsumerWarps) {
            // The producer warpgroup: hand registers to the consumers, then
            // one thread refills each slot once every consumer warp has
            // released it (tiles kStages.. of the range; the first are in flight).
            ptx::setmaxnreg_dec<kProducerRegs>();
            if (warp == kConsumerWarps && lane == 0) {
                for (int q = S::kStages; q < sc.n_units; ++q) {
                    const int s = q % S::kStages;
                    if (!ptx::mbar_wait(&empty[s], ((q / S::kStages) - 1) & 1, kWaitLimitNs)) {
                        atomicOr(&g_device_error, kErrEmptyWait);
                        break;
                    }
                    issue_stage<FMT, NB, GR>(p, smem, full, s, sc.u_last - q);
                }
            }
            return;
        }
        ptx::setmaxnreg_inc<kConsumerRegs>();
    }
    // x, y, the channel scales and the workspace may belong to the previous
    // kernel: touch them only once it has completed.
    ptx::pdl_wait_prior_grid();

    consume<FMT, NB, GR, EP>(p, smem, full, empty, sc, warp, lane);

    if constexpr (EP == kEpArgmax) {
        // The CTA that finishes last turns the maxima into (row, value) per
        // token and leaves the keys and the counter at zero for the next call.
        // (Barriers among the consumer warps only.)
        __shared__ int last_cta;
        ptx::named_barrier_sync(kBarConsumers, kConsumerThreads);   // every warp's shared-memory maxima are in
        if (threadIdx.x < p.M && s_argmax_best[threadIdx.x] != 0ull)
            atomicMax(&p.amax_key[threadIdx.x], s_argmax_best[threadIdx.x]);
        ptx::named_barrier_sync(kBarConsumers, kConsumerThreads);   // this CTA's global atomics are issued
        if (threadIdx.x == 0)
            last_cta = ptx::atomic_add_acq_rel_gpu(p.amax_done, 1) == (int)gridDim.x - 1;
        ptx::named_barrier_sync(kBarConsumers, kConsumerThreads);
        if (last_cta && threadIdx.x < p.M) {
            const unsigned long long key = ptx::ld_volatile_u64(&p.amax_key[threadIdx.x]);
            p.out_idx[threadIdx.x] = argmax_key_row(key);
            p.out_val[threadIdx.x] = argmax_key_value(key);
            p.amax_key[threadIdx.x] = 0ull;
        }
        if (last_cta && threadIdx.x == 0) *p.amax_done = 0;
    }
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

// Raise one kernel's dynamic shared-memory limit to what it uses; true on
// failure.  With a producer warpgroup, the kernel must also be launched with
// exactly the registers per thread that its warpgroups re-balance (the
// consumers' setmaxnreg.inc would otherwise wait for registers that never
// come): a build that does not match is refused here, before any launch.
template <int FMT, int NB, bool GR, int EP>
static bool set_smem()
{
    if (kProducer) {
        cudaFuncAttributes fa{};
        if (cudaFuncGetAttributes(&fa, gemm_kernel<FMT, NB, GR, EP>) != cudaSuccess || fa.numRegs != kLaunchRegs)
            return true;
    }
    return cudaFuncSetAttribute(gemm_kernel<FMT, NB, GR, EP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Smem<FMT, NB>::kBytes) != cudaSuccess;
}

// Every instance a launch of this format and token-block count can pick.
template <int FMT, int NB>
static bool set_smem_nb()
{
    if (set_smem<FMT, NB, false, kEpStore>() || set_smem<FMT, NB, false, kEpAdd>()) return true;
    if constexpr (FMT == SKINNY_FMT_NVFP4)
        return set_smem<FMT, NB, false, kEpSiluMul>() || set_smem<FMT, NB, false, kEpArgmax>() ||
               set_smem<FMT, NB, true, kEpStore>();
    return false;
}

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
        if (set_smem_nb<SKINNY_FMT_NVFP4, 1>() || set_smem_nb<SKINNY_FMT_NVFP4, 2>() ||
            set_smem_nb<SKINNY_FMT_FP8, 1>() || set_smem_nb<SKINNY_FMT_FP8, 2>())
            return SKINNY_ERR_CUDA;
        d.sms = n;
        d.ready = true;
    }
    *sms = d.sms;
    return SKINNY_OK;
}

// Workspace layout (identical for every shape and M on a device, so one
// workspace can serve calls of different shapes in turn): one partial-sum slot
// of 8 consumer warps x 32 lanes x kFinishPerWarp pairs x 2 token blocks x 2
// floats (8 KB) per CTA, for up to
// one CTA per SM, then the fused argmax's running maxima (one 64-bit key per
// token) and CTA counter.
constexpr size_t kArgmaxTailBytes = 256;
struct Plan {
    int G, C, U, P;
    size_t partial_bytes, workspace_bytes;
};

static int64_t row_tiles(int64_t N) { return (N + kTileRows - 1) / kTileRows; }

// G row tiles (all GEMMs of the launch together) of K columns each.
static int make_plan(int64_t G, int64_t K, int sms, bool split, Plan* pl)
{
    const int64_t C = (K + kTileK - 1) / kTileK;
    if (G <= 0 || G * C >= (int64_t(1) << 31)) return SKINNY_ERR_UNSUPPORTED;
    pl->G = (int)G;
    pl->C = (int)C;
    pl->U = (int)(G * C);
    const int UQ = split ? pl->U : pl->G;
    pl->P = UQ < sms ? UQ : sms;
    pl->partial_bytes = (size_t)sms * kConsumerWarps * 32 * kFinishPerWarp * 2 * sizeof(uint2);
    pl->workspace_bytes = pl->partial_bytes + kArgmaxTailBytes;
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

// A launch of one GEMM: member 0 only.
static Params single(const void* x, int M, int64_t K, const void* w_packed, const float* channel_scale,
                     float out_scale, int64_t N, void* y, const void* residual, int out_dtype)
{
    Params p{};
    p.n_members = 1;
    Member& mb = p.mem[0];
    mb.x = static_cast<const uint16_t*>(x);
    mb.codes = static_cast<const uint8_t*>(w_packed);
    mb.channel_scale = channel_scale;
    mb.y = y;
    mb.residual = residual;
    mb.out_scale = out_scale;
    mb.N = (int)N;
    mb.g_begin = 0;
    p.M = M;
    p.K = (int)K;
    p.out_f32 = out_dtype == SKINNY_OUT_F32;
    return p;
}

// The kernel instance for NB token blocks and epilogue kind ep (grouped
// launches store their outputs).
template <int FMT, int NB>
static cudaError_t launch_instance(const cudaLaunchConfig_t& cfg, const Params& p, int ep)
{
    if constexpr (FMT == SKINNY_FMT_NVFP4) {
        if (p.n_members > 1) return cudaLaunchKernelEx(&cfg, gemm_kernel<FMT, NB, true, kEpStore>, p);
        if (ep == kEpSiluMul) return cudaLaunchKernelEx(&cfg, gemm_kernel<FMT, NB, false, kEpSiluMul>, p);
        if (ep == kEpArgmax) return cudaLaunchKernelEx(&cfg, gemm_kernel<FMT, NB, false, kEpArgmax>, p);
    }
    if (ep == kEpAdd) return cudaLaunchKernelEx(&cfg, gemm_kernel<FMT, NB, false, kEpAdd>, p);
    return cudaLaunchKernelEx(&cfg, gemm_kernel<FMT, NB, false, kEpStore>, p);
}

// Launch the GEMM(s) of p, whose members' row tiles add up to G.
template <int FMT>
static int launch(Params p, int64_t G, int64_t K, void* workspace, size_t workspace_bytes, cudaStream_t stream)
{
    int sms = 0;
    int rc = current_device(&sms);
    if (rc != SKINNY_OK) return rc;
    const bool split = workspace != nullptr;
    Plan pl;
    rc = make_plan(G, K, sms, split, &pl);
    if (rc != SKINNY_OK) return rc;
    if (split && workspace_bytes < pl.workspace_bytes) return SKINNY_ERR_WORKSPACE;
    p.C = pl.C;
    p.U = pl.U;
    p.Q = split ? 1 : pl.C;
    p.partials = split ? static_cast<uint2*>(workspace) : nullptr;
    if (p.argmax) {
        if (!split) return SKINNY_ERR_WORKSPACE;
        uint8_t* tail = static_cast<uint8_t*>(workspace) + pl.partial_bytes;
        p.amax_key = reinterpret_cast<unsigned long long*>(tail);
        p.amax_done = reinterpret_cast<int*>(tail + SKINNY_MAX_M * sizeof(unsigned long long));
    }
    // Programmatic dependent launch: the kernel may start (and prefetch its
    // weights) while the previous kernel in the stream is finishing.
    const bool two_blocks = p.M > kBlockTokens;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = two_blocks ? Smem<FMT, 2>::kBytes : Smem<FMT, 1>::kBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (FMT != SKINNY_FMT_NVFP4 && (p.n_members != 1 || p.argmax || p.silu_mul)) return SKINNY_ERR_UNSUPPORTED;
    if (p.n_members > 1 && (p.argmax || p.silu_mul)) return SKINNY_ERR_UNSUPPORTED;
    const int ep = p.argmax ? kEpArgmax : p.silu_mul ? kEpSiluMul : p.mem[0].residual ? kEpAdd : kEpStore;
    const cudaError_t e = two_blocks ? launch_instance<FMT, 2>(cfg, p, ep) : launch_instance<FMT, 1>(cfg, p, ep);
    if (e != cudaSuccess) return SKINNY_ERR_CUDA;
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

extern "C" int skinny_version(void) { return 101; }

extern "C" int skinny_workspace_bytes(int fmt, int M, int64_t N, int64_t K, size_t* bytes)
{
    if (!bytes || (fmt != SKINNY_FMT_NVFP4 && fmt != SKINNY_FMT_FP8)) return SKINNY_ERR_INVALID_ARG;
    if (K <= 0 || K % 16 != 0 || N <= 0) return SKINNY_ERR_INVALID_ARG;
    if (M < 1 || M > SKINNY_MAX_M) return SKINNY_ERR_UNSUPPORTED;
    int sms = 0;
    int rc = current_device(&sms);
    if (rc != SKINNY_OK) return rc;
    Plan pl;
    rc = make_plan(row_tiles(N), K, sms, true, &pl);
    if (rc != SKINNY_OK) return rc;
    *bytes = pl.workspace_bytes;
    return SKINNY_OK;
}

// The stream-K schedule the kernels compute, evaluated on the host for
// tests: for each CTA b, out[6b..6b+5] = (u_last, n_units, first_g, last_g,
// first_owner, last_owner).  *ctas receives the grid size.
extern "C" int skinny_debug_schedule(int64_t N, int64_t K, int sms, int split, int* out, int cap, int* ctas)
{
    if (!out || !ctas || sms <= 0 || N <= 0 || K <= 0 || K % 16 != 0) return SKINNY_ERR_INVALID_ARG;
    Plan pl;
    const int rc = make_plan(row_tiles(N), K, sms, split != 0, &pl);
    if (rc != SKINNY_OK) return rc;
    *ctas = pl.P;
    if (pl.P > cap) return SKINNY_ERR_WORKSPACE;
    Params p{};
    p.C = pl.C;
    p.U = pl.U;
    p.Q = split ? 1 : pl.C;
    for (int b = 0; b < pl.P; ++b) {
        const Sched sc = make_sched(p, b, pl.P);
        int* o = out + 6 * b;
        o[0] = sc.u_last;
        o[1] = sc.n_units;
        o[2] = sc.first_g;
        o[3] = sc.last_g;
        o[4] = sc.first_owner;
        o[5] = sc.last_owner;
    }
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
    const Params p = single(x, M, K, w_packed, nullptr, global_scale, N, y, nullptr, out_dtype);
    return launch<SKINNY_FMT_NVFP4>(p, row_tiles(N), K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int skinny_fp8_gemm(const void* x, int M, int64_t K, const void* w_packed, const float* channel_scale,
                               int64_t N, void* y, int out_dtype, void* workspace, size_t workspace_bytes,
                               void* stream)
{
    int rc = check_common(x, M, K, N, y, out_dtype, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed || !channel_scale) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16) || !aligned(channel_scale, 4)) return SKINNY_ERR_ALIGNMENT;
    const Params p = single(x, M, K, w_packed, channel_scale, 1.0f, N, y, nullptr, out_dtype);
    return launch<SKINNY_FMT_FP8>(p, row_tiles(N), K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int skinny_nvfp4_gemm_add(const void* x, int M, int64_t K, const void* w_packed, float global_scale,
                                     int64_t N, const void* residual, void* y, int out_dtype, void* workspace,
                                     size_t workspace_bytes, void* stream)
{
    if (!residual) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(residual, 4)) return SKINNY_ERR_ALIGNMENT;
    int rc = check_common(x, M, K, N, y, out_dtype, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16)) return SKINNY_ERR_ALIGNMENT;
    const Params p = single(x, M, K, w_packed, nullptr, global_scale, N, y, residual, out_dtype);
    return launch<SKINNY_FMT_NVFP4>(p, row_tiles(N), K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int skinny_fp8_gemm_add(const void* x, int M, int64_t K, const void* w_packed, const float* channel_scale,
                                   int64_t N, const void* residual, void* y, int out_dtype, void* workspace,
                                   size_t workspace_bytes, void* stream)
{
    if (!residual) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(residual, 4)) return SKINNY_ERR_ALIGNMENT;
    int rc = check_common(x, M, K, N, y, out_dtype, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed || !channel_scale) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16) || !aligned(channel_scale, 4)) return SKINNY_ERR_ALIGNMENT;
    const Params p = single(x, M, K, w_packed, channel_scale, 1.0f, N, y, residual, out_dtype);
    return launch<SKINNY_FMT_FP8>(p, row_tiles(N), K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int skinny_nvfp4_gemm_silu_mul(const void* x, int M, int64_t K, const void* w_packed, float global_scale,
                                          int64_t F, void* y, int out_dtype, void* workspace, size_t workspace_bytes,
                                          void* stream)
{
    if (F <= 0 || F % 64 != 0) return SKINNY_ERR_INVALID_ARG;
    int rc = check_common(x, M, K, 2 * F, y, out_dtype, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16)) return SKINNY_ERR_ALIGNMENT;
    Params p = single(x, M, K, w_packed, nullptr, global_scale, 2 * F, y, nullptr, out_dtype);
    p.silu_mul = 1;
    return launch<SKINNY_FMT_NVFP4>(p, row_tiles(2 * F), K, workspace, workspace_bytes,
                                    static_cast<cudaStream_t>(stream));
}

extern "C" int skinny_nvfp4_gemm_argmax(const void* x, int M, int64_t K, const void* w_packed, float global_scale,
                                        int64_t N, int32_t* argmax_idx, float* argmax_val, void* workspace,
                                        size_t workspace_bytes, void* stream)
{
    int rc = check_common(x, M, K, N, argmax_val, SKINNY_OUT_F32, workspace);
    if (rc != SKINNY_OK) return rc;
    if (!w_packed || !argmax_idx) return SKINNY_ERR_INVALID_ARG;
    if (!aligned(w_packed, 16) || !aligned(argmax_idx, 4)) return SKINNY_ERR_ALIGNMENT;
    if (!workspace) return SKINNY_ERR_WORKSPACE;
    Params p = single(x, M, K, w_packed, nullptr, global_scale, N, nullptr, nullptr, SKINNY_OUT_F32);
    p.argmax = 1;
    p.out_idx = argmax_idx;
    p.out_val = argmax_val;
    return launch<SKINNY_FMT_NVFP4>(p, row_tiles(N), K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int skinny_nvfp4_gemm_grouped(const skinny_nvfp4_group_member* members, int count, int M, int64_t K,
                                         int out_dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!members || count < 1) return SKINNY_ERR_INVALID_ARG;
    if (count > SKINNY_MAX_GROUP) return SKINNY_ERR_UNSUPPORTED;
    Params p{};
    int64_t G = 0;
    for (int m = 0; m < count; ++m) {
        const skinny_nvfp4_group_member& in = members[m];
        const int rc = check_common(in.x, M, K, in.N, in.y, out_dtype, workspace);
        if (rc != SKINNY_OK) return rc;
        if (!in.w_packed) return SKINNY_ERR_INVALID_ARG;
        if (!aligned(in.w_packed, 16)) return SKINNY_ERR_ALIGNMENT;
        Member& mb = p.mem[m];
        mb.x = static_cast<const uint16_t*>(in.x);
        mb.codes = static_cast<const uint8_t*>(in.w_packed);
        mb.y = in.y;
        mb.out_scale = in.global_scale;
        mb.N = (int)in.N;
        mb.g_begin = (int)G;
        G += row_tiles(in.N);
        if (G >= (int64_t(1) << 30)) return SKINNY_ERR_UNSUPPORTED;
    }
    p.n_members = count;
    p.M = M;
    p.K = (int)K;
    p.out_f32 = out_dtype == SKINNY_OUT_F32;
    const int C = (int)((K + kTileK - 1) / kTileK);
    for (int m = 0; m < count; ++m) p.mem[m].u_begin = p.mem[m].g_begin * C;   // < 2^31: checked by make_plan
    return launch<SKINNY_FMT_NVFP4>(p, G, K, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
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
    rc = make_plan(row_tiles(N), K, sms, true, &pl);
    if (rc != SKINNY_OK) return rc;
    if (pl.workspace_bytes > kStaticWorkspaceBytes) return SKINNY_ERR_UNSUPPORTED;
    void* ws = nullptr;
    rc = static_workspace_address(&ws);
    if (rc != SKINNY_OK) return rc;
    // A completed call leaves every partial-sum slot zero, but one whose
    // device-side wait gave up may not: clear the slots this call uses, on
    // the call's stream, so every call starts from the same state.
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, pl.workspace_bytes, st) != cudaSuccess) return SKINNY_ERR_CUDA;
    return skinny_nvfp4_gemm(x, M, K, w_packed, global_scale, N, y, out_dtype, ws, kStaticWorkspaceBytes, stream);
}

// Test hook: the device address of the static scratch array on the current
// device (the same lookup skinny_nvfp4_gemm_static_ws makes).
extern "C" int skinny_debug_static_workspace_address(void** addr)
{
    if (!addr) return SKINNY_ERR_INVALID_ARG;
    return static_workspace_address(addr);
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
