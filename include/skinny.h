/*
 * skinny.h -- C ABI of the B200 weight-only skinny GEMM library (libskinny.so).
 *
 *   y[M,N] = x[M,K] . W^T,   M = 1..16 rows, W kept compressed in HBM.
 *
 * The operation.  During single-request decode (one token, or a k=7
 * speculative-verify round plus its base token: 8 rows), a language model's
 * linear layers read far more weight bytes than anything else.  The
 * v100-skinny pages describe kernels that keep those weights compressed when
 * they are read from HBM and turn them into FP16 in registers, in small
 * pieces, against FP16 activations -- "QPN2" for NVFP4 regions of the
 * checkpoint and "QPN8" for FP8 regions, with the 8-row verify round as the
 * M=8 case (taozi.news article on v100-skinny, sections "自研 QPN 内核" and
 * "v1.1 的关键改进"; aiwitness.kr post, section "내가 실제로 만든 것").  This
 * library is a from-scratch sm_100a implementation of that operation:
 *
 *   NVFP4:  W[n][k] = e2m1(code[n][k]) * ue4m3(scale[n][k/16]) * global_scale
 *   FP8:    W[n][k] = e4m3(q[n][k]) * channel_scale[n]
 *   y[m][n] = sum_k W[n][k] * x[m][k]     (x FP16, FP32 accumulation)
 *
 * E2M1 / E4M3 are the OCP microscaling / OFP8 encodings; NVFP4 groups 16
 * consecutive K elements under one unsigned E4M3 (UE4M3) scale and adds one
 * FP32 per-tensor scale.  The dequantised weight matrix never exists in
 * memory: no N x K FP16 copy is ever made.
 *
 * Conventions for every function below:
 *   - Return value: SKINNY_OK (0) or a negative skinny_status.  Nothing
 *     aborts or prints; skinny_status_string() names a status.
 *   - Ownership: the caller owns every buffer.  The library allocates no
 *     device memory and keeps no per-call state; it caches the SM count and
 *     kernel attributes per device.
 *   - "host" pointers are ordinary CPU memory; "device" pointers are global
 *     memory of the current CUDA device.
 *   - Layouts are row-major and contiguous: x is [M][K] (leading dim K),
 *     y is [M][N] (leading dim N), W is [N][K] (the nn.Linear convention).
 *   - GEMM calls are asynchronous on `stream` (a cudaStream_t, 0 = legacy
 *     default stream).  Their status covers the argument checks and the
 *     launch only; a fault inside a kernel appears on the stream as usual and
 *     a device-side wait that gave up is reported by skinny_device_error().
 *   - GEMM kernels are launched with programmatic dependent launch: one may
 *     begin while the previous kernel in the stream is still running, and
 *     starts reading the packed weights (and nothing else) before that
 *     kernel completes.  The packed weights must therefore not be written by
 *     the kernel launched just before the GEMM on the same stream; x, y, the
 *     FP8 channel scales and the workspace are touched only after it
 *     completes.  (Weights are model parameters: packed once, then read.)
 */
#ifndef SKINNY_H
#define SKINNY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SKINNY_OK = 0,
    SKINNY_ERR_INVALID_ARG = -1,  /* null pointer, K % 16 != 0, N or K <= 0, bad dtype, bad scale byte */
    SKINNY_ERR_UNSUPPORTED = -2,  /* M outside [1, 16], or a size past the library's limits */
    SKINNY_ERR_ALIGNMENT = -3,    /* a device pointer is not aligned as documented */
    SKINNY_ERR_CUDA = -4,         /* a CUDA runtime call failed (launch, attribute, device query) */
    SKINNY_ERR_WORKSPACE = -5     /* workspace non-null but smaller than skinny_workspace_bytes() */
} skinny_status;

typedef enum { SKINNY_OUT_F16 = 0, SKINNY_OUT_F32 = 1 } skinny_out_dtype;

typedef enum { SKINNY_FMT_NVFP4 = 0, SKINNY_FMT_FP8 = 1 } skinny_format;

#define SKINNY_MAX_M 16

/* Most GEMMs one skinny_nvfp4_gemm_grouped call can run. */
#define SKINNY_MAX_GROUP 8

/* Name of a skinny_status value ("SKINNY_OK", ...); never NULL. */
const char* skinny_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int skinny_version(void);

/* ------------------------------------------------------------------------
 * Host-side layout routines (pure CPU, no CUDA call).
 *
 * The kernels read W in a private tiled order: tiles of 128 output rows x
 * 512 columns, consecutive in memory along K then N, so that a run of tiles is
 * one contiguous bulk copy and each lane of a warp finds its tensor-core
 * operand bytes in one 16-byte word (NVFP4) or two (FP8), read without
 * shared-memory bank conflicts.  An NVFP4 tile carries its UE4M3 block
 * scales (32 KB codes + 4 KB scales); an FP8 tile is 64 KB.  Rows are padded
 * to a multiple of 128 and K to a multiple of 512 with zero codes and zero
 * scales, which contribute nothing.  The caller packs once per weight and
 * copies the result to the device.
 * ---------------------------------------------------------------------- */

/* Bytes of the packed NVFP4 buffer (codes and block scales) for an N x K
 * weight.  Returns 0 if N <= 0, K <= 0 or K % 16 != 0. */
size_t skinny_nvfp4_packed_bytes(int64_t N, int64_t K);

/* Pack a logical NVFP4 tensor.
 *   codes      host [N][K/2] bytes; element k of row n is in byte k/2, the low
 *              nibble holding even k and the high nibble odd k (E2M1 codes).
 *   scales     host [N][K/16] UE4M3 bytes, one per 16 consecutive k.
 *   w_packed   host, skinny_nvfp4_packed_bytes() bytes, written fully.
 * Errors: SKINNY_ERR_INVALID_ARG for null pointers, bad sizes, or a scale
 * byte that is not a finite non-negative UE4M3 value (sign bit set, or the
 * NaN pattern 0x7F).  Nothing is written on error. */
int skinny_pack_nvfp4(const uint8_t* codes, const uint8_t* scales, int64_t N, int64_t K, void* w_packed);

/* Inverse of skinny_pack_nvfp4 (host only; for tests and tooling). */
int skinny_unpack_nvfp4(const void* w_packed, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales);

/* Bytes of the packed FP8 buffer for an N x K weight; 0 if N <= 0, K <= 0 or
 * K % 16 != 0. */
size_t skinny_fp8_packed_bytes(int64_t N, int64_t K);

/* Pack a logical FP8 tensor: q host [N][K] E4M3 bytes -> w_packed host.
 * SKINNY_ERR_INVALID_ARG for null pointers, bad sizes, or a NaN code
 * (0x7F / 0xFF).  The per-channel scales are not packed: they are passed to
 * skinny_fp8_gemm as a plain float[N] device array. */
int skinny_pack_fp8(const uint8_t* q, int64_t N, int64_t K, void* w_packed);

/* Inverse of skinny_pack_fp8 (host only). */
int skinny_unpack_fp8(const void* w_packed, int64_t N, int64_t K, uint8_t* q);

/* ------------------------------------------------------------------------
 * Device GEMMs.
 * ---------------------------------------------------------------------- */

/* Size of the optional split-K workspace for one GEMM of this format and
 * shape on the CURRENT device (it depends on the SM count only: 8 KB per SM
 * plus 256 bytes for the fused argmax's running maxima).
 * A workspace lets the kernel split K across CTAs so that every SM streams
 * the same number of weight bytes (a short-N shape such as 5120 x 5120 has
 * too few 128-row tiles to fill 148 SMs otherwise).  It holds one slot of
 * FP32 partial sums per CTA.  It must be ZERO-filled before its first use,
 * and every call that completes without a device error leaves it zero again,
 * so zero-fill it once (cudaMemset) and reuse it; after a call that set
 * skinny_device_error(), zero-fill it again.  Its layout is the same for
 * every shape on a device, so one workspace serves calls of any shape in
 * turn; it must not be shared by calls that can run at the same time.
 * Residency: with a workspace, the CTA that finishes a row tile waits
 * (bounded, 1 s) for the partial sums of lower-numbered CTAs of the same
 * grid.  The grid has at most one CTA per SM and the wait ends as soon as
 * those CTAs have run, so it assumes that they can run: the whole GPU, or
 * CTAs dispatched in increasing order.  Where the GPU is shared so that only
 * part of the grid can be resident (an MPS client limited to fewer SMs than
 * the device has, say), pass no workspace: the whole-tile schedule has no
 * wait between CTAs.
 * Returns SKINNY_OK and *bytes, or SKINNY_ERR_INVALID_ARG / _UNSUPPORTED /
 * _CUDA. */
int skinny_workspace_bytes(int fmt, int M, int64_t N, int64_t K, size_t* bytes);

/* NVFP4 weight-only GEMM: y = x . W^T with W from skinny_pack_nvfp4.
 * This is the "QPN2" operation of the v100-skinny pages (taozi.news article,
 * section "自研 QPN 内核": NVFP4 weights stay 4-bit on their way out of HBM
 * and become FP16 in registers, against FP16 activations; M=1 is one decode
 * token and M=8 the k=7 verify round; aiwitness.kr post, section
 * "내가 실제로 만든 것").
 *   x            device [M][K] FP16, 16-byte aligned, read-only during the call.
 *   M            1..16 (rows of x: the tokens of one decode step or verify
 *                round: 1, or a base token plus k drafts; 9..16 covers a
 *                deeper draft or two requests' verify rounds).
 *   K            multiple of 16.
 *   w_packed     device, from skinny_pack_nvfp4 (codes and block scales), 16-byte aligned.
 *   global_scale FP32 per-tensor scale, applied to the FP32 sum.
 *   N            output features.
 *   y            device [M][N], FP16 (RNE) or FP32 per out_dtype, 4-byte aligned.
 *   workspace    device or NULL; if non-NULL, at least
 *                skinny_workspace_bytes(SKINNY_FMT_NVFP4, M, N, K) bytes,
 *                16-byte aligned, zero-filled (see above).  NULL selects
 *                whole-tile scheduling (no split-K, nothing written besides y).
 *   stream       cudaStream_t.
 * Rounding: products of decoded weights and x are exact; only the FP32
 * summation order differs from exact arithmetic, and it is fixed, so results
 * are bitwise reproducible run to run for a given shape and device.
 * Errors: see skinny_status. */
int skinny_nvfp4_gemm(const void* x, int M, int64_t K, const void* w_packed, float global_scale, int64_t N,
                      void* y, int out_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* FP8 (E4M3) weight-only GEMM with a per-output-channel FP32 scale.
 * This is the "QPN8" operation that serves the checkpoint's FP8 regions
 * (taozi.news article, section "v1.1 的关键改进": FP4 regions stay FP4 and
 * FP8 regions stay FP8, with FP16 activations; its M=1..4 bandwidth is quoted
 * in section "自研 QPN 内核").
 *   w_packed       device, from skinny_pack_fp8, 16-byte aligned.
 *   channel_scale  device float[N], 4-byte aligned.
 * Other arguments as skinny_nvfp4_gemm (workspace sized with SKINNY_FMT_FP8). */
int skinny_fp8_gemm(const void* x, int M, int64_t K, const void* w_packed,
                    const float* channel_scale, int64_t N, void* y, int out_dtype,
                    void* workspace, size_t workspace_bytes, void* stream);

/* GEMM fused with a residual add, for the projections whose output joins
 * the residual stream (the attention output projection and the MLP down
 * projection of a decoder layer):
 *   y[m][n] = (scale * sum_k w[n][k] x[m][k]) + residual[m][n]
 * with the sum and the add in FP32 and one rounding to the output type.
 *   residual  device [M][N] of the OUTPUT type (FP16 or FP32 per out_dtype),
 *             4-byte aligned; it may be y itself (in-place update of the
 *             residual stream).
 * Other arguments and errors as skinny_nvfp4_gemm / skinny_fp8_gemm; a null
 * residual is INVALID_ARG. */
int skinny_nvfp4_gemm_add(const void* x, int M, int64_t K, const void* w_packed, float global_scale, int64_t N,
                          const void* residual, void* y, int out_dtype, void* workspace, size_t workspace_bytes,
                          void* stream);
int skinny_fp8_gemm_add(const void* x, int M, int64_t K, const void* w_packed, const float* channel_scale, int64_t N,
                        const void* residual, void* y, int out_dtype, void* workspace, size_t workspace_bytes,
                        void* stream);

/* Gate+up weights for the fused SiLU*mul GEMM: logical codes [2F][K/2] and
 * scales [2F][K/16] (rows 0..F-1 = gate, F..2F-1 = up, encodings as in
 * skinny_pack_nvfp4) are packed so that every 128-row tile holds 64 gate rows
 * and the 64 up rows of the same outputs.  F must be a multiple of 64.
 * w_packed: host, skinny_nvfp4_packed_bytes(2F, K) bytes.  Pure CPU.
 * Errors: INVALID_ARG (null pointer, F % 64 != 0, bad shape, bad scale byte). */
int skinny_pack_nvfp4_gate_up(const uint8_t* codes, const uint8_t* scales, int64_t F, int64_t K, void* w_packed);

/* NVFP4 gate+up GEMM fused with the SiLU*mul activation of a gated MLP
 * (the 34816-wide gate+up projection of the pages' model feeding its
 * 17408-wide down projection):
 *   y[m][j] = silu(g[m][j]) * u[m][j],  silu(z) = z / (1 + e^-z),
 * where g = x . Wgate^T and u = x . Wup^T are the two halves of the GEMM
 * (FP32 sums, times global_scale), evaluated in FP32 with expf and rounded
 * once to the output type.  No M x 2F intermediate is written.
 *   w_packed  from skinny_pack_nvfp4_gate_up (F output columns, 2F weight rows).
 *   F         outputs per token, a multiple of 64.
 *   y         device [M][F], FP16 or FP32 per out_dtype, 4-byte aligned.
 *   workspace optional, sized with skinny_workspace_bytes(SKINNY_FMT_NVFP4, M, 2F, K).
 * Other arguments and errors as skinny_nvfp4_gemm; F % 64 != 0 is INVALID_ARG. */
int skinny_nvfp4_gemm_silu_mul(const void* x, int M, int64_t K, const void* w_packed, float global_scale, int64_t F,
                               void* y, int out_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* NVFP4 GEMM fused with a per-token argmax over the N outputs: the greedy
 * pick of an lm_head (vocabulary projection), or the local argmax of a
 * speculative-verify round, without writing the M x N logits.  (Taozi.news
 * article, section "自研 QPN 内核", and the aiwitness.kr post, section
 * "내가 실제로 만든 것": the drafter and the verify round take the greedy /
 * local argmax of the vocabulary projection.)
 *   argmax_idx   device int32[M]: for token m, the row n with the largest
 *                y[m][n]; ties go to the smallest n, a NaN output counts as
 *                larger than any number (as torch.argmax), -0.0 equals +0.0.
 *   argmax_val   device float[M]: that y[m][n], bitwise the value the FP32
 *                output of skinny_nvfp4_gemm would hold with the same
 *                workspace size (same schedule and summation order).
 *   workspace    REQUIRED (the running maxima live in its tail); sized and
 *                zero-filled as for skinny_nvfp4_gemm, and left zero again.
 * Other arguments as skinny_nvfp4_gemm.  A NULL workspace returns
 * SKINNY_ERR_WORKSPACE; null or unaligned outputs return INVALID_ARG /
 * ALIGNMENT.  The outputs are written by one CTA at the end of the kernel. */
int skinny_nvfp4_gemm_argmax(const void* x, int M, int64_t K, const void* w_packed, float global_scale, int64_t N,
                             int32_t* argmax_idx, float* argmax_val, void* workspace, size_t workspace_bytes,
                             void* stream);

/* One GEMM of a grouped launch (see skinny_nvfp4_gemm_grouped).  Plain
 * pointers; the struct is read on the host during the call. */
typedef struct {
    const void* x;         /* device [M][K] FP16, 16-byte aligned */
    const void* w_packed;  /* device, from skinny_pack_nvfp4 with this N and the call's K, 16-byte aligned */
    float global_scale;    /* FP32 per-tensor scale */
    int64_t N;             /* output features of this GEMM */
    void* y;               /* device [M][N], FP16 or FP32 per the call's out_dtype, 4-byte aligned */
} skinny_nvfp4_group_member;

/* Several independent NVFP4 GEMMs of the same K, M and output type in ONE
 * launch: y_i = x_i . W_i^T for i < count.  The attention projections of a
 * decoder layer (the 5120-wide q, k/v and o shapes the v100-skinny pages
 * measure: taozi.news article, section "自研 QPN 内核") each stream only
 * ~15 MB, too little to amortise a launch's ramp-up and tail on their own;
 * their row tiles are concatenated into one tile sequence that the stream-K
 * schedule spreads over all SMs, so the fixed cost is paid once.  Members
 * may share x (q, k and v read the same activations) but their y must not
 * overlap each other or any x.  Each y_i is exactly what skinny_nvfp4_gemm
 * computes for member i up to FP32 summation order (the split points of K
 * differ); the order is fixed for a given member list, so results are
 * bitwise reproducible.
 *   members    host array of `count` entries.
 *   count      1..SKINNY_MAX_GROUP (more: UNSUPPORTED; 0 or null: INVALID_ARG).
 *   workspace  optional, as for skinny_nvfp4_gemm (same size: it depends on
 *              the device only).
 * Errors: per member as skinny_nvfp4_gemm. */
int skinny_nvfp4_gemm_grouped(const skinny_nvfp4_group_member* members, int count, int M, int64_t K,
                              int out_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* NVFP4 GEMM for callers that cannot allocate device memory.
 *
 * There is no counterpart of this entry point on the v100-skinny pages; it
 * exists for code that may not call cudaMalloc -- for example a serving
 * engine that has handed all free HBM to its own pool (KV cache and weights)
 * and forbids raw allocations, a plugin running inside a host framework that
 * gives it no allocator, or a latency-critical caller that must not hit
 * cudaMalloc's implicit device synchronisation.
 *
 * It computes exactly what skinny_nvfp4_gemm computes with a workspace (same
 * kernel, same split-K schedule, same arguments and errors), but its split-K
 * scratch lives in one static device array of skinny_static_workspace_capacity()
 * bytes (4 MiB) that every GPU which loads this library holds until the
 * process exits.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.  The scratch needed is 8 KB per SM, whatever
 * the shape; a device with more SMs than the array has slots for returns
 * SKINNY_ERR_UNSUPPORTED.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, which may load the library's device code); make that
 * first call outside any stream capture.  Every call enqueues, on `stream`, a
 * clear of the partial-sum slots it uses (so a call that follows one with a
 * device error starts clean), then the GEMM.  All calls on a device
 * share the one array, so calls that can overlap on the GPU (different
 * streams, or concurrent graph branches) race and corrupt each other's
 * results: serialise them. */
int skinny_nvfp4_gemm_static_ws(const void* x, int M, int64_t K, const void* w_packed, float global_scale,
                                int64_t N, void* y, int out_dtype, void* stream);

/* Test hook (host only, no CUDA call): the stream-K schedule the GEMM kernels
 * use for an N x K weight on a device with `sms` SMs, with split-K (split != 0,
 * as with a workspace) or whole row tiles.  For each CTA b of the grid,
 * out[6b .. 6b+5] = (last tile of its range, tiles in its range, first row
 * tile, last row tile, lowest CTA sharing the first row tile, highest CTA
 * sharing the last row tile); tiles are numbered row tile * ceil(K/512) + K
 * tile.  *ctas receives the grid size; SKINNY_ERR_WORKSPACE if it exceeds cap. */
int skinny_debug_schedule(int64_t N, int64_t K, int sms, int split, int* out, int cap, int* ctas);

/* Size in bytes of the static scratch array used by skinny_nvfp4_gemm_static_ws. */
size_t skinny_static_workspace_capacity(void);

/* Test hook: *addr receives the device address of that static array on the
 * current device (looked up with cudaGetSymbolAddress, as the entry point
 * does), so that a test can overwrite it between calls.  Returns SKINNY_OK,
 * SKINNY_ERR_INVALID_ARG (null addr) or SKINNY_ERR_CUDA. */
int skinny_debug_static_workspace_address(void** addr);

/* ------------------------------------------------------------------------
 * Measurement.
 * ---------------------------------------------------------------------- */

/* Read `bytes` of device memory once, as fast as this GPU allows, and
 * discard them: the read-only bandwidth ceiling that the GEMMs' effective
 * bandwidth is normalised to (the v100-skinny pages quote their kernels
 * against the read-only limit: aiwitness.kr post, section "내가 실제로 만든
 * 것").  method 0: 16-byte loads from every thread (ld.global.nc, no L1
 * allocation), 8 in flight per thread; it reads bytes rounded down to a
 * multiple of 16.  method 1: one CTA per SM, contiguous 36 KB bulk copies
 * into a 4-slot shared-memory ring, as the GEMMs stream their weights; it
 * reads bytes rounded down to a multiple of 36864.  Asynchronous on
 * `stream`; time it with events.  `sink` (device, may be NULL) is written
 * only if the loaded data XOR to a fixed constant, which keeps the loads
 * live.  Returns SKINNY_OK, INVALID_ARG (null buf, bytes < 16, bad method),
 * ALIGNMENT (buf not 16-byte aligned), UNSUPPORTED or CUDA. */
int skinny_stream_read(const void* buf, size_t bytes, int method, unsigned* sink, void* stream);

/* Device-side error word of the current device.  Every wait inside the
 * kernels is bounded; a wait that gives up sets a bit here instead of
 * hanging (1 = wait for a weight tile, 2 = wait for a free ring slot,
 * 4 = drain of copies in flight after an abort, 8 = split-K finisher waiting
 * for another CTA's partial sums) and its CTA winds down, leaving y
 * incomplete.  Synchronises the device, stores the
 * word in *flags and, if clear != 0, resets it.  Returns SKINNY_OK or
 * SKINNY_ERR_CUDA. */
int skinny_device_error(int clear, unsigned* flags);

#ifdef __cplusplus
}
#endif

#endif /* SKINNY_H */
