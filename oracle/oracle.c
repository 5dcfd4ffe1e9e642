/*
 * oracle.c -- plain float64 CPU oracle for the weight-only skinny GEMM
 *             y[M,N] = x[M,K] . W^T  (M = 1..8 rows, W kept in NVFP4 or FP8).
 *
 * TEST INFRASTRUCTURE ONLY.  This file exists to check the CUDA path.  It is
 * loaded by the tests, by __graft_entry__.smoke() and by the CPU-baseline leg
 * of bench.py, and by nothing else.  It shares no code, header, table or
 * constant with the CUDA library: every decoder below is written from the
 * format definitions, and the GEMM is the textbook triple loop.
 *
 * What is computed, and where it comes from:
 *   - The pages describe kernels ("QPN2" for NVFP4 regions, "QPN8" for FP8
 *     regions) that keep weights compressed when they are read from HBM, turn
 *     them into FP16 in registers and multiply them against FP16 activations
 *     (taozi.news article on v100-skinny, section "自研 QPN 内核"; the
 *     aiwitness.kr post, section "내가 실제로 만든 것", and its list of
 *     which regions stay FP4 / FP8 and that activations are FP16).  The
 *     result of such a kernel is, up to the order of the FP32 sums, exactly
 *     "dequantise W, then multiply" -- so this oracle is that definition.
 *   - The pages only name NVFP4.  Its encoding is taken from the public
 *     format definitions: 4-bit E2M1 element codes (OCP Microscaling Formats
 *     v1.0, FP4 E2M1), one unsigned E4M3 scale per 16 consecutive elements
 *     along K, and one FP32 per-tensor scale (NVIDIA's NVFP4 description).
 *     The dequantised weight is the product of the three.
 *   - FP8 weights are OCP FP8 E4M3 ("FN": no infinities, S.1111.111 is NaN)
 *     with one FP32 scale per output channel n.
 *   - FP16 activations are IEEE 754 binary16, subnormals included.
 *
 * Every product w*x below is exact in float64 (at most 6+24+11 significant
 * bits), so the only rounding in the oracle is the K-term float64 sum.
 *
 * Parity status: every function here is pinned by tests/test_oracle_pins.py
 * (closed forms, library decoders, exact rational brute force, invariants).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scalar decoders.                                                          */
/* ------------------------------------------------------------------------ */

/* FP4 E2M1 (OCP MX v1.0): bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa.  Exponent 0 is subnormal: 0.5*m.  No Inf/NaN.  The resulting
 * magnitudes are {0, 0.5, 1, 1.5, 2, 3, 4, 6}. */
double oracle_e2m1(unsigned code)
{
    unsigned s = (code >> 3) & 1u;
    unsigned e = (code >> 1) & 3u;
    unsigned m = code & 1u;
    double mag;
    if (e == 0)
        mag = 0.5 * (double)m;
    else
        mag = ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* FP8 E4M3 "FN" (OCP 8-bit floating point spec): bit 7 sign, bits 6..3
 * exponent (bias 7), bits 2..0 mantissa.  Exponent 0 is subnormal
 * (m/8 * 2^-6).  Only S.1111.111 is NaN; there are no infinities, so the
 * largest finite magnitude is 1.75 * 2^8 = 448.  The unsigned UE4M3 block
 * scale of NVFP4 is the same decode with the sign bit required to be 0. */
double oracle_e4m3(unsigned byte)
{
    unsigned s = (byte >> 7) & 1u;
    unsigned e = (byte >> 3) & 15u;
    unsigned m = byte & 7u;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* IEEE 754 binary16: bit 15 sign, bits 14..10 exponent (bias 15), bits 9..0
 * fraction.  Exponent 0 is subnormal (f * 2^-24); exponent 31 is Inf/NaN. */
double oracle_f16(unsigned bits)
{
    unsigned s = (bits >> 15) & 1u;
    unsigned e = (bits >> 10) & 31u;
    unsigned f = bits & 1023u;
    double mag;
    if (e == 31)
        mag = f ? NAN : INFINITY;
    else if (e == 0)
        mag = ldexp((double)f, -24);
    else
        mag = ldexp(1.0 + (double)f / 1024.0, (int)e - 15);
    return s ? -mag : mag;
}

/* ------------------------------------------------------------------------ */
/* The GEMM: decode W row by row into float64, then the plain dot products.  */
/* ------------------------------------------------------------------------ */

enum { FMT_NVFP4 = 0, FMT_FP8 = 1 };

typedef struct {
    int fmt;
    const double* xd;        /* [M][K], decoded activations */
    int64_t M, K, N;
    const uint8_t* codes;    /* NVFP4: [N][K/2] (low nibble = even k); FP8: [N][K] */
    const uint8_t* scales;   /* NVFP4: [N][K/16] UE4M3 bytes */
    double global_scale;     /* NVFP4 per-tensor scale */
    const float* channel_scale; /* FP8: [N] */
    double* y;               /* [M][N] */
    double* bound;           /* [M][N], sum_k |w*x|, may be NULL */
    int64_t n0, n1;          /* rows handled by this worker */
} job_t;

/* Dequantised weight W[n][k] of the NVFP4 tensor:
 *   e2m1(code[n][k]) * ue4m3(scale[n][k/16]) * global_scale. */
static double nvfp4_weight(const job_t* j, int64_t n, int64_t k)
{
    uint8_t byte = j->codes[n * (j->K / 2) + k / 2];
    unsigned code = (k % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4);
    double s = oracle_e4m3(j->scales[n * (j->K / 16) + k / 16]);
    return oracle_e2m1(code) * s * j->global_scale;
}

/* Dequantised weight W[n][k] of the FP8 tensor: e4m3(q[n][k]) * s[n]. */
static double fp8_weight(const job_t* j, int64_t n, int64_t k)
{
    return oracle_e4m3(j->codes[n * j->K + k]) * (double)j->channel_scale[n];
}

static void* run_rows(void* arg)
{
    const job_t* j = (const job_t*)arg;
    double* w = (double*)malloc((size_t)j->K * sizeof(double));
    if (!w)
        return (void*)1;
    for (int64_t n = j->n0; n < j->n1; ++n) {
        for (int64_t k = 0; k < j->K; ++k)
            w[k] = (j->fmt == FMT_NVFP4) ? nvfp4_weight(j, n, k) : fp8_weight(j, n, k);
        for (int64_t m = 0; m < j->M; ++m) {
            const double* xr = j->xd + m * j->K;
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < j->K; ++k) {
                double p = w[k] * xr[k];
                acc += p;
                mag += fabs(p);
            }
            j->y[m * j->N + n] = acc;
            if (j->bound)
                j->bound[m * j->N + n] = mag;
        }
    }
    free(w);
    return NULL;
}

static int run(job_t base, const uint16_t* x, int nthreads)
{
    if (base.M < 1 || base.K < 1 || base.N < 1 || !x || !base.codes || !base.y)
        return -1;
    double* xd = (double*)malloc((size_t)(base.M * base.K) * sizeof(double));
    if (!xd)
        return -2;
    for (int64_t i = 0; i < base.M * base.K; ++i)
        xd[i] = oracle_f16(x[i]);
    base.xd = xd;

    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > base.N)
        nthreads = (int)base.N;
    pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    int rc = 0;
    if (!tid || !jobs) {
        rc = -2;
        goto out;
    }
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = base;
        jobs[t].n0 = base.N * t / nthreads;
        jobs[t].n1 = base.N * (t + 1) / nthreads;
    }
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&tid[t], NULL, run_rows, &jobs[t]) != 0)
            rc = -3;
    if (run_rows(&jobs[0]) != NULL)
        rc = -2;
    for (int t = 1; t < nthreads; ++t) {
        void* r = NULL;
        pthread_join(tid[t], &r);
        if (r != NULL)
            rc = -2;
    }
out:
    free(jobs);
    free(tid);
    free(xd);
    return rc;
}

/* NVFP4 weight-only GEMM, float64.
 *   x      [M][K] binary16 bit patterns
 *   codes  [N][K/2] bytes, element k of row n in byte k/2, low nibble = even k
 *   scales [N][K/16] UE4M3 bytes (one per 16 consecutive k)
 *   y, bound [M][N] float64 outputs (bound = sum_k |w*x|, may be NULL)
 * Returns 0, or a negative value for bad arguments / allocation failure. */
int oracle_nvfp4_gemm(const uint16_t* x, int64_t M, int64_t K, const uint8_t* codes,
                      const uint8_t* scales, float global_scale, int64_t N, double* y,
                      double* bound, int nthreads)
{
    if (K % 16 != 0 || !scales)
        return -1;
    job_t j;
    memset(&j, 0, sizeof(j));
    j.fmt = FMT_NVFP4;
    j.M = M;
    j.K = K;
    j.N = N;
    j.codes = codes;
    j.scales = scales;
    j.global_scale = (double)global_scale;
    j.y = y;
    j.bound = bound;
    return run(j, x, nthreads);
}

/* FP8 (E4M3) weight-only GEMM with an FP32 scale per output channel, float64.
 *   q [N][K] E4M3 bytes, channel_scale [N] float32; other arguments as above. */
int oracle_fp8_gemm(const uint16_t* x, int64_t M, int64_t K, const uint8_t* q,
                    const float* channel_scale, int64_t N, double* y, double* bound,
                    int nthreads)
{
    if (!channel_scale)
        return -1;
    job_t j;
    memset(&j, 0, sizeof(j));
    j.fmt = FMT_FP8;
    j.M = M;
    j.K = K;
    j.N = N;
    j.codes = q;
    j.channel_scale = channel_scale;
    j.y = y;
    j.bound = bound;
    return run(j, x, nthreads);
}
