/*
 * nvfp4_oracle.c -- plain FP64 CPU reference for the block-scaled NVFP4 matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke() check and
 * the CPU-baseline leg of bench.py may load this library.  The GPU product path
 * never calls it, and it shares no code, header, table or helper with the CUDA
 * library (block_scaled_precision_nvfp4_b200/csrc).
 *
 * What it computes (metrale_circuit `hardware::exec` module doc, bullets 1-2,
 * and the block-scaled formats named there):
 *
 *   Y[m,n] = gA * gW * sum_g  sA[m,g] * sW[n,g] * sum_{k in g} e2m1(A[m,k]) * e2m1(W[n,k])
 *
 * with groups g of 16 consecutive k, E2M1 codes packed two per byte (even k in
 * the low nibble, odd k in the high nibble), E4M3 group scales stored one byte
 * per (row, group) row-major as [rows][K/16], and per-tensor FP32 scales gA, gW.
 * Everything inside the sum is evaluated in FP64, where every product and
 * every 16-term group sum is exact; only the sum over groups rounds (at 2^-53).
 *
 * Each output element is computed independently by one function; threads only
 * split the list of output elements.  There is no blocking, fusion or
 * reordering of the arithmetic beyond the definition above.
 *
 * Parity pins for every function are in tests/test_oracle_pins.py.  The one
 * thing no pin fixes is the last bit of the GPU's FP32 accumulation order,
 * which only the tolerance covers ("parity unpinned" for that bit alone).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Format tables                                                              */
/* ------------------------------------------------------------------------- */

/* E2M1 (FP4): 1 sign bit (bit 3), 2 exponent bits (bits 2-1, bias 1), 1
 * mantissa bit (bit 0).  Exponent field 0 is subnormal: 0 or 0.5.  The table is
 * indexed by the 4-bit code.  Code 8 is negative zero. */
static const double E2M1[16] = {
    0.0,  0.5,  1.0,  1.5,  2.0,  3.0,  4.0,  6.0,
    -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0,
};

/* E4M3 (OCP "FN" variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal (2^-6 * M/8); 0x7F and 0xFF are NaN;
 * there is no infinity; the largest finite value is 448.  Filled once from
 * the field definition. */
static double E4M3[256];
static pthread_once_t e4m3_once = PTHREAD_ONCE_INIT;

static void e4m3_build(void) {
    for (int b = 0; b < 256; ++b) {
        int s = (b >> 7) & 1, E = (b >> 3) & 15, M = b & 7;
        double mag;
        if (E == 15 && M == 7)
            mag = NAN;
        else if (E == 0)
            mag = ldexp((double)M / 8.0, -6);
        else
            mag = ldexp(1.0 + (double)M / 8.0, E - 7);
        E4M3[b] = s ? -mag : mag;
    }
}

static inline double e4m3(uint8_t b) { return E4M3[b]; }

/* Code k of a packed row: even k in the low nibble, odd k in the high one. */
static inline int code_at(const uint8_t* row, int64_t k) {
    uint8_t byte = row[k >> 1];
    return (k & 1) ? (byte >> 4) : (byte & 0x0F);
}

double oracle_e2m1_value(int code) { return E2M1[code & 15]; }

double oracle_e4m3_value(int byte) {
    pthread_once(&e4m3_once, e4m3_build);
    return E4M3[byte & 255];
}

/* The exact E2M1 -> E4M3 conversion of the `hardware::exec` module doc,
 * bullet 2, applied to a 32-bit word holding four codes, each in the HIGH
 * nibble of its byte: (q & 0x80808080) | ((q & 0x70707070) >> 2).  Each
 * resulting byte, read as E4M3, is the code's E2M1 value times 2^-6. */
uint32_t oracle_e2m1_to_e4m3_word(uint32_t q) {
    return (q & 0x80808080u) | ((q & 0x70707070u) >> 2);
}

/* ------------------------------------------------------------------------- */
/* One output element per path                                               */
/* ------------------------------------------------------------------------- */

/* W4A4: the block-scaled FP4 MMA path (module doc, bullet 1, NVFP4 row). */
static double elem_w4a4(const uint8_t* A, const uint8_t* sA, const uint8_t* W,
                        const uint8_t* sW, double alpha, int64_t K, int64_t m,
                        int64_t n) {
    const int64_t G = K / 16;
    const uint8_t* a = A + m * (K / 2);
    const uint8_t* w = W + n * (K / 2);
    double acc = 0.0;
    for (int64_t g = 0; g < G; ++g) {
        double p = 0.0; /* exact: at most 16 terms of magnitude <= 36 on a 1/4 grid */
        for (int64_t k = 16 * g; k < 16 * g + 16; ++k)
            p += E2M1[code_at(a, k)] * E2M1[code_at(w, k)];
        acc += e4m3(sA[m * G + g]) * e4m3(sW[n * G + g]) * p;
    }
    return alpha * acc;
}

/* The exact FP8 path (module doc, bullet 2), in the pages' own steps: every
 * code is moved to the high nibble of a byte, converted by the bit identity to
 * an E4M3 byte worth value * 2^-6, decoded from the E4M3 table; the 16-term
 * group partial is formed from these FP8 values, and the group scales carry
 * the folded 2^6 each, applied per K=16 step.  The result must equal
 * elem_w4a4 exactly (all terms are exact in FP64). */
static double elem_via_fp8(const uint8_t* A, const uint8_t* sA, const uint8_t* W,
                           const uint8_t* sW, double alpha, int64_t K, int64_t m,
                           int64_t n) {
    const int64_t G = K / 16;
    const uint8_t* a = A + m * (K / 2);
    const uint8_t* w = W + n * (K / 2);
    double acc = 0.0;
    for (int64_t g = 0; g < G; ++g) {
        double p = 0.0;
        for (int64_t k = 16 * g; k < 16 * g + 16; ++k) {
            uint32_t qa = (uint32_t)code_at(a, k) << 4;
            uint32_t qw = (uint32_t)code_at(w, k) << 4;
            uint8_t a8 = (uint8_t)(oracle_e2m1_to_e4m3_word(qa) & 0xFF);
            uint8_t w8 = (uint8_t)(oracle_e2m1_to_e4m3_word(qw) & 0xFF);
            p += e4m3(a8) * e4m3(w8);
        }
        double sa = e4m3(sA[m * G + g]) * 64.0; /* 2^6 folded into the group scale */
        double sw = e4m3(sW[n * G + g]) * 64.0;
        acc += p * sa * sw;
    }
    return alpha * acc;
}

/* BF16 bits -> value (exact). */
static inline double bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* W4A16: BF16 activations times NVFP4 weights widened to their values
 * (module doc, bullet 1, BF16 row: "any weight format widened"). */
static double elem_w4a16(const uint16_t* A, const uint8_t* W, const uint8_t* sW,
                         double gW, int64_t K, int64_t m, int64_t n) {
    const int64_t G = K / 16;
    const uint16_t* a = A + m * K;
    const uint8_t* w = W + n * (K / 2);
    double acc = 0.0;
    for (int64_t g = 0; g < G; ++g) {
        double p = 0.0;
        for (int64_t k = 16 * g; k < 16 * g + 16; ++k)
            p += bf16_value(a[k]) * E2M1[code_at(w, k)];
        acc += e4m3(sW[n * G + g]) * p;
    }
    return gW * acc;
}

/* W4A8: FP8 (E4M3) activations under NVFP4 weights (module doc, exec_of:
 * "W4A8 with group-16 E4M3 scales ... take the exact E4M3 path").  The
 * activations carry only their per-tensor scale gA; the weights their group
 * scales and gW:  Y = gA*gW * sum_g sW[n,g] * sum_{k in g} e4m3(A[m,k]) * e2m1(W[n,k]).
 * A is one E4M3 byte per element [M][K]; NaN bytes (0x7F, 0xFF) are not inputs. */
static double elem_w4a8(const uint8_t* A, const uint8_t* W, const uint8_t* sW, double alpha,
                        int64_t K, int64_t m, int64_t n) {
    const int64_t G = K / 16;
    const uint8_t* a = A + m * K;
    const uint8_t* w = W + n * (K / 2);
    double acc = 0.0;
    for (int64_t g = 0; g < G; ++g) {
        double p = 0.0; /* exact: 16 products on a 2^-10 grid, |p| <= 16 * 448 * 6 */
        for (int64_t k = 16 * g; k < 16 * g + 16; ++k)
            p += e4m3(a[k]) * E2M1[code_at(w, k)];
        acc += e4m3(sW[n * G + g]) * p;
    }
    return alpha * acc;
}

/* ------------------------------------------------------------------------- */
/* Threaded drivers over a list of output elements                            */
/* ------------------------------------------------------------------------- */

enum { P_W4A4 = 0, P_VIA_FP8 = 1, P_W4A16 = 2, P_GROUPED = 3, P_W4A8 = 4 };

typedef struct {
    int path;
    const void* A;
    const uint8_t *sA, *W, *sW;
    double gA, gW;
    const double* gWe;      /* grouped: per-expert weight scale */
    const int64_t* offsets; /* grouped: [E+1] row offsets */
    int64_t E, M, N, K;
    const int64_t *rows, *cols; /* sampled mode; NULL = all M*N row-major */
    int64_t count;
    double* out;
    int64_t begin, end;
} job_t;

static int64_t expert_of(const int64_t* offsets, int64_t E, int64_t row) {
    int64_t lo = 0, hi = E; /* find e with offsets[e] <= row < offsets[e+1] */
    while (hi - lo > 1) {
        int64_t mid = (lo + hi) / 2;
        if (offsets[mid] <= row) lo = mid; else hi = mid;
    }
    while (lo < E && offsets[lo + 1] <= row) ++lo; /* skip empty experts */
    return lo;
}

static double one(const job_t* j, int64_t m, int64_t n) {
    switch (j->path) {
    case P_W4A4:
        return elem_w4a4((const uint8_t*)j->A, j->sA, j->W, j->sW, j->gA * j->gW, j->K, m, n);
    case P_VIA_FP8:
        return elem_via_fp8((const uint8_t*)j->A, j->sA, j->W, j->sW, j->gA * j->gW, j->K, m, n);
    case P_W4A16:
        return elem_w4a16((const uint16_t*)j->A, j->W, j->sW, j->gW, j->K, m, n);
    case P_W4A8:
        return elem_w4a8((const uint8_t*)j->A, j->W, j->sW, j->gA * j->gW, j->K, m, n);
    case P_GROUPED: {
        int64_t e = expert_of(j->offsets, j->E, m);
        const uint8_t* We = j->W + e * j->N * (j->K / 2);
        const uint8_t* sWe = j->sW + e * j->N * (j->K / 16);
        return elem_w4a4((const uint8_t*)j->A, j->sA, We, sWe, j->gA * j->gWe[e], j->K, m, n);
    }
    }
    return NAN;
}

static void* worker(void* arg) {
    job_t* j = (job_t*)arg;
    for (int64_t i = j->begin; i < j->end; ++i) {
        int64_t m, n;
        if (j->rows) { m = j->rows[i]; n = j->cols[i]; }
        else { m = i / j->N; n = i % j->N; }
        j->out[i] = one(j, m, n);
    }
    return NULL;
}

static int run(job_t proto, int nthreads) {
    pthread_once(&e4m3_once, e4m3_build);
    if (proto.count <= 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > proto.count) nthreads = (int)proto.count;
    pthread_t th[256];
    job_t jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = proto;
        jobs[t].begin = proto.count * t / nthreads;
        jobs[t].end = proto.count * (t + 1) / nthreads;
    }
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, worker, &jobs[t]) != 0) return -1;
    worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    return 0;
}

static int bad_shape(int64_t M, int64_t N, int64_t K) {
    return M < 0 || N < 0 || K < 16 || (K % 16) != 0 || (K % 2) != 0;
}

/* ------------------------------------------------------------------------- */
/* Public entry points (dense: all M*N outputs row-major; _at: sampled)       */
/* ------------------------------------------------------------------------- */

int oracle_gemm_w4a4(const uint8_t* A, const uint8_t* sA, double gA, const uint8_t* W,
                     const uint8_t* sW, double gW, int64_t M, int64_t N, int64_t K,
                     double* Y, int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_W4A4, A, sA, W, sW, gA, gW, NULL, NULL, 0, M, N, K, NULL, NULL, M * N, Y, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_w4a4_at(const uint8_t* A, const uint8_t* sA, double gA, const uint8_t* W,
                        const uint8_t* sW, double gW, int64_t M, int64_t N, int64_t K,
                        const int64_t* rows, const int64_t* cols, int64_t count, double* out,
                        int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_W4A4, A, sA, W, sW, gA, gW, NULL, NULL, 0, M, N, K, rows, cols, count, out, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_via_fp8(const uint8_t* A, const uint8_t* sA, double gA, const uint8_t* W,
                        const uint8_t* sW, double gW, int64_t M, int64_t N, int64_t K,
                        double* Y, int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_VIA_FP8, A, sA, W, sW, gA, gW, NULL, NULL, 0, M, N, K, NULL, NULL, M * N, Y, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_via_fp8_at(const uint8_t* A, const uint8_t* sA, double gA, const uint8_t* W,
                           const uint8_t* sW, double gW, int64_t M, int64_t N, int64_t K,
                           const int64_t* rows, const int64_t* cols, int64_t count,
                           double* out, int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_VIA_FP8, A, sA, W, sW, gA, gW, NULL, NULL, 0, M, N, K, rows, cols, count, out, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_w4a8(const uint8_t* A, double gA, const uint8_t* W, const uint8_t* sW, double gW,
                     int64_t M, int64_t N, int64_t K, double* Y, int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_W4A8, A, NULL, W, sW, gA, gW, NULL, NULL, 0, M, N, K, NULL, NULL, M * N, Y, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_w4a8_at(const uint8_t* A, double gA, const uint8_t* W, const uint8_t* sW,
                        double gW, int64_t M, int64_t N, int64_t K, const int64_t* rows,
                        const int64_t* cols, int64_t count, double* out, int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_W4A8, A, NULL, W, sW, gA, gW, NULL, NULL, 0, M, N, K, rows, cols, count, out, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_w4a16(const uint16_t* A, const uint8_t* W, const uint8_t* sW, double gW,
                      int64_t M, int64_t N, int64_t K, double* Y, int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_W4A16, A, NULL, W, sW, 1.0, gW, NULL, NULL, 0, M, N, K, NULL, NULL, M * N, Y, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_w4a16_at(const uint16_t* A, const uint8_t* W, const uint8_t* sW, double gW,
                         int64_t M, int64_t N, int64_t K, const int64_t* rows,
                         const int64_t* cols, int64_t count, double* out, int nthreads) {
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_W4A16, A, NULL, W, sW, 1.0, gW, NULL, NULL, 0, M, N, K, rows, cols, count, out, 0, 0};
    return run(j, nthreads);
}

/* Grouped (per-expert) W4A4: rows offsets[e] .. offsets[e+1]-1 of A use expert
 * e's weights W[e] ([N][K/2] bytes), scales sW[e] ([N][K/16]) and gW[e]. */
static int bad_offsets(const int64_t* offsets, int64_t E) {
    if (E < 1 || offsets[0] != 0) return 1;
    for (int64_t e = 0; e < E; ++e)
        if (offsets[e + 1] < offsets[e]) return 1;
    return 0;
}

int oracle_gemm_grouped_w4a4(const uint8_t* A, const uint8_t* sA, double gA, const uint8_t* W,
                             const uint8_t* sW, const double* gW, const int64_t* offsets,
                             int64_t E, int64_t N, int64_t K, double* Y, int nthreads) {
    if (bad_offsets(offsets, E)) return -3;
    int64_t M = offsets[E];
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_GROUPED, A, sA, W, sW, gA, 1.0, gW, offsets, E, M, N, K, NULL, NULL, M * N, Y, 0, 0};
    return run(j, nthreads);
}

int oracle_gemm_grouped_w4a4_at(const uint8_t* A, const uint8_t* sA, double gA,
                                const uint8_t* W, const uint8_t* sW, const double* gW,
                                const int64_t* offsets, int64_t E, int64_t N, int64_t K,
                                const int64_t* rows, const int64_t* cols, int64_t count,
                                double* out, int nthreads) {
    if (bad_offsets(offsets, E)) return -3;
    int64_t M = offsets[E];
    if (bad_shape(M, N, K)) return -2;
    job_t j = {P_GROUPED, A, sA, W, sW, gA, 1.0, gW, offsets, E, M, N, K, rows, cols, count, out, 0, 0};
    return run(j, nthreads);
}
