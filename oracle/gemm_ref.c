/*
 * gemm_ref.c -- TEST INFRASTRUCTURE ONLY.  The plain, slow CPU oracle for the dense
 * matrix multiply C = alpha*A*B + beta*C that the persistent GEMM computes.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load this
 * library.  It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (the definition, written out):
 *   "Triton Low-Level Extensions" producer/consumer matmul (page "Meta presente TLX...",
 *   section "Comment cela fonctionne") and the Hopper sketch on page "Triton 3.7 permite
 *   extender el compilador de GPU sin forks", section "NVIDIA H100 (Hopper): GEMM
 *   persistente": an fp32 accumulator starts at zero and gathers A_tile*B_tile over the
 *   K loop, then the result is stored.  With the alpha/beta update of a BLAS GEMM:
 *
 *     C_ref[i][j] = alpha * sum_{k=0..K-1} a(i,k)*b(k,j) + beta * c0(i,j)
 *     R[i][j]     = |alpha| * sum_k |a(i,k)|*|b(k,j)| + |beta| * |c0(i,j)|
 *
 *   in float64, k ascending, one running sum per output element.  a, b and c0 are the
 *   exact values of the bfloat16, IEEE binary16 (fp16) or float32 inputs: decoding any of
 *   them to double is exact, and the product of two 16-bit values (at most 11 significant
 *   bits each) is exact in double, so only the additions round.  The pages' own GEMM
 *   measurements are FP16 GEMMs (page "Triton 3.7 permite extender el compilador de GPU sin
 *   forks", section "NVIDIA H100 (Hopper): resultados de rendimiento"), hence the fp16
 *   operand type beside bf16.
 *   R is the magnitude bound used by the tolerance.
 *   beta == 0 means c0 is not read at all (a NaN in C does not propagate), as in BLAS.
 *
 * Layouts (element addresses, 0-based):
 *   a(i,k) = A[i*lda + k]                          (A row-major M x K)
 *   b(k,j) = B[j*ldb + k]   when b_kmajor != 0     (B stored N x K row-major, "K-major")
 *          = B[k*ldb + j]   when b_kmajor == 0     (B stored K x N row-major, "N-major")
 *   c0(i,j)= C0[i*ldc0 + j] of type c0_type (0: none, 1: float32, 2: bfloat16 bits,
 *            3: fp16 bits)
 *   A and B hold 16-bit patterns of type in_type (0: bfloat16, 1: fp16).
 *
 * Outputs are dense nrows x N float64 arrays (row r of the output is matrix row rows[r]).
 * OpenMP splits the output rows across threads; each element's summation order is the
 * same whatever the thread count.  Four columns are summed side by side (four separate
 * running sums) only to use the FPU's parallelism; the order inside each sum is k ascending.
 *
 * ORACLE_PLANT (compile-time, default 0) plants one deliberate mistake so that the tests
 * can show that the oracle's pins catch it.  The default build plants nothing.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

static double bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * exponent 0: subnormal, fraction * 2^-24; exponent 31: infinity (fraction 0) or NaN;
 * otherwise (1024 + fraction) * 2^(exponent - 25).  ldexp of a small integer is exact. */
static double f16_value(uint16_t h) {
    int sign = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);
    } else if (e == 31) {
        v = f == 0 ? INFINITY : NAN;
    } else {
#if ORACLE_PLANT == 9 /* planted: fp16 exponent bias off by one */
        v = ldexp((double)(1024 + f), e - 24);
#else
        v = ldexp((double)(1024 + f), e - 25);
#endif
    }
    return sign ? -v : v;
}

static double in_value(uint16_t h, int in_type) { return in_type ? f16_value(h) : bf16_value(h); }

static double c0_value(const void* C0, int c0_type, long long idx) {
    if (c0_type == 1) return (double)((const float*)C0)[idx];
    if (c0_type == 2) return bf16_value(((const uint16_t*)C0)[idx]);
    if (c0_type == 3) return f16_value(((const uint16_t*)C0)[idx]);
    return 0.0;
}

static double b_value(const uint16_t* B, long long ldb, int b_kmajor, long long k, long long j,
                      int K, int N, int in_type) {
#if ORACLE_PLANT == 3 /* planted: operand B read transposed (indices wrapped to stay in bounds) */
    long long kk = j % K, jj = k % N;
    return in_value(b_kmajor ? B[jj * ldb + kk] : B[kk * ldb + jj], in_type);
#elif ORACLE_PLANT == 6 /* planted: column index off by one (wrapped) */
    j = (j + 1) % N;
    return in_value(b_kmajor ? B[j * ldb + k] : B[k * ldb + j], in_type);
#else
    (void)K; (void)N;
    return in_value(b_kmajor ? B[j * ldb + k] : B[k * ldb + j], in_type);
#endif
}

/* Exact values of n 16-bit patterns of type in_type (0: bfloat16, 1: fp16). */
void oracle_decode(int in_type, const uint16_t* h, long long n, double* out) {
    for (long long i = 0; i < n; ++i) out[i] = in_value(h[i], in_type);
}

int oracle_version(void) { return 2; }

int oracle_plant(void) { return ORACLE_PLANT; }

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One output row (matrix row i) into out[0..N-1], bound into rb[0..N-1] (rb may be NULL). */
static void gemm_row(int N, int K, const uint16_t* A, long long lda, const uint16_t* B,
                     long long ldb, int b_kmajor, const void* C0, long long ldc0, int c0_type,
                     double alpha, double beta, long long i, double* out, double* rb, int in_type) {
    const uint16_t* arow = A + i * lda;
    int kend = K, kbeg = 0;
#if ORACLE_PLANT == 1 /* planted: last k term dropped */
    kend = K > 0 ? K - 1 : 0;
#elif ORACLE_PLANT == 8 /* planted: first k term dropped */
    kbeg = 1;
#endif
    int j = 0;
    for (; j + 4 <= N; j += 4) {
        double s0 = 0, s1 = 0, s2 = 0, s3 = 0, r0 = 0, r1 = 0, r2 = 0, r3 = 0;
        for (int k = kbeg; k < kend; ++k) {
            double a = in_value(arow[k], in_type);
            double p0 = a * b_value(B, ldb, b_kmajor, k, j + 0, K, N, in_type);
            double p1 = a * b_value(B, ldb, b_kmajor, k, j + 1, K, N, in_type);
            double p2 = a * b_value(B, ldb, b_kmajor, k, j + 2, K, N, in_type);
            double p3 = a * b_value(B, ldb, b_kmajor, k, j + 3, K, N, in_type);
#if ORACLE_PLANT == 7 /* planted: running sums rounded to float32 */
            s0 = (float)(s0 + p0); s1 = (float)(s1 + p1); s2 = (float)(s2 + p2); s3 = (float)(s3 + p3);
#else
            s0 += p0; s1 += p1; s2 += p2; s3 += p3;
#endif
            r0 += fabs(p0); r1 += fabs(p1); r2 += fabs(p2); r3 += fabs(p3);
        }
        double s[4] = {s0, s1, s2, s3}, r[4] = {r0, r1, r2, r3};
        for (int t = 0; t < 4; ++t) {
            double v = alpha * s[t];
            double bound = fabs(alpha) * r[t];
            if (beta != 0.0) {
                double c = c0_value(C0, c0_type, i * ldc0 + j + t);
#if ORACLE_PLANT == 2 /* planted: wrong sign on the beta term */
                v -= beta * c;
#elif ORACLE_PLANT == 4 /* planted: alpha also scales the old C */
                v += alpha * beta * c;
#else
                v += beta * c;
#endif
                bound += fabs(beta) * fabs(c);
            }
            out[j + t] = v;
            if (rb) rb[j + t] = bound;
        }
    }
    for (; j < N; ++j) {
        double s = 0, r = 0;
        for (int k = kbeg; k < kend; ++k) {
            double p = in_value(arow[k], in_type) * b_value(B, ldb, b_kmajor, k, j, K, N, in_type);
#if ORACLE_PLANT == 7
            s = (float)(s + p);
#else
            s += p;
#endif
            r += fabs(p);
        }
        double v = alpha * s;
        double bound = fabs(alpha) * r;
        if (beta != 0.0) {
            double c = c0_value(C0, c0_type, i * ldc0 + j);
#if ORACLE_PLANT == 2
            v -= beta * c;
#elif ORACLE_PLANT == 4
            v += alpha * beta * c;
#else
            v += beta * c;
#endif
            bound += fabs(beta) * fabs(c);
        }
        out[j] = v;
        if (rb) rb[j] = bound;
    }
}

/*
 * oracle_gemm: rows[0..nrows-1] of C_ref (and R) for one GEMM.  rows == NULL means all
 * M rows (nrows must then equal M).  in_type: 0 = A and B are bfloat16, 1 = fp16.
 * Returns 0, or -1 on a bad argument.
 */
int oracle_gemm(int M, int N, int K, const uint16_t* A, long long lda, const uint16_t* B,
                long long ldb, int b_kmajor, const void* C0, long long ldc0, int c0_type,
                double alpha, double beta, const int* rows, int nrows, double* Cref, double* R,
                int in_type) {
    if (M < 0 || N < 0 || K < 0 || nrows < 0) return -1;
    if (in_type != 0 && in_type != 1) return -1;
    if (!rows && nrows != M) return -1;
    if (beta != 0.0 && c0_type == 0) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        long long i = rows ? rows[r] : r;
#if ORACLE_PLANT == 5 /* planted: output row taken from the next row of A */
        i = (i + 1) % (M > 0 ? M : 1);
#endif
        gemm_row(N, K, A, lda, B, ldb, b_kmajor, C0, ldc0, c0_type, alpha, beta, i,
                 Cref + (long long)r * N, R ? R + (long long)r * N : (double*)0, in_type);
    }
    return 0;
}

/*
 * oracle_gemm_batched: Y_ref[b] = alpha * W * X[b] + beta * Y0[b] for b in [0, batch),
 * with W shared (M x K row-major, ldw), X[b] = X + b*stride_x stored K x N row-major
 * (ldx) and Y0[b] = Y0 + b*stride_y (ldy).  Only the rows listed in rows[0..nrows-1]
 * (all M when rows == NULL) of each batch are produced; output batch b occupies
 * Cref[b*nrows*N ...].  This is the single-GEMM definition applied to each b in turn.
 *
 * With index != NULL (the deduplicated form: the request holds only the distinct feature
 * entries, page "Meta accelere un noyau GPU d'un facteur 4 avec TLX...", sections "Comment le
 * chargement des donnees gene le calcul" and "Ce que signifie une acceleration d'un facteur
 * quatre"), item b's operand is the distinct entry index[b]: X[b] = X + index[b]*stride_x,
 * 0 <= index[b] < n_x.  Each item is still its own plain GEMM.
 */
int oracle_gemm_batched(int batch, int M, int N, int K, const uint16_t* W, long long ldw,
                        const uint16_t* X, long long ldx, long long stride_x, const void* Y0,
                        long long ldy, long long stride_y, int y_type, double alpha,
                        double beta, const int* rows, int nrows, double* Cref, double* R,
                        int in_type, const int* index, int n_x) {
    if (batch < 0) return -1;
    if (!rows && nrows != M) return -1;
    long long per = (long long)nrows * N;
    for (int b = 0; b < batch; ++b) {
        long long xb = b;
        if (index) {
#if ORACLE_PLANT == 10 /* planted: the item's own position used instead of its distinct entry */
            xb = b % (n_x > 0 ? n_x : 1);
#else
            xb = index[b];
#endif
            if (xb < 0 || xb >= n_x) return -1;
        }
        const void* yb = 0;
        if (y_type == 1) yb = (const float*)Y0 + (long long)b * stride_y;
        if (y_type == 2 || y_type == 3) yb = (const uint16_t*)Y0 + (long long)b * stride_y;
        int rc = oracle_gemm(M, N, K, W, ldw, X + xb * stride_x, ldx, 0, yb, ldy,
                             y_type, alpha, beta, rows, nrows, Cref + b * per,
                             R ? R + b * per : (double*)0, in_type);
        if (rc) return rc;
    }
    return 0;
}
