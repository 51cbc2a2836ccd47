/*
 * oracle/gemv_oracle.c -- plain fp64 CPU oracle for the decode projection
 * y = x W^T of a bf16 linear layer with a small number of rows M.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline / reference leg of bench.py may load this library.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * What it computes (AstrAI commit 7540acb4, astrai/extension/ops/gemv.py and
 * docs/developer/decode_linear_benchmark.md, commit logs: the bf16 GEMV that
 * decode-time linear layers dispatch to for M = 1..8 rows, on weights laid out as
 * [out_features, in_features]):
 *
 *     y[m][n] = sum_k x[m][k] * W[n][k]        m < M, n < N, k < K
 *
 * The page names the operation (a linear layer's forward at decode) without
 * writing it out; this is the nn.Linear definition with no bias.  Inputs are bf16
 * widened to double exactly; every product of two bf16 values is exact in
 * double; the K-term sum is IEEE double in index order.  The companion function
 * gives sum_k |x[m][k] * W[n][k]|, the scale of the rounding error of any
 * summation order, for the tolerance of the tests.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_value(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* x: bf16 [M][ldx], w: bf16 [N][ldw], y (out): double [M][N] row-major.
 * absy (out, may be NULL): double [M][N] of sum_k |x w|.  Returns 0, or 1 on bad
 * arguments. */
int oracle_gemv(const uint16_t* x, int64_t ldx, const uint16_t* w, int64_t ldw, int M, int N, int K, double* y,
                double* absy, int nthreads) {
    if (!x || !w || !y || M < 0 || N < 0 || K < 0 || ldx < K || ldw < K) return 1;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int n = 0; n < N; ++n) {
        for (int m = 0; m < M; ++m) {
            double s = 0.0, a = 0.0;
            for (int k = 0; k < K; ++k) {
                const double p = bf16_value(x[(int64_t)m * ldx + k]) * bf16_value(w[(int64_t)n * ldw + k]);
                s += p;
                a += fabs(p);
            }
            y[(int64_t)m * N + n] = s;
            if (absy) absy[(int64_t)m * N + n] = a;
        }
    }
    return 0;
}
