/*
 * fp64 CPU oracle for the tiled tensor-core GEMM and its fused bias + GELU
 * epilogue.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code with the CUDA kernels.
 *
 * What it computes ("TileLang tutorial": the tiled tensor-core matrix
 * multiplication section, C = A B, and the fused-epilogue section, which adds
 * a bias and applies GELU to the accumulator before the single store):
 *
 *   acc[i, j] = sum_k A[i, k] B[k, j]                       (fp64, k in order)
 *   epilogue 0:  C[i, j] = acc[i, j]
 *   epilogue 1:  C[i, j] = acc[i, j] + bias[j]
 *   epilogue 2:  C[i, j] = GELU(acc[i, j] + bias[j]),  GELU(x) = x * Phi(x)
 *                        = x/2 * (1 + erf(x / sqrt 2))     (the exact form)
 *
 * A is [M, K] and B is [K, N], both row-major bf16 bit patterns widened
 * exactly; bias is bf16 [N].  C is fp64 [M, N].  K = 0 gives acc = 0.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_value(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double gelu_exact(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }

static double epilogue(double acc, const uint16_t* bias, int64_t j, int mode) {
    if (mode == 0) return acc;
    const double pre = acc + bf16_value(bias[j]);
    return mode == 1 ? pre : gelu_exact(pre);
}

static double dot_column(const uint16_t* a, const uint16_t* b, int64_t N, int64_t K, int64_t i,
                         int64_t j) {
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) acc += bf16_value(a[i * K + k]) * bf16_value(b[k * N + j]);
    return acc;
}

static void set_threads(int threads) {
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#else
    (void)threads;
#endif
}

/* Full C [M, N].  Returns 0, or -1 on bad arguments. */
int oracle_gemm(const uint16_t* a, const uint16_t* b, const uint16_t* bias, double* c, int64_t M,
                int64_t N, int64_t K, int mode, int threads) {
    if (!c || M < 0 || N < 0 || K < 0 || mode < 0 || mode > 2) return -1;
    if (K > 0 && (!a || !b)) return -1;
    if (mode > 0 && N > 0 && !bias) return -1;
    set_threads(threads);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < N; ++j) c[i * N + j] = epilogue(dot_column(a, b, N, K, i, j), bias, j, mode);
    return 0;
}

/* Selected entries only: idx[r] = i * N + j.  out[r] = C[i, j] with the
 * arithmetic of oracle_gemm. */
int oracle_gemm_entries(const uint16_t* a, const uint16_t* b, const uint16_t* bias, int64_t M,
                        int64_t N, int64_t K, int mode, const int64_t* idx, int64_t n,
                        double* out, int threads) {
    if (!idx || !out || M <= 0 || N <= 0 || K < 0 || mode < 0 || mode > 2) return -1;
    if (K > 0 && (!a || !b)) return -1;
    if (mode > 0 && !bias) return -1;
    for (int64_t r = 0; r < n; ++r)
        if (idx[r] < 0 || idx[r] >= M * N) return -1;
    set_threads(threads);
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < n; ++r) {
        const int64_t i = idx[r] / N, j = idx[r] % N;
        out[r] = epilogue(dot_column(a, b, N, K, i, j), bias, j, mode);
    }
    return 0;
}
