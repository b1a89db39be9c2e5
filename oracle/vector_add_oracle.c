/*
 * fp64 CPU oracle for the vector addition of the "TileLang tutorial" (its first
 * kernel, an elementwise C = A + B used as a memory-bandwidth probe).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests and the benchmark's CPU-baseline leg do.
 *
 *   z[i] = x[i] + y[i]   for fp32 x, y, taken in fp64.  The fp64 sum is exact
 *                        unless the exponents differ by more than 29, and then
 *                        the smaller operand is below a quarter fp32 ulp of the
 *                        larger, so rounding z to fp32 always gives the
 *                        correctly rounded fp32 sum.
 */
#include <stdint.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_vector_add(const float* x, const float* y, double* z, int64_t n, int threads) {
    if (n < 0 || (n > 0 && (!x || !y || !z))) return -1;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#else
    (void)threads;
#endif
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) z[i] = (double)x[i] + (double)y[i];
    return 0;
}
