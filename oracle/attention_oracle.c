/*
 * fp64 CPU oracle for the fused attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code with the CUDA kernels.
 *
 * What it computes (the plain definition of the result the fused kernel
 * reaches without materialising the scores; "TileLang tutorial", FlashAttention
 * section: a fused forward pass over query/key/value tiles, validated against
 * PyTorch scaled-dot-product attention, causal and non-causal):
 *
 *   for every (b, h) and every query row i:
 *     S[i, j] = scale * sum_t Q[i, t] K[j, t]            (all j, fp64)
 *     S[i, j] = -inf  if causal and j > i                 (top-left causal mask)
 *     m_i     = max_j S[i, j]
 *     l_i     = sum_j exp(S[i, j] - m_i)
 *     P[i, j] = exp(S[i, j] - m_i) / l_i                  (row softmax)
 *     O[i, :] = sum_j P[i, j] V[j, :]
 *     LSE_i   = m_i + ln l_i        (natural log of sum_j exp(S[i, j]))
 *
 * The score row S[i, :] and the probability row P[i, :] are materialised in
 * full for every query row; nothing is blocked, fused or reordered.  A row
 * whose keys are all masked (it cannot occur with the top-left causal mask and
 * equal query/key lengths) gets O = 0 and LSE = -inf.
 *
 * Inputs are bf16 bit patterns (uint16, [B, H, N, d], contiguous), widened
 * exactly to fp64.  Outputs are fp64: O [B, H, N, d] and LSE [B, H, N].
 *
 * Also here: the row-wise softmax of the tutorial's softmax section (a row's
 * maximum and sum reductions, then normalisation):
 *     y[r, c] = exp(scale * x[r, c] - max_c' scale * x[r, c']) / sum_c' exp(...)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* One complete query row of one (b, h) slice.  q_row: d values; kh, vh: N x d
 * values of the slice; s and p: scratch rows of length N. */
static void attention_row(const double* q_row, const double* kh, const double* vh,
                          int64_t N, int64_t d, int64_t i, int causal, double scale,
                          double* s, double* p, double* o_row, double* lse_out) {
    /* scores */
    for (int64_t j = 0; j < N; ++j) {
        if (causal && j > i) {
            s[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t) acc += q_row[t] * kh[j * d + t];
        s[j] = scale * acc;
    }
    /* row softmax, two passes over the complete row */
    double m = -INFINITY;
    for (int64_t j = 0; j < N; ++j)
        if (s[j] > m) m = s[j];
    if (m == -INFINITY) {
        for (int64_t t = 0; t < d; ++t) o_row[t] = 0.0;
        *lse_out = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int64_t j = 0; j < N; ++j) l += exp(s[j] - m);
    for (int64_t j = 0; j < N; ++j) p[j] = exp(s[j] - m) / l;
    /* O = P V */
    for (int64_t t = 0; t < d; ++t) o_row[t] = 0.0;
    for (int64_t j = 0; j < N; ++j) {
        if (p[j] == 0.0) continue; /* exact: adds nothing */
        for (int64_t t = 0; t < d; ++t) o_row[t] += p[j] * vh[j * d + t];
    }
    *lse_out = m + log(l);
}

static void widen_slice(const uint16_t* src, double* dst, int64_t count) {
    for (int64_t x = 0; x < count; ++x) dst[x] = bf16_to_double(src[x]);
}

static void set_threads(int threads) {
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#else
    (void)threads;
#endif
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Full forward pass over every (b, h, i).  Returns 0, or -1 on bad arguments /
 * allocation failure.  threads <= 0 keeps the OpenMP default. */
int oracle_attention_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, double* o,
                         double* lse, int64_t B, int64_t H, int64_t N, int64_t d, int causal,
                         double scale, int threads) {
    if (!q || !k || !v || !o || !lse || B < 0 || H < 0 || N < 0 || d <= 0) return -1;
    set_threads(threads);
    const int64_t BH = B * H;
    int status = 0;
    for (int64_t bh = 0; bh < BH && status == 0; ++bh) {
        const int64_t base = bh * N * d;
        double* qh = (double*)malloc(sizeof(double) * (size_t)(N * d + 1));
        double* kh = (double*)malloc(sizeof(double) * (size_t)(N * d + 1));
        double* vh = (double*)malloc(sizeof(double) * (size_t)(N * d + 1));
        if (!qh || !kh || !vh) {
            free(qh); free(kh); free(vh);
            return -1;
        }
        widen_slice(q + base, qh, N * d);
        widen_slice(k + base, kh, N * d);
        widen_slice(v + base, vh, N * d);
#pragma omp parallel
        {
            double* s = (double*)malloc(sizeof(double) * (size_t)(N + 1));
            double* p = (double*)malloc(sizeof(double) * (size_t)(N + 1));
            if (!s || !p) {
#pragma omp atomic write
                status = -1;
            } else {
#pragma omp for schedule(dynamic, 4)
                for (int64_t i = 0; i < N; ++i)
                    attention_row(qh + i * d, kh, vh, N, d, i, causal, scale, s, p,
                                  o + base + i * d, lse + bh * N + i);
            }
            free(s);
            free(p);
        }
        free(qh); free(kh); free(vh);
    }
    return status;
}

/* Selected rows only: rows[r] = (bh, i) pairs flattened as bh * N + i.  The
 * arithmetic of each row is that of oracle_attention_fwd.  o: nrows x d,
 * lse: nrows. */
int oracle_attention_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          int64_t B, int64_t H, int64_t N, int64_t d, int causal, double scale,
                          const int64_t* rows, int64_t nrows, double* o, double* lse,
                          int threads) {
    if (!q || !k || !v || !rows || !o || !lse || N <= 0 || d <= 0) return -1;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= B * H * N) return -1;
    set_threads(threads);
    int status = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(N + 1));
        double* p = (double*)malloc(sizeof(double) * (size_t)(N + 1));
        double* qr = (double*)malloc(sizeof(double) * (size_t)(d + 1));
        double* kh = (double*)malloc(sizeof(double) * (size_t)(N * d + 1));
        double* vh = (double*)malloc(sizeof(double) * (size_t)(N * d + 1));
        int64_t cached_bh = -1;
        if (!s || !p || !qr || !kh || !vh) {
#pragma omp atomic write
            status = -1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                const int64_t bh = rows[r] / N, i = rows[r] % N;
                if (bh != cached_bh) {
                    widen_slice(k + bh * N * d, kh, N * d);
                    widen_slice(v + bh * N * d, vh, N * d);
                    cached_bh = bh;
                }
                widen_slice(q + (bh * N + i) * d, qr, d);
                attention_row(qr, kh, vh, N, d, i, causal, scale, s, p, o + r * d, lse + r);
            }
        }
        free(s); free(p); free(qr); free(kh); free(vh);
    }
    return status;
}

/* Row-wise softmax of bf16 bits x [rows, cols] (fp64).  y: rows x cols fp64.
 * Returns 0, or -1 on bad arguments. */
int oracle_row_softmax(const uint16_t* x, double* y, int64_t rows, int64_t cols, double scale,
                       int threads) {
    if (!x || !y || rows < 0 || cols <= 0) return -1;
    set_threads(threads);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* xr = x + r * cols;
        double* yr = y + r * cols;
        double m = -INFINITY;
        for (int64_t c = 0; c < cols; ++c) {
            const double v = scale * bf16_to_double(xr[c]);
            if (v > m) m = v;
        }
        double l = 0.0;
        for (int64_t c = 0; c < cols; ++c) l += exp(scale * bf16_to_double(xr[c]) - m);
        for (int64_t c = 0; c < cols; ++c) yr[c] = exp(scale * bf16_to_double(xr[c]) - m) / l;
    }
    return 0;
}
