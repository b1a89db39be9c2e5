/*
 * Seeded synthetic inputs for the attention forward pass and the other kernels
 * of the library: bf16 (or fp32) tensors whose elements are independent
 * N(0, sigma^2) draws.
 *
 * This module holds none of the kernels' arithmetic.  Both the fp64 oracle and the
 * CUDA path read the bytes it writes, so the two see identical inputs.
 *
 * Generator, stated from its published definitions:
 *   - Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *     easy as 1, 2, 3", SC'11): a 4x32-bit counter, a 2x32-bit key, ten rounds
 *     of two 32x32->64 multiplies with the key bumped by the Weyl constants
 *     after each round.
 *       key     = { seed low 32 bits, seed high 32 bits XOR tensor_id }
 *       counter = { element_index / 4 (low 32), (high 32), 0, 0 }
 *     One Philox call yields four 32-bit words, which feed elements
 *     4c .. 4c+3 of the tensor.
 *   - Box-Muller (Box & Muller 1958): words (x0, x1) give two normals
 *       u_i = (x_i + 0.5) / 2^32  in (0, 1)
 *       r   = sqrt(-2 ln u0),  t = 2 pi u1
 *       z0  = r cos t,  z1 = r sin t
 *     and words (x2, x3) give the next two, all in double precision.
 *   - value = sigma * z (double), rounded once, to nearest-even, to bf16.
 *
 * The tensor is written as raw bf16 bit patterns (uint16), row-major, in the
 * order of the flat element index.  seeded_normal_f32 writes the same draws
 * rounded once (nearest-even) to fp32 instead.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void philox_round(uint32_t ctr[4], const uint32_t key[2]) {
    uint64_t p0 = (uint64_t)PHILOX_M0 * ctr[0];
    uint64_t p1 = (uint64_t)PHILOX_M1 * ctr[2];
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ ctr[1] ^ key[0];
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ ctr[3] ^ key[1];
    uint32_t n3 = lo0;
    ctr[0] = n0; ctr[1] = n1; ctr[2] = n2; ctr[3] = n3;
}

/* Philox4x32 with R rounds (R = 10 for the generator proper). */
void seeded_philox4x32(const uint32_t ctr_in[4], const uint32_t key_in[2], int rounds,
                       uint32_t out[4]) {
    uint32_t ctr[4] = {ctr_in[0], ctr_in[1], ctr_in[2], ctr_in[3]};
    uint32_t key[2] = {key_in[0], key_in[1]};
    for (int r = 0; r < rounds; ++r) {
        if (r > 0) { key[0] += PHILOX_W0; key[1] += PHILOX_W1; }
        philox_round(ctr, key);
    }
    memcpy(out, ctr, sizeof(ctr));
}

/* Round a double to the nearest bf16 (ties to even) and return its bit pattern.
 * The quantum of bf16 at |x| in [2^e, 2^(e+1)) is 2^(e-7) (8 significant
 * bits); below the fp32/bf16 normal range the quantum stays 2^-133. */
uint16_t seeded_round_bf16(double x) {
    if (isnan(x)) return 0x7FC0;
    if (isinf(x)) return x > 0 ? 0x7F80 : 0xFF80;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
    int E;
    (void)frexp(x, &E);          /* |x| in [2^(E-1), 2^E) */
    int e = E - 1;
    if (e < -126) e = -126;
    double q = ldexp(1.0, e - 7);
    double r = nearbyint(x / q) * q; /* default rounding mode: ties to even */
    float f = (float)r;              /* exact: r has <= 8 significant bits */
    if (isinf(f)) return f > 0 ? 0x7F80 : 0xFF80;
    uint32_t bits;
    memcpy(&bits, &f, 4);
    return (uint16_t)(bits >> 16);
}

/* The four N(0,1) draws of Philox call c for (seed, tensor_id). */
static void normal4(uint64_t seed, uint32_t tensor_id, int64_t c, double z[4]) {
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_2_32 = 1.0 / 4294967296.0;
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32) ^ tensor_id};
    uint32_t ctr[4] = {(uint32_t)c, (uint32_t)((uint64_t)c >> 32), 0u, 0u};
    uint32_t w[4];
    seeded_philox4x32(ctr, key, 10, w);
    for (int p = 0; p < 2; ++p) {
        double u0 = ((double)w[2 * p] + 0.5) * inv_2_32;
        double u1 = ((double)w[2 * p + 1] + 0.5) * inv_2_32;
        double r = sqrt(-2.0 * log(u0));
        double t = two_pi * u1;
        z[2 * p] = r * cos(t);
        z[2 * p + 1] = r * sin(t);
    }
}

/* Fill out[0 .. n) with fp32(sigma * N(0,1)) for (seed, tensor_id); the same
 * draws as seeded_normal_bf16, rounded to fp32 instead of bf16. */
void seeded_normal_f32(float* out, int64_t n, uint64_t seed, uint32_t tensor_id, double sigma) {
    int64_t ncalls = (n + 3) / 4;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < ncalls; ++c) {
        double z[4];
        normal4(seed, tensor_id, c, z);
        for (int i = 0; i < 4; ++i) {
            int64_t idx = 4 * c + i;
            if (idx < n) out[idx] = (float)(sigma * z[i]);
        }
    }
}

/* Fill out[0 .. n) with bf16(sigma * N(0,1)) for (seed, tensor_id). */
void seeded_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint32_t tensor_id,
                        double sigma) {
    int64_t ncalls = (n + 3) / 4;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < ncalls; ++c) {
        double z[4];
        normal4(seed, tensor_id, c, z);
        for (int i = 0; i < 4; ++i) {
            int64_t idx = 4 * c + i;
            if (idx < n) out[idx] = seeded_round_bf16(sigma * z[i]);
        }
    }
}
