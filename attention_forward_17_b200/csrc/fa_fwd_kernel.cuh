// Fused attention forward pass for sm_100a (B200).
//
// Computes, per (batch, head) slice and query row i,
//   O[i, :] = sum_j softmax_j(scale * q_i . k_j  [j <= i when causal]) v_j
//   LSE[i]  = ln sum_j exp(scale * q_i . k_j)
// without writing the score matrix anywhere: query, key and value tiles are
// streamed through shared memory and the softmax is updated online with a
// running row maximum, a running normaliser and rescaling factors, while both
// products (Q K^T and P V) run on the tensor cores ("TileLang tutorial",
// FlashAttention section).
//
// Blackwell mapping (one CTA = 256 query rows of one (b, h) slice, as two
// 128-row tiles t = 0, 1 processed in ping-pong; 384 threads, and the
// softmax warpgroups take registers from the third warpgroup with setmaxnreg):
//   warp 8      TMA producer: Q tiles once, then K_j / V_j tiles through a
//               ring of shared-memory slots (mbarrier full/empty pairs).
//   warp 9      MMA issuer (one thread): S_t = Q_t K_j^T into tensor memory
//               (TMEM), and O_t += P_t V_j with P_t read from TMEM.
//   warps 0-7   two softmax warpgroups; thread = query row = TMEM lane.  They
//               read S_t from TMEM, apply the causal / length mask, keep the
//               running max m (base-2, scaled) and sum l, rescale O_t in TMEM
//               only when m grows by more than 2^8 (lazy rescale; the final
//               O / l uses the same stale m, so it is exact), write P_t as
//               bf16 into TMEM over S_t, and finally normalise and store O_t
//               and LSE.  O is divided by the sum of the bf16-rounded weights
//               the P V product actually used, so every O row is an exact
//               convex combination of V rows (a one-hot row returns its V row
//               unchanged); LSE uses the fp32 sum of the unrounded weights.
//
// TMEM columns (512 allocated): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D).  P_t (bf16, two per column) sits in the upper half of
// S_t, columns [64,128) of that tile.
//
// Every mbarrier wait is bounded in time.  A wait that gives up records
// FA_ERR_TIMEOUT in the optional status word, marks the CTA as aborted (later
// waits then give up after about a millisecond), and the CTA runs its static
// schedule to the end without hanging; its rows get LSE = NaN.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "ptx.cuh"

namespace fa {

constexpr int kThreads = 384;     // 2 softmax warpgroups + 1 warpgroup (producer, MMA, 2 spare)
constexpr int kBlockM = 128;      // query rows per tile (= TMEM lanes)
constexpr int kBlockN = 128;      // key rows per tile
constexpr int kTilesPerCta = 2;   // ping-pong query tiles
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kStatusTimeout = -7;  // FA_ERR_TIMEOUT
// Per-thread registers after the warpgroups rebalance (launch: 384 x 168).
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsOther = 88;
constexpr int kRegSplitTotal = 2 * 128 * kRegsSoftmax + 128 * kRegsOther;  // 64512 = 384 x 168
// Every kEmuEvery-th pair of exponentials is evaluated on the FMA pipe by
// polynomial instead of on the special-function unit (0 = never).
constexpr int kEmuEvery = 4;
constexpr uint64_t kWaitLimitNs = 2000000000ull;      // 2 s
constexpr uint64_t kWaitLimitAbortNs = 1000000ull;    // 1 ms once the CTA has aborted

template <int D>
struct TileCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int kTileBytes = kBlockM * D * 2;      // one Q, K or V tile (bf16)
    static constexpr int kBoxes = D / 64;                   // 64-column (128-byte) TMA boxes
    static constexpr int kBoxBytes = 128 * 128;             // 128 rows x 128 bytes
    static constexpr int kSlots = (D == 128) ? 4 : 8;       // K/V ring depth
    static constexpr int kQOff = 0;
    static constexpr int kSlotOff = kTilesPerCta * kTileBytes;
    static constexpr int kBarOff = kSlotOff + kSlots * kTileBytes;
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOff + 512;
    __host__ __device__ static constexpr uint32_t col_s(int t) { return 128u * t; }
    __host__ __device__ static constexpr uint32_t col_o(int t) { return 256u + D * t; }
    static constexpr uint32_t kColP = 64;                   // offset of P inside S
    static constexpr uint32_t kTmemCols = 512;
};

template <int kSlots>
struct alignas(8) Barriers {
    uint64_t q_full[2];
    uint64_t kv_full[kSlots];
    uint64_t kv_empty[kSlots];
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t o_full[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    volatile uint32_t abort;
};

struct FwdParams {
    __nv_bfloat16* o;     // [BH, N, D]
    float* lse;           // [BH, N]
    int* status;          // optional device status word (may be null)
    int N;
    int BH;
    int n_qblk;           // ceil(N / 256)
    float scale_log2;     // scale * log2(e)
};

// ---------------------------------------------------------------- bounded waits
__device__ __forceinline__ void wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                       int* status) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return;
        if ((it & 31u) == 0) {
            const uint64_t limit = *abort ? kWaitLimitAbortNs : kWaitLimitNs;
            if (global_timer_ns() - t0 > limit) {
                if (!*abort) {
                    *abort = 1u;
                    if (status) atomicExch(status, kStatusTimeout);
                }
                return;
            }
        }
    }
}

__device__ __forceinline__ void wait_bar(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                         int* status) {
    if (!mbar_try_wait(bar, parity)) wait_slow(bar, parity, abort, status);
}

// ---------------------------------------------------------------- exp2 on the FMA pipe
// 2^x for two values without the special-function unit (Cody-Waite style
// split x = j + f):
//   j = floor(x): add 1.5 * 2^23 rounding toward -inf, so the sum's low
//       mantissa bits hold j; subtract the constant back (exact);
//   f = x - j in [0, 1) (exact);
//   2^f ~ 1 + f (a1 + f (a2 + f a3)), a degree-3 minimax fit in relative
//       error with p(0) = 1 (fit_exp2_poly.py: max relative error 8.6e-5);
//   2^j is applied by adding j << 23 to the bits of 2^f (the low bits of the
//       rounded sum shifted into the exponent field).
// x is clamped to >= -126 so the result stays a normal float (and -inf maps
// to 2^-126, which vanishes next to the row maximum's weight >= 1).
constexpr float kExp2A1 = 0.6951167583465576f;
constexpr float kExp2A2 = 0.22764499485492706f;
constexpr float kExp2A3 = 0.07706703990697861f;

__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const uint64_t x = f2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
    const uint64_t t = add2_rm(x, f2(kMagic, kMagic));
    const uint64_t jf = add2(t, f2(-kMagic, -kMagic));
    const uint64_t fr = fma2(jf, f2(-1.f, -1.f), x);
    uint64_t q = fma2(f2(kExp2A3, kExp2A3), fr, f2(kExp2A2, kExp2A2));
    q = fma2(q, fr, f2(kExp2A1, kExp2A1));
    q = fma2(q, fr, f2(1.f, 1.f));
    float q0, q1, t0, t1;
    f2_split(q, q0, q1);
    f2_split(t, t0, t1);
    y0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
    y1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// ---------------------------------------------------------------- the kernel
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = TileCfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);
    auto* bars = reinterpret_cast<Barriers<C::kSlots>*>(smem + C::kBarOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: CTAs of one (b, h) slice are adjacent in launch order so the
    // slice's K/V stay in L2; under the causal mask the longest q-blocks of a
    // slice launch first.
    const int bh = blockIdx.x / p.n_qblk;
    const int qi = blockIdx.x % p.n_qblk;
    const int qb = CAUSAL ? (p.n_qblk - 1 - qi) : qi;
    const int q0 = qb * (kBlockM * kTilesPerCta);
    const int n_kv_all = (p.N + kBlockN - 1) / kBlockN;
    const int n_kv = CAUSAL ? min(n_kv_all, 2 * qb + 2) : n_kv_all;

    const uint32_t bar_q_full = smem_u32(&bars->q_full[0]);
    const uint32_t bar_kv_full = smem_u32(&bars->kv_full[0]);
    const uint32_t bar_kv_empty = smem_u32(&bars->kv_empty[0]);
    const uint32_t bar_s_full = smem_u32(&bars->s_full[0]);
    const uint32_t bar_p_full = smem_u32(&bars->p_full[0]);
    const uint32_t bar_o_full = smem_u32(&bars->o_full[0]);
    const uint32_t bar_mma_done = smem_u32(&bars->mma_done);
    volatile uint32_t* abort = &bars->abort;

    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_q_full + 8 * t, 1);
            mbar_init(bar_s_full + 8 * t, 1);
            mbar_init(bar_p_full + 8 * t, kBlockM);
            mbar_init(bar_o_full + 8 * t, 1);
        }
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(bar_kv_full + 8 * s, 1);
            mbar_init(bar_kv_empty + 8 * s, 1);
        }
        mbar_init(bar_mma_done, 1);
        bars->abort = 0u;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(smem_u32(&bars->tmem_base), C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp < 8) {
        regs_increase<kRegsSoftmax>();
        // ============================================================ softmax
        const int t = warp >> 2;                  // query tile of this warpgroup
        const int r = threadIdx.x & 127;          // row within the tile = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_off + C::col_s(t);
        const uint32_t t_p = t_s + C::kColP;
        const uint32_t t_o = tmem + lane_off + C::col_o(t);
        const int tile_row0 = q0 + t * kBlockM;
        const int row = tile_row0 + r;
        const float c = p.scale_log2;

        float m_run = -INFINITY;   // running max of scale*log2(e)*s (possibly stale by < 8)
        float l_run = 0.f;         // running sum of 2^(c*s - m_run), fp32 (for LSE)
        float lh_run = 0.f;        // running sum of the same weights rounded to bf16 (for O)

        const uint64_t c2 = f2(c, c);
        for (int j = 0; j < n_kv; ++j) {
            wait_bar(bar_s_full + 8 * t, j & 1, abort, p.status);
            tc_fence_after();
            uint32_t s[4][32];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld32(t_s + 32 * q, s[q]);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 4; ++q) reg_fence32(s[q]);

            const int k0 = j * kBlockN;
            const bool masked = (k0 + kBlockN > p.N) || (CAUSAL && k0 + kBlockN - 1 > tile_row0);
            if (masked) {
                const int lim = (CAUSAL ? min(p.N, row + 1) : p.N) - k0;
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (32 * q + i >= lim) s[q][i] = __float_as_uint(-INFINITY);
            }
            // row max: eight independent 3-input max chains
            float mx[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) mx[a] = __uint_as_float(s[a >> 1][(a & 1) * 16]);
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int q = a >> 1, b0 = (a & 1) * 16;
#pragma unroll
                for (int i = 1; i < 15; i += 2)
                    mx[a] = max3f(mx[a], __uint_as_float(s[q][b0 + i]), __uint_as_float(s[q][b0 + i + 1]));
                mx[a] = fmaxf(mx[a], __uint_as_float(s[q][b0 + 15]));
            }
            const float m_new =
                max3f(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * c;
            const bool grow = m_new > m_run + 8.0f;
            float alpha = 1.f;
            if (grow) {
                alpha = ex2_approx(m_run - m_new);
                m_run = m_new;
                l_run *= alpha;
                lh_run *= alpha;
            }
            if (j > 0 && __any_sync(0xffffffffu, grow)) {
                // O_t holds sum_{j' < j} P V with the old reference max: scale
                // it by 2^(m_old - m_new).  The commit that signalled S_t(j)
                // also covers the P V product of step j-1.
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    tmem_ld32(t_o + 32 * q, o);
                    tmem_wait_ld();
                    reg_fence32(o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(t_o + 32 * q, o);
                }
            }
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
            const uint64_t negm2 = f2(-m_use, -m_use);
            // p = 2^(c*s - m): pairs of columns through packed FMAs; sums of the
            // fp32 weights (l, for LSE) and of their bf16 roundings (for O)
            uint64_t l2a = 0, l2b = 0, h2a = 0, h2b = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int col = 64 * h + 2 * i;
                    const uint64_t x2 = fma2(f2(__uint_as_float(s[col >> 5][col & 31]),
                                                __uint_as_float(s[col >> 5][(col & 31) + 1])),
                                             c2, negm2);
                    float x0, x1;
                    f2_split(x2, x0, x1);
                    float p0, p1;
                    if (kEmuEvery > 0 && (i % kEmuEvery) == kEmuEvery - 1) {
                        exp2_poly2(x0, x1, p0, p1);
                    } else {
                        p0 = ex2_approx(x0);
                        p1 = ex2_approx(x1);
                    }
                    const uint32_t w = pack_bf16x2(p0, p1);
                    const uint64_t pr = f2(p0, p1);
                    const uint64_t ph = f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
                    if (i & 1) {
                        l2b = add2(l2b, pr);
                        h2b = add2(h2b, ph);
                    } else {
                        l2a = add2(l2a, pr);
                        h2a = add2(h2a, ph);
                    }
                    pk[i] = w;
                }
                tmem_st32(t_p + 32 * h, pk);
            }
            float la0, la1, lb0, lb1, ha0, ha1, hb0, hb1;
            f2_split(l2a, la0, la1);
            f2_split(l2b, lb0, lb1);
            f2_split(h2a, ha0, ha1);
            f2_split(h2b, hb0, hb1);
            l_run += (la0 + la1) + (lb0 + lb1);
            lh_run += (ha0 + ha1) + (hb0 + hb1);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar_p_full + 8 * t);
        }

        // ------------------------------------------------------------ epilogue
        wait_bar(bar_o_full + 8 * t, 0, abort, p.status);
        tc_fence_after();
        const bool valid = row < p.N;
        const float inv_l = lh_run > 0.f ? 1.f / lh_run : 0.f;
        __nv_bfloat16* orow = p.o + (static_cast<int64_t>(bh) * p.N + row) * D;
#pragma unroll 1
        for (int q = 0; q < D / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(t_o + 32 * q, o);
            tmem_wait_ld();
            reg_fence32(o);
            if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
                    w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
                    w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
                    w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
                    dst[v] = w;
                }
            }
        }
        if (valid) {
            float lse = l_run > 0.f ? (m_run + lg2_approx(l_run)) * 0.69314718055994531f : -INFINITY;
            if (*abort) lse = __int_as_float(0x7fc00000);
            p.lse[static_cast<int64_t>(bh) * p.N + row] = lse;
        }
    } else if (warp == kProducerWarp) {
        regs_decrease<kRegsOther>();
        // ============================================================ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const uint32_t q_smem = base + C::kQOff;
            const uint32_t slot_smem = base + C::kSlotOff;
            auto load_q = [&](int t) {
                mbar_arrive_expect_tx(bar_q_full + 8 * t, C::kTileBytes);
#pragma unroll
                for (int b = 0; b < C::kBoxes; ++b)
                    tma_load_3d(q_smem + t * C::kTileBytes + b * C::kBoxBytes, &tm_q, 64 * b,
                                q0 + t * kBlockM, bh, bar_q_full + 8 * t, pol_q);
            };
            // load index i: K_{i/2} for even i, V_{i/2} for odd i
            auto load_kv = [&](int i) {
                const int slot = i % C::kSlots;
                const int use = i / C::kSlots;
                if (use > 0) wait_bar(bar_kv_empty + 8 * slot, (use - 1) & 1, abort, p.status);
                const CUtensorMap* map = (i & 1) ? &tm_v : &tm_k;
                mbar_arrive_expect_tx(bar_kv_full + 8 * slot, C::kTileBytes);
#pragma unroll
                for (int b = 0; b < C::kBoxes; ++b)
                    tma_load_3d(slot_smem + slot * C::kTileBytes + b * C::kBoxBytes, map, 64 * b,
                                (i >> 1) * kBlockN, bh, bar_kv_full + 8 * slot, pol_kv);
            };
            load_q(0);
            load_kv(0);
            load_q(1);
            for (int i = 1; i < 2 * n_kv; ++i) load_kv(i);
            // Every load above is waited for by the MMA issuer; in an aborted
            // CTA make sure none is still landing in shared memory at exit.
            if (*abort) {
                for (int i = max(0, 2 * n_kv - C::kSlots); i < 2 * n_kv; ++i)
                    wait_bar(bar_kv_full + 8 * (i % C::kSlots), (i / C::kSlots) & 1, abort, p.status);
                wait_bar(bar_q_full, 0, abort, p.status);
                wait_bar(bar_q_full + 8, 0, abort, p.status);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        regs_decrease<kRegsOther>();
        // ============================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, true);
            const uint32_t q_smem = base + C::kQOff;
            const uint32_t slot_smem = base + C::kSlotOff;
            auto slot_addr = [&](int i) { return slot_smem + (i % C::kSlots) * C::kTileBytes; };
            auto wait_kv = [&](int i) {
                wait_bar(bar_kv_full + 8 * (i % C::kSlots), (i / C::kSlots) & 1, abort, p.status);
                tc_fence_after();
            };
            // Descriptors are built once; the start-address field (bits 0..13,
            // address >> 4) is advanced by plain integer adds, which never carry
            // out of the field for shared-memory addresses below 256 KiB.  This
            // keeps the issuing thread's instruction count per MMA minimal.
            const uint64_t desc_k = smem_desc_sw128(0, 16, 1024);
            const uint64_t desc_v = smem_desc_sw128(0, C::kBoxBytes, 1024);
            const uint64_t desc_q0 = desc_k + (q_smem >> 4);
            const uint64_t desc_q1 = desc_k + ((q_smem + C::kTileBytes) >> 4);
            // S_t = Q_t K^T: K-major A and B, 128-byte swizzle, 16 columns of d per MMA.
            auto issue_s = [&](int t, uint32_t k_smem) {
                const uint64_t a0 = t ? desc_q1 : desc_q0;
                const uint64_t b0 = desc_k + (k_smem >> 4);
                const uint32_t d_tmem = tmem + C::col_s(t);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                    mma_ss(d_tmem, a0 + off, b0 + off, idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // O_t += P_t V: P_t from TMEM (8 columns per 16 keys); V is MN-major
            // (d contiguous): 8-key groups 1024 bytes apart, 64-column halves
            // of d one box (16 KiB) apart; 16 keys = 2048 bytes per MMA.
            auto issue_pv = [&](int t, uint32_t v_smem, bool acc) {
                const uint64_t b0 = desc_v + (v_smem >> 4);
                const uint32_t d_tmem = tmem + C::col_o(t);
                const uint32_t a_tmem = tmem + C::col_s(t) + C::kColP;
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk)
                    mma_ts(d_tmem, a_tmem + kk * 8, b0 + kk * (2048 >> 4), idesc_o,
                           (acc || kk > 0) ? 1u : 0u);
            };

            wait_bar(bar_q_full, 0, abort, p.status);
            wait_kv(0);
            issue_s(0, slot_addr(0));
            mma_commit(bar_s_full);
            wait_bar(bar_q_full + 8, 0, abort, p.status);
            tc_fence_after();
            issue_s(1, slot_addr(0));
            mma_commit(bar_s_full + 8);
            mma_commit(bar_kv_empty + 8 * (0 % C::kSlots));
            for (int j = 0; j < n_kv; ++j) {
                const int iv = 2 * j + 1, ik = 2 * j + 2;
                const bool more = j + 1 < n_kv;
                wait_kv(iv);
                wait_bar(bar_p_full, j & 1, abort, p.status);
                tc_fence_after();
                issue_pv(0, slot_addr(iv), j > 0);
                if (more) {
                    wait_kv(ik);
                    issue_s(0, slot_addr(ik));
                    mma_commit(bar_s_full);
                } else {
                    mma_commit(bar_o_full);
                }
                wait_bar(bar_p_full + 8, j & 1, abort, p.status);
                tc_fence_after();
                issue_pv(1, slot_addr(iv), j > 0);
                mma_commit(bar_kv_empty + 8 * (iv % C::kSlots));
                if (more) {
                    issue_s(1, slot_addr(ik));
                    mma_commit(bar_s_full + 8);
                    mma_commit(bar_kv_empty + 8 * (ik % C::kSlots));
                } else {
                    mma_commit(bar_o_full + 8);
                }
            }
            mma_commit(bar_mma_done);
            wait_bar(bar_mma_done, 0, abort, p.status);
        }
        __syncwarp();
    } else {
        regs_decrease<kRegsOther>();   // spare warps of the third warpgroup
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
