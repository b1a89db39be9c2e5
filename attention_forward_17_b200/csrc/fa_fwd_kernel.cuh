// Fused attention forward pass for sm_100a (B200).
//
// Computes, per (batch, head) slice and query row i,
//   O[i, :] = sum_j softmax_j(scale * q_i . k_j  [j <= i when causal]) v_j
//   LSE[i]  = ln sum_j exp(scale * q_i . k_j)
// without writing the score matrix anywhere: query, key and value tiles are
// streamed through on-chip memory and the softmax is updated online with a
// running row maximum, a running normaliser and rescaling factors, while both
// products (Q K^T and P V) run on the tensor cores ("TileLang tutorial",
// FlashAttention section).
//
// Blackwell mapping.  A CTA works on 128-row query tiles of (b, h) slices,
// one per CTA or, in the persistent launch, several in turn (TileCursor);
// 384 threads in three warpgroups:
//   warpgroups 0 and 1  softmax.  Each warp owns 16 query rows (TMEM lanes
//               32*quarter + 16*g ..) through the 16-lane TMEM access shapes; a
//               row's 128 scores sit in four adjacent threads, so row maxima
//               need two shuffles and the eight softmax warps run without any
//               barrier between them.
//   warp 8      TMA producer: the Q tile once, then K_j and V_j tiles through
//               one ring of shared-memory slots (mbarrier full/empty pairs).
//   warp 9      score issuer (one thread): S_b = Q K_j^T on tcgen05, Q and K_j
//               from shared memory, S_b into tensor memory (TMEM).
//   warp 10     output issuer (one thread): O += P_b V_j on tcgen05, P_b from
//               TMEM, V_j from shared memory.
//               A thread issues one tcgen05.mma about every 48 cycles while a
//               128x128x16 product takes 64 on the tensor pipe, so one issuing
//               thread alone leaves the pipe idle; two keep it fed.
//               The score tile is triple-buffered (b = j mod 3): S for steps
//               j+1 and j+2 is computed while the softmax works on step j, and
//               buffer b is rewritten only after the product that read its P
//               has completed.
// The softmax keeps the running max m (base 2, scaled) and sums l; O is
// rescaled in TMEM only when m grows by more than 2^8 (lazy rescale: the final
// O / l uses the same stale m, so it is exact).  O is divided by the sum of the
// bf16-rounded weights the P V product actually used, so every O row is an
// exact convex combination of V rows; LSE uses the fp32 sum of the unrounded
// weights.  A share of the exponentials runs on the FMA pipe (exp2_poly2).
//
// TMEM columns (512 allocated): S_0 [0,128), S_1 [128,256), S_2 [256,384),
// O [384, 384+D).  P_b (bf16, two per column) sits in columns [64,128) of S_b:
// keys 0-63 then keys 64-127.
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

constexpr int kThreads = 384;     // 2 softmax warpgroups + producer, 2 MMA issuers, 1 spare
constexpr int kSBufs = 3;         // score / probability buffers in TMEM
constexpr int kBlockM = 128;      // query rows per CTA (= TMEM lanes)
constexpr int kBlockN = 128;      // key rows per tile
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;       // score issuer; also allocates TMEM
constexpr int kPvWarp = 10;       // output issuer
constexpr int kStatusTimeout = -7;  // FA_ERR_TIMEOUT
constexpr uint64_t kWaitLimitNs = 2000000000ull;      // 2 s
constexpr uint64_t kWaitLimitAbortNs = 1000000ull;    // 1 ms once the CTA has aborted
// Per-thread registers after the warpgroups rebalance (launch: 384 x 168).
constexpr uint32_t kRegsSoftmax = 208;
constexpr uint32_t kRegsOther = 88;
constexpr int kRegSplitTotal = 2 * 128 * kRegsSoftmax + 128 * kRegsOther;  // 64512 = 384 x 168

// Schedule knobs (template parameters of the kernel, chosen per problem by
// the host from a table the schedule search writes):
//   EMU    every EMU-th pair of exponentials is evaluated on the FMA pipe by
//          polynomial instead of on the special-function unit (0 = never);
//   SLOTS  depth of the K/V shared-memory ring.
template <int D, int SLOTS>
struct TileCfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    // A parity wait on a ring slot is only sound if the slot's previous load
    // has already landed when the wait starts (else the wait can mistake that
    // older phase for the one it wants).  The score issuer waits K_m after
    // PV(m-3) completed and the output issuer waits V_t after P_t, which
    // cover every earlier load that can share the slot once the ring holds
    // at least four tiles: V_t (sequence position 2t+3) then shares a slot
    // with V_{t'<t} or K_{m<=t} only.  With three slots V_t would share K_{t+1}'s.
    static_assert(SLOTS >= 4, "K/V ring depth");
    static constexpr int kTileBytes = kBlockN * D * 2;      // one K or V tile (bf16)
    static constexpr int kBoxes = D / 64;                   // 64-column (128-byte) TMA boxes
    static constexpr int kBoxBytes = 128 * 128;             // 128 rows x 128 bytes
    static constexpr int kSlots = SLOTS;                    // K/V ring depth
    static constexpr int kQOff = 0;
    static constexpr int kSlotOff = kTileBytes;             // after the Q tile
    static constexpr int kBarOff = kSlotOff + kSlots * kTileBytes;
    static constexpr int kRedOff = kBarOff + 512;           // row-max / sum exchange
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + kRedOff + 4 * 2 * 128 * 4;
    __host__ __device__ static constexpr uint32_t col_s(int b) { return 128u * b; }
    static constexpr uint32_t kColO = 128 * kSBufs;
    static constexpr uint32_t kColP = 64;                   // offset of P inside S_b
    static constexpr uint32_t kTmemCols = 512;
};

template <int kSlots>
struct alignas(16) Barriers {
    uint32_t clc_resp[2][4];    // cluster-launch-control responses (16-byte aligned)
    uint64_t kv_full[kSlots];
    uint64_t kv_empty[kSlots];
    uint64_t q_full;            // Q tile landed in shared memory
    uint64_t q_empty;           // every score product of the current tile done (Q reusable)
    uint64_t s_full[kSBufs];    // S_b computed
    uint64_t p_full[kSBufs];    // P_b written (and O rescaled)
    uint64_t pv_done[kSBufs];   // O += P_b V of the latest use of buffer b completed
    uint64_t o_full;            // every product of the current tile done
    uint64_t o_empty;           // the epilogue has read O out of TMEM
    uint64_t clc_full[2];       // response of a cancellation request landed
    uint64_t clc_empty[2];      // every role has read that response
    uint32_t tmem_base;
    volatile uint32_t abort;
};

struct FwdParams {
    __nv_bfloat16* o;        // [BH, N, D]
    float* lse;              // [BH, N]
    int* status;             // optional device status word (may be null)
    int N;
    int BH;
    int n_qtile;             // ceil(N / 128)
    int group;               // causal launch order: heads per group (>= 1)
    float scale_log2;        // scale * log2(e)
    // optional (may be null): [0] += (warp, key tile) steps that rescaled O,
    // [1] += (row, key tile) rescales; counted by the two-query-tile kernel
    unsigned long long* rescale_stats;
};

// Load sequence of the K/V ring: K_0 .. K_{min(3,n)-1}, then for each step t
// V_t followed by K_{t+3} (while t + 3 < n).  Each load's slot is released by
// the issuer that consumes it; a release only ever depends on loads earlier in
// the sequence, so the ring cannot deadlock.
__device__ __forceinline__ int load_index_k(int m) { return m < kSBufs ? m : 2 * m - kSBufs + 1; }
__device__ __forceinline__ int load_index_v(int t, int n) {
    return min(kSBufs, n) + t + min(t, max(0, n - kSBufs));
}

// ---------------------------------------------------------------- bounded waits
// Polls the mbarrier phase until it completes or `limit_ns` (globaltimer)
// passes; on time-out marks the CTA aborted and records FA_ERR_TIMEOUT.  Once
// aborted, further waits give up after `limit_abort_ns`.
__device__ __forceinline__ void wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
                                          int* status, uint64_t limit_ns, uint64_t limit_abort_ns) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return;
        if ((it & 31u) == 0) {
            const uint64_t limit = *abort ? limit_abort_ns : limit_ns;
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
    if (!mbar_try_wait(bar, parity))
        wait_slow(bar, parity, abort, status, kWaitLimitNs, kWaitLimitAbortNs);
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
// The query tiles one CTA processes, in order.
//   PERSIST = 0: one tile per CTA.  Without the mask, the CTAs of one (b, h)
//     slice are adjacent in launch order so the slice's K/V stay in L2.  Under
//     the causal mask the slices are taken `group` at a time and, inside a
//     group, query tiles launch longest first (all the group's last tiles,
//     then the tiles before them, ...), which keeps the group's K/V in L2
//     while the short tiles fill the end of the grid.
//   PERSIST = 1: one CTA per SM walks several tiles, so one tile's epilogue
//     and the next tile's Q load and first score products overlap instead of
//     paying a CTA launch, barrier set-up and TMEM allocation per tile.
//     Without the mask: tiles blockIdx.x, +gridDim.x, ... in (b, h)-major
//     order.  Under the mask: units of two tiles of one slice, qt = n-1-k then
//     qt = k (one tile when they coincide), so every unit holds n+1 key tiles
//     of work and a plain round-robin of units balances the CTAs.
//   PERSIST = 2: the grid and tile order of PERSIST = 0, but a CTA that is
//     about to finish a tile asks the scheduler (cluster launch control) to
//     cancel the next CTA that has not launched yet and takes over its tile,
//     so tiles overlap as in PERSIST = 1 while the hardware's launch order and
//     dynamic balance are kept.  The producer issues the request; every role
//     reads the response from one of two shared-memory slots (full / empty
//     mbarriers).  After the first refusal no further request is made.
template <bool CAUSAL>
__device__ __forceinline__ void map_tile(const FwdParams& p, int id, int& bh, int& qt) {
    if constexpr (CAUSAL) {
        const int span = p.group * p.n_qtile;
        const int g0 = (id / span) * p.group;
        const int heads = min(p.group, p.BH - g0);
        const int rr = id % span;
        bh = g0 + rr % heads;
        qt = p.n_qtile - 1 - rr / heads;
    } else {
        bh = id / p.n_qtile;
        qt = id % p.n_qtile;
    }
}

constexpr int kClcReaders = 11;   // 8 softmax warps, producer, two MMA issuers

template <bool CAUSAL, int PERSIST>
struct TileCursor {
    int r = 0;      // tiles handed out so far
    int half = 0;   // PERSIST 1, causal: 0 = long tile of the unit next, 1 = short tile next
    bool done = false;
    // PERSIST 2
    uint32_t resp = 0, full = 0, empty = 0;   // slot 0 addresses (slot 1: +16 / +8 / +8)
    volatile uint32_t* abort = nullptr;
    int* status = nullptr;

    // The producer's request for the tile after the current one.
    __device__ __forceinline__ void request() {
        if constexpr (PERSIST == 2) {
            if (done || *abort) {
                done = true;
                return;
            }
            const int q = r - 1, slot = q & 1, use = q >> 1;
            if (use > 0) wait_bar(empty + 8 * slot, (use - 1) & 1, abort, status);
            mbar_arrive_expect_tx(full + 8 * slot, 16);
            clc_try_cancel(resp + 16 * slot, full + 8 * slot);
        }
    }

    // WARP: called by all 32 lanes of a warp (one arrival for the warp).
    template <bool WARP>
    __device__ __forceinline__ bool next(const FwdParams& p, int& bh, int& qt) {
        if constexpr (PERSIST == 0) {
            if (r++ > 0) return false;
            map_tile<CAUSAL>(p, blockIdx.x, bh, qt);
            return true;
        } else if constexpr (PERSIST == 2) {
            if (r == 0) {
                ++r;
                map_tile<CAUSAL>(p, blockIdx.x, bh, qt);
                return true;
            }
            if (done) return false;
            const int q = r - 1, slot = q & 1, use = q >> 1;
            const uint32_t fb = full + 8 * slot;
            wait_bar(fb, use & 1, abort, status);
            uint32_t x = 0;
            const bool got = mbar_try_wait(fb, use & 1) && clc_query(resp + 16 * slot, x);
            if constexpr (WARP) {
                __syncwarp();
                if ((threadIdx.x & 31) == 0) mbar_arrive(empty + 8 * slot);
            } else {
                mbar_arrive(empty + 8 * slot);
            }
            if (!got || static_cast<int64_t>(x) >= static_cast<int64_t>(p.BH) * p.n_qtile) {
                done = true;
                return false;
            }
            ++r;
            map_tile<CAUSAL>(p, static_cast<int>(x), bh, qt);
            return true;
        } else if constexpr (!CAUSAL) {
            const int64_t i = blockIdx.x + static_cast<int64_t>(r) * gridDim.x;
            if (i >= static_cast<int64_t>(p.BH) * p.n_qtile) return false;
            ++r;
            bh = static_cast<int>(i / p.n_qtile);
            qt = static_cast<int>(i % p.n_qtile);
            return true;
        } else {
            const int units = (p.n_qtile + 1) / 2;
            const int64_t u = blockIdx.x + static_cast<int64_t>(r) * gridDim.x;
            if (u >= static_cast<int64_t>(p.BH) * units) return false;
            bh = static_cast<int>(u / units);
            const int k = static_cast<int>(u % units);
            const int hi = p.n_qtile - 1 - k;
            if (half == 0) {
                qt = hi;
                if (hi == k) ++r;       // the middle tile of an odd count stands alone
                else half = 1;
            } else {
                qt = k;
                half = 0;
                ++r;
            }
            return true;
        }
    }
};

template <int D, bool CAUSAL, int EMU, int SLOTS, int PERSIST>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = TileCfg<D, SLOTS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);
    auto* bars = reinterpret_cast<Barriers<C::kSlots>*>(smem + C::kBarOff);
    // final per-row statistics handed to the epilogue: m [0,128), l [128,256), l-hat [256,384)
    float* red = reinterpret_cast<float*>(smem + C::kRedOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int n_kv_all = (p.N + kBlockN - 1) / kBlockN;
    // keys of query tile qt: all tiles, or up to the diagonal under the mask
    const auto kv_tiles = [&](int qt) { return CAUSAL ? min(n_kv_all, qt + 1) : n_kv_all; };

    const uint32_t bar_kv_full = smem_u32(&bars->kv_full[0]);
    const uint32_t bar_kv_empty = smem_u32(&bars->kv_empty[0]);
    const uint32_t bar_q_full = smem_u32(&bars->q_full);
    const uint32_t bar_q_empty = smem_u32(&bars->q_empty);
    const uint32_t bar_s_full = smem_u32(&bars->s_full[0]);
    const uint32_t bar_p_full = smem_u32(&bars->p_full[0]);
    const uint32_t bar_pv_done = smem_u32(&bars->pv_done[0]);
    const uint32_t bar_o_full = smem_u32(&bars->o_full);
    const uint32_t bar_o_empty = smem_u32(&bars->o_empty);
    volatile uint32_t* abort = &bars->abort;
    const auto make_cursor = [&]() {
        TileCursor<CAUSAL, PERSIST> c;
        c.resp = smem_u32(&bars->clc_resp[0][0]);
        c.full = smem_u32(&bars->clc_full[0]);
        c.empty = smem_u32(&bars->clc_empty[0]);
        c.abort = abort;
        c.status = p.status;
        return c;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(bar_kv_full + 8 * s, 1);
            mbar_init(bar_kv_empty + 8 * s, 1);
        }
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 1);
        for (int b = 0; b < kSBufs; ++b) {
            mbar_init(bar_s_full + 8 * b, 1);
            mbar_init(bar_p_full + 8 * b, 256);
            mbar_init(bar_pv_done + 8 * b, 1);
        }
        mbar_init(bar_o_full, 1);
        mbar_init(bar_o_empty, 256);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&bars->clc_full[i]), 1);
            mbar_init(smem_u32(&bars->clc_empty[i]), kClcReaders);
        }
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

    // Every role walks the same tile sequence (TileCursor).  Across tiles the
    // score buffers and their barriers are indexed by a global step count
    // (gs), the K/V ring by a global load count (lb = loads of earlier
    // tiles), and the per-tile barriers (Q, O) by the tile count.
    if (warp < 8) {
        regs_increase<kRegsSoftmax>();
        // ============================================================ softmax
        // Warp (g, quarter) owns the 16 tile rows L .. L+15, L = 32*quarter +
        // 16*g, through the 16-lane TMEM access shapes: thread t holds rows
        // ra = L + t/4 and rb = ra + 8, keys 8m + 2(t%4) + {0,1} (m = 0..15) of
        // each score tile, so a row's 128 keys live in four adjacent threads.
        const int quarter = warp & 3;
        const int g = warp >> 2;
        const int L = 32 * quarter + 16 * g;
        const int ra = L + (lane >> 2), rb = ra + 8;
        const int kq = 2 * (lane & 3);            // key offset inside each 8-key chunk
        const uint32_t lane_w = static_cast<uint32_t>(L) << 16;
        const float c = p.scale_log2;
        const uint64_t c2 = f2(c, c);
        auto cur = make_cursor();
        int bh, qt, gs = 0, tile = 0;
        while (cur.template next<true>(p, bh, qt)) {
        const int q0 = qt * kBlockM;
        const int n_kv = kv_tiles(qt);
        float m_a = -INFINITY, m_b = -INFINITY;   // running max of c*s per row (stale by < 8)
        float l_a = 0.f, l_b = 0.f;               // fp32 sums of 2^(c*s - m) (for LSE), this thread's keys
        float lh_a = 0.f, lh_b = 0.f;             // the same weights rounded to bf16 (for O)

            for (int j = 0; j < n_kv; ++j) {
                const int gj = gs + j;                // global step: buffer and phase
                const int bb = gj % kSBufs;
                const uint32_t t_s = tmem + lane_w + C::col_s(bb);
                wait_bar(bar_s_full + 8 * bb, (gj / kSBufs) & 1, abort, p.status);
                tc_fence_after();
                uint32_t s[64];
                tmem_ld16x256b_x16(t_s, s);
                tmem_wait_ld();
                reg_fence64(s);

                const bool masked =
                    (j * kBlockN + kBlockN > p.N) || (CAUSAL && j * kBlockN + kBlockN - 1 > q0);
                if (masked) {
                    const int lim_a = (CAUSAL ? min(p.N, q0 + ra + 1) : p.N) - j * kBlockN;
                    const int lim_b = (CAUSAL ? min(p.N, q0 + rb + 1) : p.N) - j * kBlockN;
    #pragma unroll
                    for (int m = 0; m < 16; ++m)
    #pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int key = 8 * m + kq + e;
                            if (key >= lim_a) s[4 * m + e] = __float_as_uint(-INFINITY);
                            if (key >= lim_b) s[4 * m + 2 + e] = __float_as_uint(-INFINITY);
                        }
                }
                // row maxima: 32 values per row in this thread, then across the 4 threads
                float xa0 = fmaxf(__uint_as_float(s[0]), __uint_as_float(s[1]));
                float xb0 = fmaxf(__uint_as_float(s[2]), __uint_as_float(s[3]));
                float xa1 = fmaxf(__uint_as_float(s[4]), __uint_as_float(s[5]));
                float xb1 = fmaxf(__uint_as_float(s[6]), __uint_as_float(s[7]));
    #pragma unroll
                for (int m = 2; m < 16; m += 2) {
                    xa0 = max3f(xa0, __uint_as_float(s[4 * m]), __uint_as_float(s[4 * m + 1]));
                    xb0 = max3f(xb0, __uint_as_float(s[4 * m + 2]), __uint_as_float(s[4 * m + 3]));
                    xa1 = max3f(xa1, __uint_as_float(s[4 * m + 4]), __uint_as_float(s[4 * m + 5]));
                    xb1 = max3f(xb1, __uint_as_float(s[4 * m + 6]), __uint_as_float(s[4 * m + 7]));
                }
                float mxa = fmaxf(xa0, xa1), mxb = fmaxf(xb0, xb1);
                mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
                mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
                mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
                mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
                const float mna = mxa * c, mnb = mxb * c;
                const bool ga = mna > m_a + 8.0f, gb = mnb > m_b + 8.0f;
                float alpha_a = 1.f, alpha_b = 1.f;
                if (ga) {
                    alpha_a = ex2_approx(m_a - mna);
                    m_a = mna;
                    l_a *= alpha_a;
                    lh_a *= alpha_a;
                }
                if (gb) {
                    alpha_b = ex2_approx(m_b - mnb);
                    m_b = mnb;
                    l_b *= alpha_b;
                    lh_b *= alpha_b;
                }
                if (j > 0 && __any_sync(0xffffffffu, ga || gb)) {
                    // O holds sum_{j' < j} P V with the old reference maxima: scale
                    // these 16 rows by 2^(m_old - m_new) once the product of step
                    // j-1 has landed.
                    wait_bar(bar_pv_done + 8 * ((gj - 1) % kSBufs), ((gj - 1) / kSBufs) & 1, abort,
                             p.status);
                    tc_fence_after();
                    const uint32_t t_o = tmem + lane_w + C::kColO;
                    if constexpr (D == 128) {
                        uint32_t o[64];
                        tmem_ld16x256b_x16(t_o, o);
                        tmem_wait_ld();
                        reg_fence64(o);
    #pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            o[4 * m] = __float_as_uint(__uint_as_float(o[4 * m]) * alpha_a);
                            o[4 * m + 1] = __float_as_uint(__uint_as_float(o[4 * m + 1]) * alpha_a);
                            o[4 * m + 2] = __float_as_uint(__uint_as_float(o[4 * m + 2]) * alpha_b);
                            o[4 * m + 3] = __float_as_uint(__uint_as_float(o[4 * m + 3]) * alpha_b);
                        }
                        reg_fence64(o);
                        tmem_st16x256b_x16(t_o, o);
                    } else {
                        uint32_t o[32];
                        tmem_ld16x256b_x8(t_o, o);
                        tmem_wait_ld();
                        reg_fence32(o);
    #pragma unroll
                        for (int m = 0; m < 8; ++m) {
                            o[4 * m] = __float_as_uint(__uint_as_float(o[4 * m]) * alpha_a);
                            o[4 * m + 1] = __float_as_uint(__uint_as_float(o[4 * m + 1]) * alpha_a);
                            o[4 * m + 2] = __float_as_uint(__uint_as_float(o[4 * m + 2]) * alpha_b);
                            o[4 * m + 3] = __float_as_uint(__uint_as_float(o[4 * m + 3]) * alpha_b);
                        }
                        reg_fence32(o);
                        tmem_st16x256b_x8(t_o, o);
                    }
                }
                const float ua = (m_a == -INFINITY) ? 0.f : m_a;
                const float ub = (m_b == -INFINITY) ? 0.f : m_b;
                const uint64_t nega = f2(-ua, -ua), negb = f2(-ub, -ub);
                // p = 2^(c*s - m) pairwise through packed FMAs; sums of the fp32
                // weights (for LSE) and of their bf16 roundings (for O).  P word
                // 2m / 2m+1 = keys 8m + kq + {0,1} of row a / row b, which is the
                // 16x128b store layout at column 4m + t%4 of the P region.
                uint64_t la2 = 0, lb2 = 0, ha2 = 0, hb2 = 0;
                uint32_t pk[32];
                // The exponentials of the tile are evaluated in three passes:
                // pass 1, exponents c*s - m, in place
    #pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int m = i >> 1;
                    const int o = 4 * m + 2 * (i & 1);
                    const uint64_t x2 = fma2(f2(__uint_as_float(s[o]), __uint_as_float(s[o + 1])), c2,
                                             (i & 1) ? negb : nega);
                    float x0, x1;
                    f2_split(x2, x0, x1);
                    s[o] = __float_as_uint(x0);
                    s[o + 1] = __float_as_uint(x1);
                }
                // pass 2: exponentials in place
    #pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int o = 4 * (i >> 1) + 2 * (i & 1);
                    float p0, p1;
                    if (EMU > 0 && (i % (EMU > 0 ? EMU : 1)) == EMU - 1) {
                        exp2_poly2(__uint_as_float(s[o]), __uint_as_float(s[o + 1]), p0, p1);
                    } else {
                        p0 = ex2_approx(__uint_as_float(s[o]));
                        p1 = ex2_approx(__uint_as_float(s[o + 1]));
                    }
                    s[o] = __float_as_uint(p0);
                    s[o + 1] = __float_as_uint(p1);
                }
                // pass 3: bf16 pairs and the two sums
    #pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int o = 4 * (i >> 1) + 2 * (i & 1);
                    const float p0 = __uint_as_float(s[o]), p1 = __uint_as_float(s[o + 1]);
                    const uint32_t w = pack_bf16x2(p0, p1);
                    const uint64_t pr = f2(p0, p1);
                    const uint64_t ph = f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
                    if (i & 1) {
                        lb2 = add2(lb2, pr);
                        hb2 = add2(hb2, ph);
                    } else {
                        la2 = add2(la2, pr);
                        ha2 = add2(ha2, ph);
                    }
                    pk[i] = w;
                }
                // The TMEM store is an asm statement with register inputs, and
                // neither it nor tcgen05.wait::st below tells the compiler that the
                // hardware may still read those registers after the statement
                // issues.  The fences make the packed words fully computed before
                // the store and keep their registers unreused until the wait
                // (without them the multi-pass form above stored stale score
                // values on sm_100a).  They emit no instruction.
                reg_fence32(pk);
                tmem_st16x128b_x16(t_s + C::kColP, pk);
                float u0, u1;
                f2_split(la2, u0, u1);
                l_a += u0 + u1;
                f2_split(lb2, u0, u1);
                l_b += u0 + u1;
                f2_split(ha2, u0, u1);
                lh_a += u0 + u1;
                f2_split(hb2, u0, u1);
                lh_b += u0 + u1;
                tmem_wait_st();
                reg_fence32(pk);
                tc_fence_before();
                mbar_arrive(bar_p_full + 8 * bb);
            }
        gs += n_kv;

        // ------------------------------------------------------------ epilogue
        // Row totals over the four threads of each row, published per tile row
        // for the 32-lane epilogue layout (thread = row); the exchange buffer
        // alternates between tiles so a fast warp cannot overwrite values a
        // slower partner warp has not read yet.
#pragma unroll
        for (int sh = 1; sh <= 2; sh <<= 1) {
            l_a += __shfl_xor_sync(0xffffffffu, l_a, sh);
            l_b += __shfl_xor_sync(0xffffffffu, l_b, sh);
            lh_a += __shfl_xor_sync(0xffffffffu, lh_a, sh);
            lh_b += __shfl_xor_sync(0xffffffffu, lh_b, sh);
        }
        float* rt = red + 384 * (tile & 1);
        if ((lane & 3) == 0) {
            rt[ra] = m_a;
            rt[128 + ra] = l_a;
            rt[256 + ra] = lh_a;
            rt[rb] = m_b;
            rt[128 + rb] = l_b;
            rt[256 + rb] = lh_b;
        }
        named_barrier_sync(1 + quarter, 64);
        const int r = 32 * quarter + lane;        // epilogue row of this thread
        const int row = q0 + r;
        const float m_r = rt[r], l_r = rt[128 + r], lh_r = rt[256 + r];
        wait_bar(bar_o_full, tile & 1, abort, p.status);
        tc_fence_after();
        // this thread's half of the O row, out of TMEM before anything else so
        // the next tile's first P V product can overwrite O
        const uint32_t t_o =
            tmem + (static_cast<uint32_t>(32 * quarter) << 16) + C::kColO + g * (D / 2);
        uint32_t o0[32], o1[32];
        tmem_ld32(t_o, o0);
        if constexpr (D == 128) tmem_ld32(t_o + 32, o1);
        tmem_wait_ld();
        reg_fence32(o0);
        if constexpr (D == 128) reg_fence32(o1);
        tc_fence_before();
        mbar_arrive(bar_o_empty);
        const bool valid = row < p.N;
        const float inv_l = lh_r > 0.f ? 1.f / lh_r : 0.f;
        __nv_bfloat16* orow = p.o + (static_cast<int64_t>(bh) * p.N + row) * D + g * (D / 2);
        const auto store32 = [&](const uint32_t (&o)[32], int col) {
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
                w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
                w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
                w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
                dst[v] = w;
            }
        };
        if (valid) {
            store32(o0, 0);
            if constexpr (D == 128) store32(o1, 32);
        }
        if (valid && g == 0) {
            float lse = l_r > 0.f ? (m_r + lg2_approx(l_r)) * 0.69314718055994531f : -INFINITY;
            if (*abort) lse = __int_as_float(0x7fc00000);
            p.lse[static_cast<int64_t>(bh) * p.N + row] = lse;
        }
        ++tile;
        if (*abort) break;
        }
    } else if (warp == kProducerWarp) {
        regs_decrease<kRegsOther>();
        // ============================================================ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const uint32_t slot_smem = base + C::kSlotOff;
            int i = 0, tile = 0;
            auto load = [&](bool is_v, int kv_tile, int bh) {
                const int slot = i % C::kSlots;
                const int use = i / C::kSlots;
                if (use > 0) wait_bar(bar_kv_empty + 8 * slot, (use - 1) & 1, abort, p.status);
                const CUtensorMap* map = is_v ? &tm_v : &tm_k;
                mbar_arrive_expect_tx(bar_kv_full + 8 * slot, C::kTileBytes);
#pragma unroll
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_3d(slot_smem + slot * C::kTileBytes + bx * C::kBoxBytes, map, 64 * bx,
                                kv_tile * kBlockN, bh, bar_kv_full + 8 * slot, pol_kv);
                ++i;
            };
            auto cur = make_cursor();
            int bh, qt;
            while (cur.template next<false>(p, bh, qt)) {
                const int n_kv = kv_tiles(qt);
                // the Q buffer is free once every score product of the previous tile is done
                if (tile > 0) wait_bar(bar_q_empty, (tile - 1) & 1, abort, p.status);
                mbar_arrive_expect_tx(bar_q_full, C::kTileBytes);
#pragma unroll
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_3d(base + C::kQOff + bx * C::kBoxBytes, &tm_q, 64 * bx, qt * kBlockM, bh,
                                bar_q_full, pol_q);
                for (int m = 0; m < kSBufs && m < n_kv; ++m) load(false, m, bh);
                for (int t = 0; t < n_kv; ++t) {
                    load(true, t, bh);
                    if (t + kSBufs < n_kv) load(false, t + kSBufs, bh);
                }
                // PERSIST 2: claim the next tile now that this one's loads are queued
                // (after an abort the request is skipped and the cursor ends)
                cur.request();
                ++tile;
                if (PERSIST != 2 && *abort) break;
            }
            // Every load above is waited for by an MMA issuer; in an aborted
            // CTA make sure none is still landing in shared memory at exit.
            if (*abort) {
                for (int k = max(0, i - C::kSlots); k < i; ++k)
                    wait_bar(bar_kv_full + 8 * (k % C::kSlots), (k / C::kSlots) & 1, abort, p.status);
                if (tile > 0) wait_bar(bar_q_full, (tile - 1) & 1, abort, p.status);
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp || warp == kPvWarp) {
        regs_decrease<kRegsOther>();
        if (lane == 0) {
            const uint32_t slot_smem = base + C::kSlotOff;
            auto slot_addr = [&](int i) { return slot_smem + (i % C::kSlots) * C::kTileBytes; };
            auto wait_kv = [&](int i) {
                wait_bar(bar_kv_full + 8 * (i % C::kSlots), (i / C::kSlots) & 1, abort, p.status);
                tc_fence_after();
            };
            auto cur = make_cursor();
            int bh, qt, gs = 0, lb = 0, tile = 0;
            // Descriptors are built once; the start-address field (bits 0..13,
            // address >> 4) is advanced by plain integer adds, which never carry
            // out of the field for shared-memory addresses below 256 KiB.
            if (warp == kMmaWarp) {
                // ==================================================== score issuer
                // S_b = Q K^T: Q and K K-major in shared memory, 128-byte
                // swizzle, 16 columns of d per MMA.
                constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false);
                const uint64_t desc_k = smem_desc_sw128(0, 16, 1024);
                const uint64_t a0 = desc_k + ((base + C::kQOff) >> 4);
                while (cur.template next<false>(p, bh, qt)) {
                    const int n_kv = kv_tiles(qt);
                    wait_bar(bar_q_full, tile & 1, abort, p.status);
                    tc_fence_after();
                    for (int m = 0; m < n_kv; ++m) {
                        const int gm = gs + m;
                        const int b = gm % kSBufs;
                        if (gm >= kSBufs) {
                            // buffer b still holds P of step gm - 3 until its product is done
                            wait_bar(bar_pv_done + 8 * b, ((gm - kSBufs) / kSBufs) & 1, abort, p.status);
                            tc_fence_after();
                        }
                        const int ik = lb + load_index_k(m);
                        wait_kv(ik);
                        const uint64_t b0 = desc_k + (slot_addr(ik) >> 4);
                        const uint32_t d_tmem = tmem + C::col_s(b);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                            mma_ss(d_tmem, a0 + off, b0 + off, idesc_s, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(bar_s_full + 8 * b);
                        mma_commit(bar_kv_empty + 8 * (ik % C::kSlots));
                    }
                    mma_commit(bar_q_empty);
                    gs += n_kv;
                    lb += 2 * n_kv;
                    ++tile;
                    if (*abort) break;
                }
                // every score product has completed before TMEM is released
                if (tile > 0) wait_bar(bar_q_empty, (tile - 1) & 1, abort, p.status);
            } else {
                // ==================================================== output issuer
                // O += P_b V: P_b from TMEM (8 columns per 16 keys); V is
                // MN-major (d contiguous): 8-key groups 1024 bytes apart,
                // 64-column halves of d one box (16 KiB) apart; 16 keys = 2048
                // bytes per MMA.
                constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, true);
                const uint64_t desc_v = smem_desc_sw128(0, C::kBoxBytes, 1024);
                while (cur.template next<false>(p, bh, qt)) {
                    const int n_kv = kv_tiles(qt);
                    if (tile > 0) {
                        // O of the previous tile has been read out by the epilogue
                        wait_bar(bar_o_empty, (tile - 1) & 1, abort, p.status);
                        tc_fence_after();
                    }
                    for (int t = 0; t < n_kv; ++t) {
                        const int gt = gs + t;
                        const int b = gt % kSBufs;
                        const int iv = lb + load_index_v(t, n_kv);
                        // P_t first: it implies that every K_m (m <= t) has landed,
                        // which the parity wait on V_t's slot relies on (see
                        // TileCfg).
                        wait_bar(bar_p_full + 8 * b, (gt / kSBufs) & 1, abort, p.status);
                        wait_kv(iv);
                        const uint64_t b0 = desc_v + (slot_addr(iv) >> 4);
                        const uint32_t a_tmem = tmem + C::col_s(b) + C::kColP;
#pragma unroll
                        for (int kk = 0; kk < kBlockN / 16; ++kk)
                            mma_ts(tmem + C::kColO, a_tmem + kk * 8, b0 + kk * (2048 >> 4), idesc_o,
                                   (t > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(bar_pv_done + 8 * b);
                        mma_commit(bar_kv_empty + 8 * (iv % C::kSlots));
                    }
                    mma_commit(bar_o_full);
                    gs += n_kv;
                    lb += 2 * n_kv;
                    ++tile;
                    if (*abort) break;
                }
                if (tile > 0) wait_bar(bar_o_full, (tile - 1) & 1, abort, p.status);
            }
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
