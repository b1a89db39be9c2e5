// Multi-query-tile variant of the fused attention forward pass for sm_100a.
//
// Same operation, inputs, outputs and host interface as fa_fwd_kernel (the
// FlashAttention forward pass of the "TileLang tutorial": query, key and value
// tiles streamed through on-chip memory, running row maxima, running
// normalisation sums and rescaling factors, both products on the tensor
// cores).  What differs is the work unit: a CTA owns TWO 128-row query tiles
// of one (b, h) slice (rows 256c .. 256c+255) and streams every key/value tile
// once for both of them.  At d = 64 a CTA may own THREE (NT = 3, rows 384c ..
// 384c+383): the description below is for two, and three tiles extend every
// per-tile role, barrier and buffer by one (see Q2Roles for the warps).
//
// Roles (384 threads with two tiles):
//   warps 0-3  softmax for query tile 0, warps 4-7 for query tile 1.  A thread
//              owns one query row (TMEM lane = row, 32x32b accesses): a row's
//              scores of a key tile pass through one thread's registers, so
//              row maxima and sums need no shuffles.
//   warp 8     TMA producer: Q_0 and Q_1 once, then K_0, V_0, K_1, V_1, ...
//              through one shared-memory ring (full / empty mbarriers).
//   warp 9     MMA issuer: S_i = Q_i K_j^T and O_i += P_i V_j for both tiles,
//              in a fixed alternating order.  The whole warp runs the issuing
//              loop and one elected lane issues each instruction, which keeps
//              the descriptor arithmetic warp-uniform (issuing from a lone lane
//              in a divergent branch cost 65-85 cycles per product, more than
//              the 64 the tensor core needs for one).
//   warp 10    allocates and frees TMEM.
//
// Key tiles are BN rows (BN = 64, 80, 128 or 192, a template parameter; the
// tile of queries is always 128 rows).  Tensor memory (512 columns): S_0 [0,BN),
// S_1 [BN,2BN), O_0 [2BN,2BN+D), O_1 [2BN+D,2BN+2D), which bounds BN by
// 2 BN + 2 D <= 512 (NT BN + NT D <= 512 with NT tiles).  The softmax writes P_i (bf16, two keys per column) over
// the first BN/2 columns of S_i once it has read them, and O_i += P_i V_j reads
// P_i straight from TMEM (the tensor core's TMEM-A form), so P never touches
// shared memory.
//
// Why a single issuing thread (the elected lane): tcgen05 operations of one
// thread complete in issue order, and an mbarrier commit fires once every
// earlier operation of that thread has completed.  The issuer issues
//     S_0(0), S_1(0), [PV_0(0), S_0(1)], [PV_1(0), S_1(1)], [PV_0(1), S_0(2)], ...
// so (a) S_i(j+1), which overwrites P_i(j), is issued after the product that
// reads P_i(j); (b) when the softmax sees S_i(j) complete, PV_i(j-1) has
// completed too and no product touches O_i until the softmax releases P_i(j);
// and (c) the tensor core takes the two tiles' batches strictly in turn, so
// the softmax groups run half a step apart instead of in lockstep (with one
// issuer per tile the tensor core interleaved both tiles' products, both
// groups received their scores together and competed for the exponential
// unit while the tensor core idled: 850-890 TFLOP/s against 1050-1100 for the
// one-tile kernels at B=1, H=32, N=16384, d=128).
// The lazy O rescale (a row's maximum grew by more than 2^32) is therefore done
// in place by the softmax thread that owns the row, before it releases P, with
// no wait on the tensor core: the rescale costs only the TMEM round trip of
// that row (no correction warps and no barrier round trip are needed).
// While softmax group 0 works on S_0(j), the tensor core runs tile 1's
// products, and the other way round, so the exponentials of one tile overlap
// the matrix products of the other.
//
// Epilogue: O_i / l^ is rounded to bf16 and written, row per thread, into the
// dead Q_i tile in shared memory in the 128-byte-swizzled box layout, then one
// thread stores the whole 128 x D tile with TMA (rows past N are clipped by the
// tensor map): coalesced full-line writes.  LSE (one fp32 per row, consecutive
// rows in consecutive lanes) is stored directly.
//
// Causal mask: query tile i of pair c needs the key tiles that hold keys
// 0 .. 256c + 128i + 127; the ring carries those of tile 1 and the last ones
// only feed tile 1.  The issuer waits for every ring load exactly once, in
// load order, which keeps
// every parity wait on the ring sound for any depth (it waits for load L only
// after observing load L-1), and releases each load by one commit after its
// last use.
//
// Every mbarrier wait is bounded in time (see wait_bar in fa_fwd_kernel.cuh).
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

template <int D, int SLOTS, int BN, bool DB, bool LT, int NT = 2>
struct Q2Cfg {
    static_assert(NT == 2 || NT == 3, "two or three query tiles per CTA");
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static_assert(BN == 64 || BN == 80 || BN == 128 || BN == 192, "key tile of 64, 80, 128 or 192 rows");
    // with double-buffered scores the issuer needs K_{j+2} while V_j is still
    // unreleased: four loads in flight
    static_assert(SLOTS >= (DB ? 4 : 2), "K/V ring depth");
    static constexpr int kQTileBytes = 128 * D * 2;         // one 128-row tile of Q (or O)
    static constexpr int kKVTileBytes = BN * D * 2;         // one BN-row tile of K or V
    static constexpr int kBoxes = D / 64;                   // 64-column (128-byte) TMA boxes
    static constexpr int kQBoxBytes = 128 * 128;
    static constexpr int kKVBoxBytes = BN * 128;
    static constexpr int kSlots = SLOTS;
    static constexpr int kQOff = 0;                         // Q_0, Q_1 (, Q_2) (O staging at the end)
    static constexpr int kSlotOff = NT * kQTileBytes;
    // LT: a BN-row tile of bf16 ones after the ring; the P.V product reads it as
    // 16 extra columns of V, so O gains 16 columns that each accumulate the sum
    // of the bf16 weights (l^) on the tensor core
    static_assert(!LT || D == 64, "the ones tile is addressed as V's second 64-column chunk");
    static constexpr int kOnesOff = kSlotOff + SLOTS * kKVTileBytes;
    static constexpr int kOnesBytes = LT ? BN * 128 : 0;
    static constexpr int kBarOff = kOnesOff + kOnesBytes;
    static constexpr int kDO = D + (LT ? 16 : 0);           // columns of one O buffer
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOff + 512;
    // TMEM: the score buffers of tile 0, then those of tile 1 (one each, or two
    // each with DB), then O_0 and O_1 (D columns each); P (bf16 pairs, BN/2
    // columns) over the first columns of the score buffer it was computed from
    static constexpr int kSBufs = DB ? 2 : 1;
    __host__ __device__ static constexpr uint32_t col_s(int ti, int b) {
        return static_cast<uint32_t>((ti * kSBufs + b) * BN);
    }
    static constexpr uint32_t kColO = NT * kSBufs * BN;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA (227 KiB)");
    static_assert(kColO + NT * kDO <= kTmemCols, "score and output buffers in TMEM");
    static_assert(kKVBoxBytes % 1024 == 0, "slots on 1024-byte boundaries (128-byte swizzle)");
};

template <int kSlots, int NT = 2>
struct alignas(8) Q2Barriers {
    uint64_t kv_full[kSlots];
    uint64_t kv_empty[kSlots];     // released by one commit after the load's last use
    uint64_t q_full[NT];
    uint64_t s_full[2 * NT];       // [2i + b]: S_i(j) computed into score buffer b
    // [2i + b]: the first / second half of P_i(j)'s keys in score buffer b (O_i
    // rescaled before the first), 128 arrivals.  One pair per score buffer:
    // with two buffers the softmax can release P_i(j+1) before the issuer has
    // waited for P_i(j), and a single barrier would then be two phases ahead
    // of that parity wait.
    uint64_t p_half[2 * NT];
    uint64_t p_full[2 * NT];
    uint64_t pv_done[NT];          // O_i += P_i(j) V_j completed (double-buffered scores)
    uint64_t o_full[NT];           // every product of tile i completed
    uint32_t tmem_base;
    volatile uint32_t abort;
};

// Stores N words of this thread's TMEM lane at consecutive columns from
// taddr and waits until the stores completed.  The fences keep the words fully
// computed before the asynchronous store and their registers untouched until
// the wait (neither asm statement tells the compiler that the hardware reads
// the registers after the store issues).  N is a multiple of 8: 32-column
// stores, then one of 16 and one of 8 columns for the rest.
template <int N>
__device__ __forceinline__ void store_words(uint32_t taddr, uint32_t (&w)[N]) {
    static_assert(N % 8 == 0, "whole 8-column stores");
    constexpr int k32 = N / 32, r16 = (N % 32) >= 16 ? 1 : 0, r8 = (N % 16) ? 1 : 0;
    constexpr int o16 = 32 * k32, o8 = o16 + 16 * r16;
    const auto fence_all = [&]() {
#pragma unroll
        for (int q = 0; q < k32; ++q) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&w[32 * q]));
        if constexpr (r16) reg_fence16(*reinterpret_cast<uint32_t(*)[16]>(&w[o16]));
        if constexpr (r8) reg_fence8(*reinterpret_cast<uint32_t(*)[8]>(&w[o8]));
    };
    fence_all();
#pragma unroll
    for (int q = 0; q < k32; ++q) tmem_st32(taddr + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&w[32 * q]));
    if constexpr (r16) tmem_st16(taddr + o16, *reinterpret_cast<uint32_t(*)[16]>(&w[o16]));
    if constexpr (r8) tmem_st8(taddr + o8, *reinterpret_cast<uint32_t(*)[8]>(&w[o8]));
    tmem_wait_st();
    fence_all();
}

// Lazy rescale threshold (log2 units): O and the sums are rescaled only when a
// row's maximum grows by more than this since the last rescale, so P is bounded
// by 2^32.  That is exact in range for bf16 and fp32 (relative precision does not
// depend on scale), the sums stay below 2^32 times the number of keys, the O
// accumulator below about 2^32 * max|v| * N, and the polynomial exponential's
// exponent field stays below 127 + 32.  On q, k ~ N(0, 3^2) scores a row's
// maximum grows by about 20 over the whole row, so rescales become rare: at a
// threshold of 8 they cost a tenth of the step, at 16 they still fired on 14 %
// of (warp, key tile) steps.
constexpr float kRescaleTau = 32.0f;

// Warp roles and register budgets.  setmaxnreg acts on whole warpgroups (four
// consecutive warps), so the last warpgroup always holds the producer, the
// issuer, the TMEM allocator and a spare warp.  Two query tiles: warps 0-7
// softmax (one per TMEM lane quarter and tile), 8 producer, 9 issuer, 10 TMEM
// allocation, 11 spare (384 threads launched with 168 registers; the softmax
// warps raise theirs to 208, the others drop to 88).  Three query tiles: warps
// 0-11 softmax, 12 producer, 13 issuer, 14 TMEM allocation, 15 spare (512
// threads launched with 128; softmax 144, the others 80, which also fills each
// SM partition's 512 registers a lane exactly: three softmax warps and one other).
template <int NT>
struct Q2Roles {
    static constexpr int kSoftWarps = 4 * NT;
    static constexpr int kProducer = kSoftWarps;
    static constexpr int kIssuer = kSoftWarps + 1;
    static constexpr int kAlloc = kSoftWarps + 2;
    static constexpr int kThreads = 32 * (kSoftWarps + 4);
    static constexpr int kLaunchRegs = NT == 2 ? 168 : 128;
    static constexpr uint32_t kRegsSoft = NT == 2 ? kRegsSoftmax : 144;
    static constexpr uint32_t kRegsRest = NT == 2 ? kRegsOther : 80;
    static constexpr int kRegTotal = kSoftWarps * 32 * static_cast<int>(kRegsSoft) +
                                     (kThreads - kSoftWarps * 32) * static_cast<int>(kRegsRest);
    static_assert(kRegTotal <= kThreads * kLaunchRegs, "register rebalance within the launch");
    static_assert(kThreads * kLaunchRegs <= 65536, "registers of one SM");
};

// CTA index -> (b, h) slice and group of query tiles (a pair, or a triple).
// Without the mask the groups of one slice are adjacent in launch order (the
// slice's K/V stay in L2).  Under the mask slices are taken `group` at a time
// and the tile groups of a slice group launch longest first.
template <bool CAUSAL>
__device__ __forceinline__ void map_pair(const FwdParams& p, int n_pair, int id, int& bh, int& c) {
    if constexpr (CAUSAL) {
        const int span = p.group * n_pair;
        const int g0 = (id / span) * p.group;
        const int heads = min(p.group, p.BH - g0);
        const int rr = id % span;
        bh = g0 + rr % heads;
        c = n_pair - 1 - rr / heads;
    } else {
        bh = id / n_pair;
        c = id % n_pair;
    }
}

template <int D, bool CAUSAL, int EMU, int SLOTS, int BN, bool DB, bool LT, bool P34, int NT>
__global__ void __launch_bounds__(Q2Roles<NT>::kThreads, 1)
    fa_fwd_2q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const FwdParams p) {
    using C = Q2Cfg<D, SLOTS, BN, DB, LT, NT>;
    using R = Q2Roles<NT>;
    // P is released in two parts of kW0 and kW1 words (two keys a word): halves,
    // or with P34 the first three quarters of the keys and then the last quarter.
    // The product with the first part then runs while the last quarter's weights
    // are computed and ends about when they are released, so only a quarter of
    // the key tile's P.V product follows the softmax's last release (instead of
    // half): the chain softmax -> P.V -> next scores -> softmax that bounds a
    // tile's step gets shorter by a quarter of a P.V product.
    // 80-row key tiles are released as 48 + 32 keys (a 40-key half is not a whole
    // number of 16-key products)
    static_assert(!P34 || BN == 128, "three-quarter release: key tiles of 128 rows");
    constexpr int kW0 = P34 ? 3 * BN / 8 : (BN == 80 ? 24 : BN / 4);
    constexpr int kW1 = BN / 2 - kW0;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);
    auto* bars = reinterpret_cast<Q2Barriers<SLOTS, NT>*>(smem + C::kBarOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_pair = (p.n_qtile + NT - 1) / NT;     // tile groups per slice
    int bh, c;
    map_pair<CAUSAL>(p, n_pair, blockIdx.x, bh, c);
    const int n_kv_all = (p.N + BN - 1) / BN;
    // first query row of tile i of this CTA
    const auto tile_q0 = [&](int i) { return 128 * (NT * c + i); };
    // key tiles of query tile i (0 when the tile lies past N); under the mask
    // the tiles holding keys 0 .. q0+127
    const auto kv_tiles = [&](int i) {
        const int q0 = tile_q0(i);
        if (q0 >= p.N) return 0;
        return CAUSAL ? min(n_kv_all, (q0 + 128 + BN - 1) / BN) : n_kv_all;
    };
    int n_kv = 0;
#pragma unroll
    for (int i = 0; i < NT; ++i) n_kv = max(n_kv, kv_tiles(i));

    const uint32_t bar_kv_full = smem_u32(&bars->kv_full[0]);
    const uint32_t bar_kv_empty = smem_u32(&bars->kv_empty[0]);
    const uint32_t bar_q_full = smem_u32(&bars->q_full[0]);
    const uint32_t bar_s_full = smem_u32(&bars->s_full[0]);
    const uint32_t bar_p_half = smem_u32(&bars->p_half[0]);
    const uint32_t bar_p_full = smem_u32(&bars->p_full[0]);
    const uint32_t bar_pv_done = smem_u32(&bars->pv_done[0]);
    const uint32_t bar_o_full = smem_u32(&bars->o_full[0]);
    volatile uint32_t* abort = &bars->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SLOTS; ++s) {
            mbar_init(bar_kv_full + 8 * s, 1);
            mbar_init(bar_kv_empty + 8 * s, 1);
        }
        for (int i = 0; i < 2 * NT; ++i) {
            mbar_init(bar_s_full + 8 * i, 1);
            mbar_init(bar_p_half + 8 * i, 128);
            mbar_init(bar_p_full + 8 * i, 128);
        }
        for (int i = 0; i < NT; ++i) {
            mbar_init(bar_q_full + 8 * i, 1);
            mbar_init(bar_pv_done + 8 * i, 1);
            mbar_init(bar_o_full + 8 * i, 1);
        }
        bars->abort = 0u;
        fence_barrier_init();
    }
    if (warp == R::kAlloc) {
        tmem_alloc(smem_u32(&bars->tmem_base), C::kTmemCols);
        tmem_relinquish();
    }
    if constexpr (LT) {
        // the ones tile (bf16 1.0 everywhere, so its swizzled layout needs no care),
        // written by the softmax threads and made visible to the tensor core
        if (warp < R::kSoftWarps) {
            const uint32_t ones = base + C::kOnesOff;
#pragma unroll 1
            for (int i = threadIdx.x; i < C::kOnesBytes / 16; i += 32 * R::kSoftWarps)
                st_shared_v4(ones + 16 * i, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
            fence_proxy_async_smem();
        }
    }
    if (warp == R::kProducer && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp < R::kSoftWarps) {
        regs_increase<R::kRegsSoft>();
        // ============================================================ softmax, one row per thread
        const int ti = warp >> 2;                 // query tile of this warpgroup
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;        // tile row = TMEM lane
        const int q0 = tile_q0(ti);
        const int row = q0 + r;
        const int n_i = kv_tiles(ti);
        const uint32_t lane_w = static_cast<uint32_t>(32 * quarter) << 16;
        const uint32_t t_s0 = tmem + lane_w + C::col_s(ti, 0);
        const uint32_t t_o = tmem + lane_w + C::kColO + static_cast<uint32_t>(C::kDO) * ti;
        const float cl = p.scale_log2;
        const uint64_t c2 = f2(cl, cl);


        float m = -INFINITY;                      // running max of c*s (stale by up to kRescaleTau)
        float l = 0.f, lh = 0.f;                  // sums of the weights: fp32, and bf16-rounded
        for (int j = 0; j < n_i; ++j) {
            // score buffer of this step: with DB, S_i(j) sits in buffer j % 2
            const int sb = DB ? (j & 1) : 0;
            const uint32_t t_s = t_s0 + sb * BN, t_p = t_s;
            wait_bar(bar_s_full + 8 * (2 * ti + sb), (DB ? (j >> 1) : j) & 1, abort, p.status);
            tc_fence_after();
            const bool masked =
                (j * BN + BN > p.N) || (CAUSAL && j * BN + BN - 1 > q0);
            const int lim = (CAUSAL ? min(p.N, row + 1) : p.N) - j * BN;   // keys >= lim are masked
            // Scores of this row (kRegCols held in registers; wider key tiles are
            // read twice: once for the maximum, once for the exponentials).
            constexpr int kRegCols = BN <= 128 ? BN : BN / 2;
            uint32_t s[kRegCols];
            // loads columns c0 .. c0+n-1 into s[i0 ..]; the caller waits for them
            const auto issue_loads = [&](int c0, int i0, int n) {
#pragma unroll
                for (int q = 0; q < n / 32; ++q)
                    tmem_ld32(t_s + c0 + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&s[i0 + 32 * q]));
                if (n % 32)       // 80-row key tiles: 16 more columns
                    tmem_ld32x16(t_s + c0 + n - 16, *reinterpret_cast<uint32_t(*)[16]>(&s[i0 + n - 16]));
            };
            // after tcgen05.wait::ld: pin s[i0 .. i0+n) after the wait (it carries no
            // register operands) and mask the keys past the row's limit
            const auto settle = [&](int c0, int i0, int n) {
#pragma unroll
                for (int q = 0; q < n / 32; ++q)
                    reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[i0 + 32 * q]));
                if (n % 32) reg_fence16(*reinterpret_cast<uint32_t(*)[16]>(&s[i0 + n - 16]));
                if (masked) {
#pragma unroll
                    for (int k = 0; k < n; ++k)
                        if (c0 + k >= lim) s[i0 + k] = __float_as_uint(-INFINITY);
                }
            };
            // row maximum: independent chains of three-way maxima over 16 keys each
            // (group g of 16 keys on chain g % 8), then a short tree
            float x[8];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) x[ch] = -INFINITY;
            const auto max_groups = [&](int g0, int i0, int ng) {
#pragma unroll
                for (int g = 0; g < ng; ++g) {
                    float& xc = x[(g0 + g) & 7];
#pragma unroll
                    for (int k = 0; k < 16; k += 2)
                        xc = max3f(xc, __uint_as_float(s[i0 + 16 * g + k]), __uint_as_float(s[i0 + 16 * g + k + 1]));
                }
            };
            const auto row_max = [&]() {
                return fmaxf(max3f(x[0], x[1], x[2]), max3f(x[3], x[4], fmaxf(x[5], max3f(x[6], x[7], x[7])))) * cl;
            };
            // Weights 2^(c*s - m), their sums, and P as bf16 pairs (word k = keys
            // 2k, 2k+1) for part h of the keys (2 kW0 or 2 kW1 keys, their scores
            // at s[i0 ..]).
            uint64_t la0 = 0, la1 = 0;
            float hl0 = 0.f, hh0 = 0.f, hl1 = 0.f, hh1 = 0.f;
            const auto weights_half = [&](int h, int i0, uint64_t negm, uint32_t (&pw)[kW0]) {
#pragma unroll
                for (int k = 0; k < (h ? kW1 : kW0); ++k) {
                    const int kk = (h ? kW0 : 0) + k;                    // word index in the row
                    const int sk = i0 + 2 * k;                           // its keys in s[]
                    const uint64_t x2v = fma2(f2(__uint_as_float(s[sk]), __uint_as_float(s[sk + 1])), c2, negm);
                    float e0, e1, p0, p1;
                    f2_split(x2v, e0, e1);
                    if (EMU > 0 && (kk % (EMU > 0 ? EMU : 1)) == EMU - 1) {
                        exp2_poly2(e0, e1, p0, p1);
                    } else {
                        p0 = ex2_approx(e0);
                        p1 = ex2_approx(e1);
                    }
                    const uint32_t w = pack_bf16x2(p0, p1);
                    const uint64_t pr = f2(p0, p1);
                    // the bf16 halves of w added to fp32 sums directly (mixed-precision
                    // adds), unless the tensor core sums them (LT)
                    if (k & 1) {
                        la1 = add2(la1, pr);
                        if constexpr (!LT) add_bf16x2_halves(hl1, hh1, w);
                    } else {
                        la0 = add2(la0, pr);
                        if constexpr (!LT) add_bf16x2_halves(hl0, hh0, w);
                    }
                    pw[k] = w;
                }
            };
            // Stores part h of P over the first BN/2 columns of S_i, whose scores
            // this thread has already read, and releases it to the issuer: the
            // product with the first part runs while the second is computed.
            const auto release_half = [&](int h, uint32_t (&pw)[kW0]) {
                if (h == 0)
                    store_words<kW0>(t_p, pw);
                else
                    store_words<kW1>(t_p + kW0, *reinterpret_cast<uint32_t(*)[kW1]>(&pw[0]));
                tc_fence_before();
                mbar_arrive((h == 0 ? bar_p_half : bar_p_full) + 8 * (2 * ti + sb));
            };
            // Lazy rescale of this row of O_i (warp-collective TMEM round trip when
            // any row of the warp needs it).  O_i holds the products of steps < j:
            // with one score buffer they have all completed (S_i(j) was issued after
            // PV_i(j-1)); with two, S_i(j) was issued before PV_i(j-1), so the
            // rescale first waits for that product.  The stores complete before the
            // first release of P (tcgen05.wait::st).
            const auto rescale_o = [&](bool need, float alpha) {
                if (!__any_sync(0xffffffffu, need)) return;
                if constexpr (DB) {
                    wait_bar(bar_pv_done + 8 * ti, (j - 1) & 1, abort, p.status);
                    tc_fence_after();
                }
                const unsigned rows = __popc(__ballot_sync(0xffffffffu, need));
                if (p.rescale_stats && lane == 0) {
                    atomicAdd(p.rescale_stats, 1ull);
                    atomicAdd(p.rescale_stats + 1, static_cast<unsigned long long>(rows));
                }
                __syncwarp();       // the TMEM accesses below are warp-collective
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    tmem_ld32(t_o + 32 * q, o);
                    tmem_wait_ld();
                    reg_fence32(o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    reg_fence32(o);
                    tmem_st32(t_o + 32 * q, o);
                }
                if constexpr (LT) {
                    // the l^ columns of O
                    uint32_t o[16];
                    tmem_ld32x16(t_o + D, o);
                    tmem_wait_ld();
                    reg_fence16(o);
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    reg_fence16(o);
                    tmem_st16(t_o + D, o);
                }
            };
            uint32_t pw[kW0];
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += kRegCols) {
                if (BN > 128 || c0 == 0) {
                    issue_loads(c0, 0, kRegCols);
                    tmem_wait_ld();
                    settle(c0, 0, kRegCols);
                }
                max_groups(c0 / 16, 0, kRegCols / 16);
            }
            const float mn = row_max();
            const bool grow = mn > m + kRescaleTau;
            float alpha = 1.f;
            if (grow) {
                alpha = ex2_approx(m - mn);
                m = mn;
                l *= alpha;
                lh *= alpha;
            }
            rescale_o(grow && j > 0, alpha);
            const float u = (m == -INFINITY) ? 0.f : m;
            const uint64_t negm = f2(-u, -u);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if constexpr (BN > 128) {
                    issue_loads(h * kRegCols, 0, kRegCols);
                    tmem_wait_ld();
                    settle(h * kRegCols, 0, kRegCols);
                }
                weights_half(h, BN > 128 ? 0 : 2 * (h ? kW0 : 0), negm, pw);
                release_half(h, pw);
            }
            float v0, v1;
            f2_split(add2(la0, la1), v0, v1);
            l += v0 + v1;
            lh += (hl0 + hh0) + (hl1 + hh1);
        }

        // ------------------------------------------------------------ epilogue
        if (n_i > 0) {
            wait_bar(bar_o_full + 8 * ti, 0, abort, p.status);
            tc_fence_after();
            // Q_i is dead (every product of issuer i has completed): stage O_i there
            const uint32_t stage = base + C::kQOff + ti * C::kQTileBytes;
            const uint32_t sw = static_cast<uint32_t>(r & 7);
            if constexpr (LT) {
                // l^ accumulated by the tensor core in the extra columns of O
                uint32_t t[16];
                tmem_ld32x16(t_o + D, t);
                tmem_wait_ld();
                reg_fence16(t);
                lh = __uint_as_float(t[0]);
            }
            const float inv = lh > 0.f ? 1.f / lh : 0.f;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(t_o + 32 * q, o);
                tmem_wait_ld();
                reg_fence32(o);
                // columns 32q .. 32q+31: box q/2, 16-byte chunks 4(q%2) .. 4(q%2)+3
                const uint32_t rowaddr = stage + (q >> 1) * C::kQBoxBytes + r * 128;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint32_t ch = static_cast<uint32_t>(4 * (q & 1) + v);
                    st_shared_v4(rowaddr + ((ch ^ sw) << 4),
                                 pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv),
                                 pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv),
                                 pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv),
                                 pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv));
                }
            }
            fence_proxy_async_smem();
            if (row < p.N) {
                float lse = l > 0.f ? (m + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
                if (*abort) lse = __int_as_float(0x7fc00000);
                p.lse[static_cast<int64_t>(bh) * p.N + row] = lse;
            }
            named_barrier_sync(1 + ti, 128);
            if (quarter == 0 && lane == 0) {
#pragma unroll
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_store_3d(&tm_o, stage + bx * C::kQBoxBytes, 64 * bx, q0, bh);
                bulk_commit_group();
                bulk_wait_group_read0();
            }
        }
    } else if (warp == R::kProducer) {
        regs_decrease<R::kRegsRest>();
        // ============================================================ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const uint32_t slot_smem = base + C::kSlotOff;
            for (int i = 0; i < NT; ++i) {
                if (kv_tiles(i) == 0) continue;
                mbar_arrive_expect_tx(bar_q_full + 8 * i, C::kQTileBytes);
#pragma unroll
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_3d(base + C::kQOff + i * C::kQTileBytes + bx * C::kQBoxBytes, &tm_q, 64 * bx,
                                tile_q0(i), bh, bar_q_full + 8 * i, pol_q);
            }
            int ld = 0;
            for (int j = 0; j < n_kv; ++j) {
                for (int t = 0; t < 2; ++t, ++ld) {
                    const int slot = ld % SLOTS, use = ld / SLOTS;
                    if (use > 0) wait_bar(bar_kv_empty + 8 * slot, (use - 1) & 1, abort, p.status);
                    mbar_arrive_expect_tx(bar_kv_full + 8 * slot, C::kKVTileBytes);
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx)
                        tma_load_3d(slot_smem + slot * C::kKVTileBytes + bx * C::kKVBoxBytes, t ? &tm_v : &tm_k,
                                    64 * bx, j * BN, bh, bar_kv_full + 8 * slot, pol_kv);
                }
            }
            // In an aborted CTA make sure no copy is still landing in shared
            // memory when the CTA exits.
            if (*abort) {
                for (int k = max(0, ld - SLOTS); k < ld; ++k)
                    wait_bar(bar_kv_full + 8 * (k % SLOTS), (k / SLOTS) & 1, abort, p.status);
                for (int i = 0; i < NT; ++i)
                    if (kv_tiles(i) > 0) wait_bar(bar_q_full + 8 * i, 0, abort, p.status);
            }
        }
        __syncwarp();
    } else if (warp == R::kIssuer) {
        regs_decrease<R::kRegsRest>();
        // ============================================================ MMA issuer (both tiles)
        // The whole warp runs the issuing loop (converged, so the descriptor
        // arithmetic stays warp-uniform); one elected lane issues each product
        // and commit.
        {
            int n_t[NT];                             // key tiles of each query tile
#pragma unroll
            for (int i = 0; i < NT; ++i) n_t[i] = kv_tiles(i);
            const uint32_t slot_smem = base + C::kSlotOff;
            const auto slot_addr = [&](int i) { return slot_smem + (i % SLOTS) * C::kKVTileBytes; };
            // Each ring load (K_j = load 2j, V_j = load 2j+1) is waited for once,
            // in load order (waiting for load i first waits for every earlier
            // one), and released by one commit after its last use.
            int waited = -1;
            const auto wait_kv = [&](int i) {
                if (i <= waited) return;
                while (waited < i) {
                    ++waited;
                    wait_bar(bar_kv_full + 8 * (waited % SLOTS), (waited / SLOTS) & 1, abort, p.status);
                }
                tc_fence_after();
            };
            // Descriptors are built once; the start-address field (bits 0..13,
            // address >> 4) is advanced by plain integer adds, which never carry
            // out of the field for shared-memory addresses below 256 KiB.
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, BN, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, C::kDO, true);
            const uint64_t desc_kmaj = smem_desc_sw128(0, 16, 1024);
            // V as the B operand is MN-major (d contiguous): 8-key groups 1024 bytes
            // apart, 64-column halves of d one box (BN x 128 bytes) apart
            const uint64_t desc_v = smem_desc_sw128(0, C::kKVBoxBytes, 1024);
            // S_ti(j) = Q_ti K_j^T into its score buffer, then signal the softmax
            // of tile ti
            const auto issue_s = [&](int ti, int j) {
                const int sb = DB ? (j & 1) : 0;
                const uint64_t a_q = desc_kmaj + ((base + C::kQOff + ti * C::kQTileBytes) >> 4);
                const uint64_t b_k = desc_kmaj + (slot_addr(2 * j) >> 4);
                const uint32_t d_s = tmem + C::col_s(ti, sb);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t a_off = ((kk >> 2) * C::kQBoxBytes + (kk & 3) * 32) >> 4;
                    const uint32_t b_off = ((kk >> 2) * C::kKVBoxBytes + (kk & 3) * 32) >> 4;
                    mma_ss_elect(d_s, a_q + a_off, b_k + b_off, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit_elect(bar_s_full + 8 * (2 * ti + sb));
            };
            // O_ti += P_ti(j) V_j for the keys of part h (2 kW0 or 2 kW1 keys), P
            // from TMEM (8 columns per 16 keys)
            const auto issue_pv = [&](int ti, int j, int h) {
                const uint32_t v_addr = slot_addr(2 * j + 1);
                // LT: V's second 64-column chunk (one chunk stride, LBO, further on)
                // is the ones tile, which follows the ring
                const uint64_t b_v =
                    (LT ? smem_desc_sw128(0, base + C::kOnesOff - v_addr, 1024) : desc_v) + (v_addr >> 4);
                const uint32_t a_p = tmem + C::col_s(ti, DB ? (j & 1) : 0);
                const uint32_t d_o = tmem + C::kColO + static_cast<uint32_t>(C::kDO) * ti;
#pragma unroll
                for (int k4 = 0; k4 < (h ? kW1 : kW0) / 8; ++k4) {
                    const int kk = (h ? kW0 / 8 : 0) + k4;          // 16 keys (8 P words) each
                    mma_ts_elect(d_o, a_p + kk * 8, b_v + kk * (2048 >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            // Order: S_0(0), S_1(0) (and, with two score buffers, S_0(1), S_1(1)),
            // then per key tile j the batch of tile 0 (O_0 += P_0(j) V_j, then the
            // next score product of tile 0: S_0(j+1), or S_0(j+2) with two score
            // buffers) and then that of tile 1.  The tensor core runs one tile's
            // batch while the other tile's softmax works, and the two softmax
            // groups stay half a step apart.  With two score buffers the score
            // product of a step is ready before the softmax reaches it, so the
            // softmax does not wait for the tensor core between steps.
            constexpr int kAhead = DB ? 2 : 1;       // score products issued ahead of the softmax
            for (int j = 0; j < kAhead && j < n_kv; ++j) {
                wait_kv(2 * j);
                for (int ti = 0; ti < NT; ++ti) {
                    if (j >= n_t[ti]) continue;
                    if (j == 0) {
                        wait_bar(bar_q_full + 8 * ti, 0, abort, p.status);
                        tc_fence_after();
                    }
                    issue_s(ti, j);
                }
                mma_commit_elect(bar_kv_empty + 8 * ((2 * j) % SLOTS));          // K_j
            }
            for (int j = 0; j < n_kv; ++j) {
                for (int ti = 0; ti < NT; ++ti) {
                    const int n_i = n_t[ti];
                    if (j >= n_i) continue;
                    // P_ti(j) sits in score buffer pb; its barriers' phase counts steps on that buffer
                    const int pb = 2 * ti + (DB ? (j & 1) : 0);
                    const uint32_t pph = (DB ? (j >> 1) : j) & 1;
                    wait_bar(bar_p_half + 8 * pb, pph, abort, p.status);
                    tc_fence_after();
                    wait_kv(2 * j + 1);
                    issue_pv(ti, j, 0);
                    wait_bar(bar_p_full + 8 * pb, pph, abort, p.status);
                    tc_fence_after();
                    issue_pv(ti, j, 1);
                    if constexpr (DB) mma_commit_elect(bar_pv_done + 8 * ti);
                    if (j + kAhead < n_i) {
                        wait_kv(2 * (j + kAhead));
                        issue_s(ti, j + kAhead);
                    }
                    if (j + 1 == n_i) mma_commit_elect(bar_o_full + 8 * ti);
                }
                mma_commit_elect(bar_kv_empty + 8 * ((2 * j + 1) % SLOTS));            // V_j
                if (j + kAhead < n_kv)
                    mma_commit_elect(bar_kv_empty + 8 * ((2 * (j + kAhead)) % SLOTS));   // K_{j+kAhead}
            }
            // every product has completed before TMEM is released
            for (int i = 0; i < NT; ++i)
                if (n_t[i] > 0) wait_bar(bar_o_full + 8 * i, 0, abort, p.status);
        }
        __syncwarp();
    } else {
        regs_decrease<R::kRegsRest>();   // spare warp of the third warpgroup
    }

    tc_fence_before();
    __syncthreads();
    if (warp == R::kAlloc) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
