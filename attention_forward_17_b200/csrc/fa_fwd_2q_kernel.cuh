// Two-query-tile variant of the fused attention forward pass for sm_100a.
//
// Same operation, inputs, outputs and host interface as fa_fwd_kernel (the
// FlashAttention forward pass of the "TileLang tutorial": query, key and value
// tiles streamed through on-chip memory, running row maxima, running
// normalisation sums and rescaling factors, both products on the tensor
// cores).  What differs is the work unit: a CTA owns TWO 128-row query tiles
// of one (b, h) slice (rows 256c .. 256c+255) and streams every key/value tile
// once for both of them.
//
// Roles (384 threads):
//   warps 0-3  softmax for query tile 0, warps 4-7 for query tile 1.  A thread
//              owns one query row (TMEM lane = row, 32x32b accesses): a row's
//              128 scores sit in one thread's registers, so row maxima and sums
//              need no shuffles.
//   warp 8     TMA producer: Q_0 and Q_1 once, then K_0, V_0, K_1, V_1, ...
//              through one shared-memory ring (full / empty mbarriers).
//   warp 9     MMA issuer (one thread): S_i = Q_i K_j^T and O_i += P_i V_j for
//              both tiles, in a fixed alternating order.
//   warp 10    allocates and frees TMEM.
//
// Tensor memory (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D,256+2D).  The softmax writes P_i (bf16, two keys per column) over
// columns [64,128) of S_i, and O_i += P_i V_j reads P_i straight from TMEM (the
// tensor core's TMEM-A form), so P never touches shared memory.
//
// Why a single issuing thread: tcgen05 operations of one thread complete in
// issue order, and an mbarrier commit fires once every earlier operation of
// that thread has completed.  The issuer issues
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
// The lazy O rescale (a row's maximum grew by more than 2^8) is therefore done
// in place by the softmax thread that owns the row, between its P store and
// its release of P, with no wait on the tensor core: the rescale is off the
// tensor pipe's critical path and costs only the TMEM round trip of that row.
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
// Causal mask: tile 0 of pair c needs key tiles 0..2c, tile 1 needs 0..2c+1;
// the ring carries 2c+2 key tiles and the last one only feeds tile 1.  The
// issuer waits for every ring load exactly once, in load order, which keeps
// every parity wait on the ring sound for any depth (it waits for load L only
// after observing load L-1), and releases each load by one commit after its
// last use.
//
// Every mbarrier wait is bounded in time (see wait_bar in fa_fwd_kernel.cuh).
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

template <int D, int SLOTS>
struct Q2Cfg {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static_assert(SLOTS >= 2, "K/V ring depth");
    static constexpr int kTileBytes = 128 * D * 2;          // one 128-row tile of Q, K, V or O
    static constexpr int kBoxes = D / 64;                   // 64-column (128-byte) TMA boxes
    static constexpr int kBoxBytes = 128 * 128;
    static constexpr int kSlots = SLOTS;
    static constexpr int kQOff = 0;                         // Q_0, then Q_1 (O staging at the end)
    static constexpr int kSlotOff = 2 * kTileBytes;
    static constexpr int kBarOff = kSlotOff + SLOTS * kTileBytes;
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOff + 512;
    static constexpr uint32_t kColO = 256;
    static constexpr uint32_t kColP = 64;                   // P_i inside S_i
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA (227 KiB)");
    static_assert(kColO + 2 * D <= kTmemCols, "two score and two output buffers in TMEM");
};

template <int kSlots>
struct alignas(8) Q2Barriers {
    uint64_t kv_full[kSlots];
    uint64_t kv_empty[kSlots];     // released by one commit after the load's last use
    uint64_t q_full[2];
    uint64_t s_full[2];            // S_i(j) computed (and PV_i(j-1) completed)
    uint64_t p_full[2];            // P_i(j) in TMEM, O_i rescaled (128 arrivals)
    uint64_t o_full[2];            // every product of tile i completed
    uint32_t tmem_base;
    volatile uint32_t abort;
};

constexpr int kQ2IssuerWarp = 9;       // issues every tcgen05.mma of the CTA
constexpr int kQ2AllocWarp = 10;

// CTA index -> (b, h) slice and query-tile pair.  Without the mask the pairs
// of one slice are adjacent in launch order (the slice's K/V stay in L2).
// Under the mask slices are taken `group` at a time and the pairs of a group
// launch longest first.
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

template <int D, bool CAUSAL, int EMU, int SLOTS>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_2q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                     const FwdParams p) {
    using C = Q2Cfg<D, SLOTS>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);
    auto* bars = reinterpret_cast<Q2Barriers<SLOTS>*>(smem + C::kBarOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_pair = (p.n_qtile + 1) / 2;
    int bh, c;
    map_pair<CAUSAL>(p, n_pair, blockIdx.x, bh, c);
    const int n_kv_all = (p.N + kBlockN - 1) / kBlockN;
    // key tiles of query tile i (0 when the tile lies past N)
    const auto kv_tiles = [&](int i) {
        const int q0 = 256 * c + 128 * i;
        if (q0 >= p.N) return 0;
        return CAUSAL ? min(n_kv_all, 2 * c + i + 1) : n_kv_all;
    };
    const int n_kv = max(kv_tiles(0), kv_tiles(1));

    const uint32_t bar_kv_full = smem_u32(&bars->kv_full[0]);
    const uint32_t bar_kv_empty = smem_u32(&bars->kv_empty[0]);
    const uint32_t bar_q_full = smem_u32(&bars->q_full[0]);
    const uint32_t bar_s_full = smem_u32(&bars->s_full[0]);
    const uint32_t bar_p_full = smem_u32(&bars->p_full[0]);
    const uint32_t bar_o_full = smem_u32(&bars->o_full[0]);
    volatile uint32_t* abort = &bars->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SLOTS; ++s) {
            mbar_init(bar_kv_full + 8 * s, 1);
            mbar_init(bar_kv_empty + 8 * s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar_q_full + 8 * i, 1);
            mbar_init(bar_s_full + 8 * i, 1);
            mbar_init(bar_p_full + 8 * i, 128);
            mbar_init(bar_o_full + 8 * i, 1);
        }
        bars->abort = 0u;
        fence_barrier_init();
    }
    if (warp == kQ2AllocWarp) {
        tmem_alloc(smem_u32(&bars->tmem_base), C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp < 8) {
        regs_increase<kRegsSoftmax>();
        // ============================================================ softmax, one row per thread
        const int ti = warp >> 2;                 // query tile of this warpgroup
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;        // tile row = TMEM lane
        const int q0 = 256 * c + 128 * ti;
        const int row = q0 + r;
        const int n_i = kv_tiles(ti);
        const uint32_t lane_w = static_cast<uint32_t>(32 * quarter) << 16;
        const uint32_t t_s = tmem + lane_w + 128u * ti;
        const uint32_t t_p = t_s + C::kColP;
        const uint32_t t_o = tmem + lane_w + C::kColO + static_cast<uint32_t>(D) * ti;
        const float cl = p.scale_log2;
        const uint64_t c2 = f2(cl, cl);
        const uint32_t bar_s = bar_s_full + 8 * ti, bar_p = bar_p_full + 8 * ti;

        float m = -INFINITY;                      // running max of c*s (stale by < 8)
        float l = 0.f, lh = 0.f;                  // sums of the weights: fp32, and bf16-rounded
        for (int j = 0; j < n_i; ++j) {
            wait_bar(bar_s, j & 1, abort, p.status);
            tc_fence_after();
            uint32_t s[128];
            {
                uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
                uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
                uint32_t (&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[64]);
                uint32_t (&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[96]);
                tmem_ld32(t_s, s0);
                tmem_ld32(t_s + 32, s1);
                tmem_ld32(t_s + 64, s2);
                tmem_ld32(t_s + 96, s3);
                tmem_wait_ld();
                // the wait carries no register operands: pin the loaded values after it
                reg_fence32(s0);
                reg_fence32(s1);
                reg_fence32(s2);
                reg_fence32(s3);
            }
            const bool masked =
                (j * kBlockN + kBlockN > p.N) || (CAUSAL && j * kBlockN + kBlockN - 1 > q0);
            if (masked) {
                const int lim = (CAUSAL ? min(p.N, row + 1) : p.N) - j * kBlockN;
#pragma unroll
                for (int k = 0; k < 128; ++k)
                    if (k >= lim) s[k] = __float_as_uint(-INFINITY);
            }
            // row maximum: four independent chains of three-way maxima
            float x0 = fmaxf(__uint_as_float(s[0]), __uint_as_float(s[1]));
            float x1 = fmaxf(__uint_as_float(s[2]), __uint_as_float(s[3]));
            float x2 = fmaxf(__uint_as_float(s[4]), __uint_as_float(s[5]));
            float x3 = fmaxf(__uint_as_float(s[6]), __uint_as_float(s[7]));
#pragma unroll
            for (int k = 8; k < 128; k += 8) {
                x0 = max3f(x0, __uint_as_float(s[k]), __uint_as_float(s[k + 1]));
                x1 = max3f(x1, __uint_as_float(s[k + 2]), __uint_as_float(s[k + 3]));
                x2 = max3f(x2, __uint_as_float(s[k + 4]), __uint_as_float(s[k + 5]));
                x3 = max3f(x3, __uint_as_float(s[k + 6]), __uint_as_float(s[k + 7]));
            }
            const float mn = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3)) * cl;
            const bool grow = mn > m + 8.0f;
            float alpha = 1.f;
            if (grow) {
                alpha = ex2_approx(m - mn);
                m = mn;
                l *= alpha;
                lh *= alpha;
            }
            const float u = (m == -INFINITY) ? 0.f : m;
            const uint64_t negm = f2(-u, -u);
            // weights 2^(c*s - m), their sums, and P as bf16 pairs: word k = keys 2k, 2k+1
            uint64_t la0 = 0, la1 = 0, ha0 = 0, ha1 = 0;
            uint32_t pw[64];
#pragma unroll
            for (int k = 0; k < 64; ++k) {
                const uint64_t x2v = fma2(f2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), c2, negm);
                float e0, e1, p0, p1;
                f2_split(x2v, e0, e1);
                if (EMU > 0 && (k % (EMU > 0 ? EMU : 1)) == EMU - 1) {
                    exp2_poly2(e0, e1, p0, p1);
                } else {
                    p0 = ex2_approx(e0);
                    p1 = ex2_approx(e1);
                }
                const uint32_t w = pack_bf16x2(p0, p1);
                const uint64_t pr = f2(p0, p1);
                const uint64_t ph = f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
                if (k & 1) {
                    la1 = add2(la1, pr);
                    ha1 = add2(ha1, ph);
                } else {
                    la0 = add2(la0, pr);
                    ha0 = add2(ha0, ph);
                }
                pw[k] = w;
            }
            {
                uint32_t (&p0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pw[0]);
                uint32_t (&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&pw[32]);
                reg_fence32(p0);
                reg_fence32(p1);
                tmem_st32(t_p, p0);
                tmem_st32(t_p + 32, p1);
                // Lazy rescale of this row of O_i (O_i holds the products of steps
                // < j, all completed: S_i(j) was issued after PV_i(j-1)).
                const bool need = grow && j > 0;
                if (__any_sync(0xffffffffu, need)) {
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
                }
                tmem_wait_st();
                // keep the stored registers untouched until the stores completed
                reg_fence32(p0);
                reg_fence32(p1);
            }
            tc_fence_before();
            mbar_arrive(bar_p);
            float v0, v1, v2, v3;
            f2_split(add2(la0, la1), v0, v1);
            f2_split(add2(ha0, ha1), v2, v3);
            l += v0 + v1;
            lh += v2 + v3;
        }

        // ------------------------------------------------------------ epilogue
        if (n_i > 0) {
            wait_bar(bar_o_full + 8 * ti, 0, abort, p.status);
            tc_fence_after();
            // Q_i is dead (every product of issuer i has completed): stage O_i there
            const uint32_t stage = base + C::kQOff + ti * C::kTileBytes;
            const uint32_t sw = static_cast<uint32_t>(r & 7);
            const float inv = lh > 0.f ? 1.f / lh : 0.f;
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t o[32];
                tmem_ld32(t_o + 32 * q, o);
                tmem_wait_ld();
                reg_fence32(o);
                // columns 32q .. 32q+31: box q/2, 16-byte chunks 4(q%2) .. 4(q%2)+3
                const uint32_t rowaddr = stage + (q >> 1) * C::kBoxBytes + r * 128;
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
                    tma_store_3d(&tm_o, stage + bx * C::kBoxBytes, 64 * bx, q0, bh);
                bulk_commit_group();
                bulk_wait_group_read0();
            }
        }
    } else if (warp == kProducerWarp) {
        regs_decrease<kRegsOther>();
        // ============================================================ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const uint32_t slot_smem = base + C::kSlotOff;
            for (int i = 0; i < 2; ++i) {
                if (kv_tiles(i) == 0) continue;
                mbar_arrive_expect_tx(bar_q_full + 8 * i, C::kTileBytes);
#pragma unroll
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_3d(base + C::kQOff + i * C::kTileBytes + bx * C::kBoxBytes, &tm_q, 64 * bx,
                                256 * c + 128 * i, bh, bar_q_full + 8 * i, pol_q);
            }
            int ld = 0;
            for (int j = 0; j < n_kv; ++j) {
                for (int t = 0; t < 2; ++t, ++ld) {
                    const int slot = ld % SLOTS, use = ld / SLOTS;
                    if (use > 0) wait_bar(bar_kv_empty + 8 * slot, (use - 1) & 1, abort, p.status);
                    mbar_arrive_expect_tx(bar_kv_full + 8 * slot, C::kTileBytes);
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx)
                        tma_load_3d(slot_smem + slot * C::kTileBytes + bx * C::kBoxBytes, t ? &tm_v : &tm_k,
                                    64 * bx, j * kBlockN, bh, bar_kv_full + 8 * slot, pol_kv);
                }
            }
            // In an aborted CTA make sure no copy is still landing in shared
            // memory when the CTA exits.
            if (*abort) {
                for (int k = max(0, ld - SLOTS); k < ld; ++k)
                    wait_bar(bar_kv_full + 8 * (k % SLOTS), (k / SLOTS) & 1, abort, p.status);
                for (int i = 0; i < 2; ++i)
                    if (kv_tiles(i) > 0) wait_bar(bar_q_full + 8 * i, 0, abort, p.status);
            }
        }
        __syncwarp();
    } else if (warp == kQ2IssuerWarp) {
        regs_decrease<kRegsOther>();
        // ============================================================ MMA issuer (both tiles)
        if (lane == 0) {
            const int n0 = kv_tiles(0), n1 = kv_tiles(1);
            const uint32_t slot_smem = base + C::kSlotOff;
            const auto slot_addr = [&](int i) { return slot_smem + (i % SLOTS) * C::kTileBytes; };
            // Each ring load (K_j = load 2j, V_j = load 2j+1) is waited for once,
            // in load order, and released by one commit after its last use.
            int waited = -1;
            const auto wait_kv = [&](int i) {
                if (i <= waited) return;
                wait_bar(bar_kv_full + 8 * (i % SLOTS), (i / SLOTS) & 1, abort, p.status);
                tc_fence_after();
                waited = i;
            };
            // Descriptors are built once; the start-address field (bits 0..13,
            // address >> 4) is advanced by plain integer adds, which never carry
            // out of the field for shared-memory addresses below 256 KiB.
            constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false);
            constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, true);
            const uint64_t desc_kmaj = smem_desc_sw128(0, 16, 1024);
            // V as the B operand is MN-major (d contiguous): 8-key groups 1024 bytes
            // apart, 64-column halves of d one box (16 KiB) apart
            const uint64_t desc_v = smem_desc_sw128(0, C::kBoxBytes, 1024);
            // S_ti(j) = Q_ti K_j^T into S_ti, then signal the softmax of tile ti
            const auto issue_s = [&](int ti, int j) {
                const uint64_t a_q = desc_kmaj + ((base + C::kQOff + ti * C::kTileBytes) >> 4);
                const uint64_t b_k = desc_kmaj + (slot_addr(2 * j) >> 4);
                const uint32_t d_s = tmem + 128u * ti;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                    mma_ss(d_s, a_q + off, b_k + off, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar_s_full + 8 * ti);
            };
            // O_ti += P_ti(j) V_j, P from TMEM (8 columns per 16 keys)
            const auto issue_pv = [&](int ti, int j) {
                const uint64_t b_v = desc_v + (slot_addr(2 * j + 1) >> 4);
                const uint32_t a_p = tmem + 128u * ti + C::kColP;
                const uint32_t d_o = tmem + C::kColO + static_cast<uint32_t>(D) * ti;
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk)
                    mma_ts(d_o, a_p + kk * 8, b_v + kk * (2048 >> 4), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            };
            // Order: S_0(0), S_1(0), then per key tile j the batch of tile 0
            // (O_0 += P_0(j) V_j, S_0(j+1)) and then that of tile 1.  The tensor
            // core runs one tile's batch while the other tile's softmax works, and
            // the two softmax groups stay half a step apart.
            wait_bar(bar_q_full, 0, abort, p.status);
            tc_fence_after();
            wait_kv(0);
            issue_s(0, 0);
            if (n1 > 0) {
                wait_bar(bar_q_full + 8, 0, abort, p.status);
                tc_fence_after();
                issue_s(1, 0);
            }
            mma_commit(bar_kv_empty);                    // K_0 (slot 0)
            for (int j = 0; j < n_kv; ++j) {
                for (int ti = 0; ti < 2; ++ti) {
                    const int n_i = ti ? n1 : n0;
                    if (j >= n_i) continue;
                    wait_bar(bar_p_full + 8 * ti, j & 1, abort, p.status);
                    tc_fence_after();
                    wait_kv(2 * j + 1);
                    issue_pv(ti, j);
                    if (j + 1 < n_i) {
                        wait_kv(2 * j + 2);
                        issue_s(ti, j + 1);
                    } else {
                        mma_commit(bar_o_full + 8 * ti);
                    }
                }
                mma_commit(bar_kv_empty + 8 * ((2 * j + 1) % SLOTS));            // V_j
                if (j + 1 < n_kv) mma_commit(bar_kv_empty + 8 * ((2 * j + 2) % SLOTS));   // K_{j+1}
            }
            // every product has completed before TMEM is released
            wait_bar(bar_o_full, 0, abort, p.status);
            if (n1 > 0) wait_bar(bar_o_full + 8, 0, abort, p.status);
        }
        __syncwarp();
    } else {
        regs_decrease<kRegsOther>();   // spare warp of the third warpgroup
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kQ2AllocWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
