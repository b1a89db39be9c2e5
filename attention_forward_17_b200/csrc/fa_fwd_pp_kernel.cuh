// Split-KV ping-pong variant of the fused attention forward pass for sm_100a.
//
// Same operation, inputs, outputs and host interface as fa_fwd_kernel (the
// FlashAttention forward pass of the "TileLang tutorial"); the difference is
// how the softmax work is spread over the warps.  Each CTA owns one 128-row
// query tile, and the key/value tiles are dealt alternately to two softmax
// groups of four warps:
//   group 0 (warps 0-3) takes key tiles 0, 2, 4, ... and group 1 (warps 4-7)
//   tiles 1, 3, 5, ...; each group keeps its own running maximum and sums for
//   every row and its own output accumulator O_g in tensor memory.  A thread
//   owns one whole row (TMEM lane = row, 32x32b access), so row maxima need no
//   shuffles.  At the end the two partial results are merged per row,
//     M = max(m_0, m_1),  O = (2^(m_0-M) O_0 + 2^(m_1-M) O_1) / (2^(m_0-M) l^_0 + 2^(m_1-M) l^_1),
//   the online-softmax combination of two partial softmaxes.
//
// P goes to shared memory (one 128 x 128 bf16 tile per group, laid out as the
// 128-byte-swizzled K-major operand the tensor core reads), not over the
// scores in TMEM.  So a group frees its score buffer as soon as it has read
// the scores, and the next score product for that group runs while the group
// is still busy with exponentials; O_g += P V then reads P from shared memory.
// Before overwriting its P tile (and before rescaling O_g), a group waits
// until the product two steps back has completed.
//
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D).  Shared memory: Q tile, K/V ring, P_0, P_1, barriers;
// the per-row statistics exchange of the epilogue reuses the Q tile, which is
// dead once every product has completed.
//
// With P out of TMEM the score issuer no longer waits on a P V product, so it
// observes only K loads; the ring's parity waits stay sound when a K tile's
// slot predecessor is always a K tile, i.e. for an even ring depth of at least
// four (the load sequence alternates V and K after the first three K tiles).
//
// Roles, the K/V load sequence, bounded waits and the epilogue conventions are
// those of fa_fwd_kernel.
#pragma once

#include "fa_fwd_kernel.cuh"

namespace fa {

template <int D, int SLOTS>
struct PPCfg {
    static_assert(SLOTS >= 4 && SLOTS % 2 == 0, "even K/V ring depth of at least four");
    static constexpr int kTileBytes = kBlockN * D * 2;     // one K or V tile; also the Q tile
    static constexpr int kBoxes = D / 64;
    static constexpr int kBoxBytes = 128 * 128;
    static constexpr int kSlots = SLOTS;
    static constexpr int kQOff = 0;
    static constexpr int kSlotOff = kTileBytes;
    static constexpr int kPOff = kSlotOff + SLOTS * kTileBytes;
    static constexpr int kPBytes = 128 * 128 * 2;           // one P tile: two 64-key 128B-swizzled boxes
    static constexpr int kBarOff = kPOff + 2 * kPBytes;
    static constexpr int kSmemBytes = 1024 /* alignment slack */ + kBarOff + 512;
    static constexpr uint32_t kTmemCols = 512;
    static_assert(kSmemBytes <= 232448, "shared memory per CTA (227 KiB)");
    static_assert(256 + 2 * D <= 512, "two score and two output buffers in TMEM");
};

template <int kSlots>
struct alignas(8) PPBarriers {
    uint64_t kv_full[kSlots];
    uint64_t kv_empty[kSlots];
    uint64_t q_full;
    uint64_t s_full[2];     // S_b computed
    uint64_t s_free[2];     // the group has read S_b out of TMEM
    uint64_t p_full[2];     // P_b written to shared memory (and O_b rescaled)
    uint64_t pv_done[2];    // O_b += P_b V of the latest step on b completed
    uint64_t o_full;
    uint32_t tmem_base;
    volatile uint32_t abort;
};

template <int D, bool CAUSAL, int EMU, int SLOTS>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = PPCfg<D, SLOTS>;
    constexpr uint32_t kColO0 = 256;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_addr);
    auto* bars = reinterpret_cast<PPBarriers<C::kSlots>*>(smem + C::kBarOff);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    int bh, qt;
    map_tile<CAUSAL>(p, blockIdx.x, bh, qt);
    const int q0 = qt * kBlockM;
    const int n_kv_all = (p.N + kBlockN - 1) / kBlockN;
    const int n_kv = CAUSAL ? min(n_kv_all, qt + 1) : n_kv_all;

    const uint32_t bar_kv_full = smem_u32(&bars->kv_full[0]);
    const uint32_t bar_kv_empty = smem_u32(&bars->kv_empty[0]);
    const uint32_t bar_q_full = smem_u32(&bars->q_full);
    const uint32_t bar_s_full = smem_u32(&bars->s_full[0]);
    const uint32_t bar_s_free = smem_u32(&bars->s_free[0]);
    const uint32_t bar_p_full = smem_u32(&bars->p_full[0]);
    const uint32_t bar_pv_done = smem_u32(&bars->pv_done[0]);
    const uint32_t bar_o_full = smem_u32(&bars->o_full);
    volatile uint32_t* abort = &bars->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(bar_kv_full + 8 * s, 1);
            mbar_init(bar_kv_empty + 8 * s, 1);
        }
        mbar_init(bar_q_full, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_s_full + 8 * b, 1);
            mbar_init(bar_s_free + 8 * b, 128);
            mbar_init(bar_p_full + 8 * b, 128);
            mbar_init(bar_pv_done + 8 * b, 1);
        }
        mbar_init(bar_o_full, 1);
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
        // ============================================================ softmax groups
        const int g = warp >> 2;                  // key tiles j with j % 2 == g
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;        // tile row = TMEM lane of this thread
        const uint32_t lane_w = static_cast<uint32_t>(32 * quarter) << 16;
        const float c = p.scale_log2;
        const uint64_t c2 = f2(c, c);
        const uint32_t t_s = tmem + lane_w + 128u * g;
        const uint32_t t_o = tmem + lane_w + kColO0 + g * D;
        // this row of P_g in shared memory: box (keys 64a..), row r, 16-byte
        // chunk c stored at chunk position c ^ (r % 8) (128-byte swizzle)
        const uint32_t p_row = base + C::kPOff + g * C::kPBytes + r * 128;
        const uint32_t sw = static_cast<uint32_t>(r & 7);

        float m = -INFINITY;                      // running max of c*s (stale by < 8)
        float l = 0.f, lh = 0.f;                  // sums of the weights, fp32 and bf16-rounded

        for (int j = g; j < n_kv; j += 2) {
            wait_bar(bar_s_full + 8 * g, (j >> 1) & 1, abort, p.status);
            tc_fence_after();
            uint32_t s0[32], s1[32], s2[32], s3[32];
            tmem_ld32(t_s, s0);
            tmem_ld32(t_s + 32, s1);
            tmem_ld32(t_s + 64, s2);
            tmem_ld32(t_s + 96, s3);
            tmem_wait_ld();
            reg_fence32(s0);
            reg_fence32(s1);
            reg_fence32(s2);
            reg_fence32(s3);
            // S_g may be overwritten by the next score product from here on
            tc_fence_before();
            mbar_arrive(bar_s_free + 8 * g);

            const bool masked =
                (j * kBlockN + kBlockN > p.N) || (CAUSAL && j * kBlockN + kBlockN - 1 > q0);
            if (masked) {
                const int lim = (CAUSAL ? min(p.N, q0 + r + 1) : p.N) - j * kBlockN;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (i >= lim) s0[i] = __float_as_uint(-INFINITY);
                    if (32 + i >= lim) s1[i] = __float_as_uint(-INFINITY);
                    if (64 + i >= lim) s2[i] = __float_as_uint(-INFINITY);
                    if (96 + i >= lim) s3[i] = __float_as_uint(-INFINITY);
                }
            }
            float x0 = fmaxf(__uint_as_float(s0[0]), __uint_as_float(s0[1]));
            float x1 = fmaxf(__uint_as_float(s1[0]), __uint_as_float(s1[1]));
            float x2 = fmaxf(__uint_as_float(s2[0]), __uint_as_float(s2[1]));
            float x3 = fmaxf(__uint_as_float(s3[0]), __uint_as_float(s3[1]));
#pragma unroll
            for (int i = 2; i < 32; i += 2) {
                x0 = max3f(x0, __uint_as_float(s0[i]), __uint_as_float(s0[i + 1]));
                x1 = max3f(x1, __uint_as_float(s1[i]), __uint_as_float(s1[i + 1]));
                x2 = max3f(x2, __uint_as_float(s2[i]), __uint_as_float(s2[i + 1]));
                x3 = max3f(x3, __uint_as_float(s3[i]), __uint_as_float(s3[i + 1]));
            }
            const float mn = fmaxf(fmaxf(x0, x1), fmaxf(x2, x3)) * c;
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
            uint64_t la2 = 0, ha2 = 0;
            const auto pair = [&](uint32_t a, uint32_t b, int pi) -> uint32_t {
                const uint64_t x2 = fma2(f2(__uint_as_float(a), __uint_as_float(b)), c2, negm);
                float e0, e1, p0, p1;
                f2_split(x2, e0, e1);
                if (EMU > 0 && (pi % (EMU > 0 ? EMU : 1)) == EMU - 1) {
                    exp2_poly2(e0, e1, p0, p1);
                } else {
                    p0 = ex2_approx(e0);
                    p1 = ex2_approx(e1);
                }
                const uint32_t w = pack_bf16x2(p0, p1);
                la2 = add2(la2, f2(p0, p1));
                ha2 = add2(ha2, f2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)));
                return w;
            };
            // word i = keys 2i, 2i+1
            uint32_t pw0[32], pw1[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                pw0[i] = pair(s0[2 * i], s0[2 * i + 1], i);
                pw0[16 + i] = pair(s1[2 * i], s1[2 * i + 1], 16 + i);
                pw1[i] = pair(s2[2 * i], s2[2 * i + 1], 32 + i);
                pw1[16 + i] = pair(s3[2 * i], s3[2 * i + 1], 48 + i);
            }
            float v0, v1;
            f2_split(la2, v0, v1);
            l += v0 + v1;
            f2_split(ha2, v0, v1);
            lh += v0 + v1;

            if (j >= 2) {
                // the product of step j-2 has read P_g and is the last update of O_g
                wait_bar(bar_pv_done + 8 * g, ((j - 2) >> 1) & 1, abort, p.status);
                tc_fence_after();
                if (__any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32(t_o + 32 * q, o);
                        tmem_wait_ld();
                        reg_fence32(o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        reg_fence32(o);
                        tmem_st32(t_o + 32 * q, o);
                    }
                    tmem_wait_st();
                }
            }
            // P row into shared memory: box 0 = words 0..31 (keys 0..63), box 1 = words 32..63
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t off = ((static_cast<uint32_t>(ch) ^ sw) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_row + off),
                             "r"(pw0[4 * ch]), "r"(pw0[4 * ch + 1]), "r"(pw0[4 * ch + 2]), "r"(pw0[4 * ch + 3])
                             : "memory");
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_row + C::kBoxBytes + off),
                             "r"(pw1[4 * ch]), "r"(pw1[4 * ch + 1]), "r"(pw1[4 * ch + 2]), "r"(pw1[4 * ch + 3])
                             : "memory");
            }
            // generic-proxy stores made visible to the tensor core's (async proxy) reads
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tc_fence_before();
            mbar_arrive(bar_p_full + 8 * g);
        }

        // ------------------------------------------------------------ merge + epilogue
        // every product is done, so Q is dead and its tile holds the statistics exchange
        wait_bar(bar_o_full, 0, abort, p.status);
        tc_fence_after();
        float* red = reinterpret_cast<float*>(smem + C::kQOff);
        red[(g * 3 + 0) * 128 + r] = m;
        red[(g * 3 + 1) * 128 + r] = l;
        red[(g * 3 + 2) * 128 + r] = lh;
        named_barrier_sync(1 + quarter, 64);      // warps `quarter` and `quarter + 4`: same rows
        const float m0 = red[r], l0 = red[128 + r], lh0 = red[256 + r];
        const bool has1 = n_kv > 1;               // group 1 saw at least one key tile
        const float m1 = has1 ? red[384 + r] : -INFINITY;
        const float l1 = has1 ? red[512 + r] : 0.f;
        const float lh1 = has1 ? red[640 + r] : 0.f;
        const float M = fmaxf(m0, m1);
        const float w0 = (M == -INFINITY || m0 == -INFINITY) ? 0.f : ex2_approx(m0 - M);
        const float w1 = (M == -INFINITY || m1 == -INFINITY) ? 0.f : ex2_approx(m1 - M);
        const float lh_t = w0 * lh0 + w1 * lh1;
        const float l_t = w0 * l0 + w1 * l1;
        const float inv = lh_t > 0.f ? 1.f / lh_t : 0.f;
        const float s_0 = w0 * inv, s_1 = w1 * inv;
        const int row = q0 + r;
        const bool valid = row < p.N;
        // this thread writes columns [g*D/2, (g+1)*D/2) of its row
        __nv_bfloat16* orow = p.o + (static_cast<int64_t>(bh) * p.N + row) * D + g * (D / 2);
#pragma unroll 1
        for (int q = 0; q < D / 64; ++q) {
            const uint32_t col = kColO0 + g * (D / 2) + 32 * q;
            uint32_t a[32], b[32];
            tmem_ld32(tmem + lane_w + col, a);
            if (has1) tmem_ld32(tmem + lane_w + col + D, b);
            tmem_wait_ld();
            reg_fence32(a);
            if (has1) reg_fence32(b);
            if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float ob = has1 ? __uint_as_float(b[8 * v + e]) * s_1 : 0.f;
                        f[e] = __uint_as_float(a[8 * v + e]) * s_0 + ob;
                    }
                    dst[v] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                        pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                }
            }
        }
        if (valid && g == 0) {
            float lse = l_t > 0.f ? (M + lg2_approx(l_t)) * 0.69314718055994531f : -INFINITY;
            if (*abort) lse = __int_as_float(0x7fc00000);
            p.lse[static_cast<int64_t>(bh) * p.N + row] = lse;
        }
    } else if (warp == kProducerWarp) {
        regs_decrease<kRegsOther>();
        // ============================================================ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = policy_evict_first();
            const uint64_t pol_kv = policy_evict_last();
            const uint32_t slot_smem = base + C::kSlotOff;
            mbar_arrive_expect_tx(bar_q_full, C::kTileBytes);
#pragma unroll
            for (int bx = 0; bx < C::kBoxes; ++bx)
                tma_load_3d(base + C::kQOff + bx * C::kBoxBytes, &tm_q, 64 * bx, q0, bh, bar_q_full, pol_q);
            int i = 0;
            auto load = [&](bool is_v, int tile) {
                const int slot = i % C::kSlots;
                const int use = i / C::kSlots;
                if (use > 0) wait_bar(bar_kv_empty + 8 * slot, (use - 1) & 1, abort, p.status);
                const CUtensorMap* map = is_v ? &tm_v : &tm_k;
                mbar_arrive_expect_tx(bar_kv_full + 8 * slot, C::kTileBytes);
#pragma unroll
                for (int bx = 0; bx < C::kBoxes; ++bx)
                    tma_load_3d(slot_smem + slot * C::kTileBytes + bx * C::kBoxBytes, map, 64 * bx,
                                tile * kBlockN, bh, bar_kv_full + 8 * slot, pol_kv);
                ++i;
            };
            for (int m = 0; m < kSBufs && m < n_kv; ++m) load(false, m);
            for (int t = 0; t < n_kv; ++t) {
                load(true, t);
                if (t + kSBufs < n_kv) load(false, t + kSBufs);
            }
            if (*abort) {
                for (int k = max(0, i - C::kSlots); k < i; ++k)
                    wait_bar(bar_kv_full + 8 * (k % C::kSlots), (k / C::kSlots) & 1, abort, p.status);
                wait_bar(bar_q_full, 0, abort, p.status);
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
            const uint64_t desc_kmaj = smem_desc_sw128(0, 16, 1024);
            if (warp == kMmaWarp) {
                // ==================================================== score issuer
                constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false);
                const uint64_t a0 = desc_kmaj + ((base + C::kQOff) >> 4);
                wait_bar(bar_q_full, 0, abort, p.status);
                tc_fence_after();
                for (int m = 0; m < n_kv; ++m) {
                    const int b = m & 1;
                    if (m >= 2) {
                        // the group has read S_b of step m-2
                        wait_bar(bar_s_free + 8 * b, ((m - 2) >> 1) & 1, abort, p.status);
                        tc_fence_after();
                    }
                    const int ik = load_index_k(m);
                    wait_kv(ik);
                    const uint64_t b0 = desc_kmaj + (slot_addr(ik) >> 4);
                    const uint32_t d_tmem = tmem + 128u * b;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                        mma_ss(d_tmem, a0 + off, b0 + off, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar_s_full + 8 * b);
                    mma_commit(bar_kv_empty + 8 * (ik % C::kSlots));
                }
                if (n_kv > 0)
                    wait_bar(bar_s_full + 8 * ((n_kv - 1) & 1), ((n_kv - 1) >> 1) & 1, abort, p.status);
            } else {
                // ==================================================== output issuer
                // O_b += P_b V: P_b K-major from shared memory (two 64-key boxes,
                // 16 keys = 32 bytes per MMA), V MN-major as in fa_fwd_kernel
                constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, true);
                const uint64_t desc_v = smem_desc_sw128(0, C::kBoxBytes, 1024);
                for (int t = 0; t < n_kv; ++t) {
                    const int b = t & 1;
                    const int iv = load_index_v(t, n_kv);
                    // P_t first (it implies every K_m, m <= t, has landed)
                    wait_bar(bar_p_full + 8 * b, (t >> 1) & 1, abort, p.status);
                    wait_kv(iv);
                    const uint64_t b0 = desc_v + (slot_addr(iv) >> 4);
                    const uint64_t a0 = desc_kmaj + ((base + C::kPOff + b * C::kPBytes) >> 4);
                    const uint32_t d_tmem = tmem + kColO0 + b * D;
#pragma unroll
                    for (int kk = 0; kk < kBlockN / 16; ++kk) {
                        const uint32_t a_off = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
                        mma_ss(d_tmem, a0 + a_off, b0 + kk * (2048 >> 4), idesc_o,
                               (t >= 2 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(bar_pv_done + 8 * b);
                    mma_commit(bar_kv_empty + 8 * (iv % C::kSlots));
                }
                mma_commit(bar_o_full);
                wait_bar(bar_o_full, 0, abort, p.status);
            }
        }
        __syncwarp();
    } else {
        regs_decrease<kRegsOther>();   // spare warp of the third warpgroup
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace fa
