// Tiled tensor-core GEMM with a fused epilogue for sm_100a ("TileLang
// tutorial": the tiled matrix multiplication section, and the fused-epilogue
// section, where the bias and GELU are applied to the accumulator before the
// single store of C):
//
//   C[i, j] = epi( sum_k A[i, k] B[k, j] ),   epi = identity | + bias[j] |
//             GELU(. + bias[j]) with GELU(x) = x/2 (1 + erf(x / sqrt 2)).
//
// A [M, K] and B [K, N] are bf16, row-major; bias bf16 [N]; C bf16 [M, N].
//
// Design (one persistent CTA per SM, 320 threads, warp-specialised):
//   warp 0      TMA producer: per 64-wide K block, A as one 128 x 64 box
//               (K-major) and B as four 64(K) x 64(N) boxes (N-major), all
//               128-byte swizzled, into a 4-stage ring (48 KiB a stage).
//   warp 1      allocates the 512 TMEM columns and issues, from one thread,
//               tcgen05.mma M=128 N=256 K=16 (full rate: 128 cycles a
//               product) into one of two 256-column fp32 accumulators;
//               tcgen05.commit frees ring stages and hands a finished
//               accumulator to the epilogue.
//   warps 2..9  epilogue: warp w reads TMEM lane quarter w % 4 and one half of
//               the columns with tcgen05.ld, adds the bias, applies GELU in
//               fp32, rounds to bf16 (nearest-even) and stores 16-byte
//               vectors.  With two accumulators the epilogue of tile t runs
//               while the tensor core works on tile t + 1.
// Tiles are visited in groups of 8 row blocks so the CTAs in flight share
// A and B panels in L2.
//
// That one-SM kernel runs problems of at most 128 rows (and K = 0).  Larger
// problems run gemm2_kernel (below): 256 x 256 tiles over SM pairs with
// tcgen05.mma.cta_group::2, which halves each SM's share of B and of the TMA
// traffic; the one-SM tile needs more shared-memory bandwidth than an SM has.  Every mbarrier wait is bounded in time; a wait that
// runs out records FA_ERR_TIMEOUT in the optional status word and the CTA
// finishes its schedule (C is then undefined).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "host_common.h"
#include "ptx.cuh"

namespace fa {
namespace gemm {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kABytes = kBM * kBK * 2;            // 16 KiB
constexpr int kBBoxBytes = 64 * kBK * 2;          // 8 KiB: 64 N columns x 64 K rows
constexpr int kStageBytes = kABytes + 4 * kBBoxBytes;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kGroupM = 8;
constexpr uint32_t kTmemCols = 512;
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kSmemBytes = 1024 + kBarOff + 256;  // 1 KiB for aligning the ring
constexpr int kStatusTimeout = -7;                // FA_ERR_TIMEOUT
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr uint64_t kWaitLimitAbortNs = 1000000ull;

static_assert(kSmemBytes <= 232448, "shared memory per CTA");

struct Params {
    const uint16_t* bias;
    uint16_t* c;
    int* status;
    int M, N, num_kb, m_blocks, n_blocks, tiles;
};

__device__ __noinline__ void wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* abort,
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

// Tile t -> (row block, column block), row blocks fastest inside a group of
// kGroupM row blocks.
__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
    const int per_group = kGroupM * p.n_blocks;
    const int g = t / per_group;
    const int first = g * kGroupM;
    const int rows = min(p.m_blocks - first, kGroupM);
    const int r = t - g * per_group;
    mb = first + r % rows;
    nb = r / rows;
}

__device__ __forceinline__ float gelu_erf(float x) {
    return 0.5f * x * (1.f + erff(x * 0.70710678118654752f));
}

template <int MODE>
__device__ __forceinline__ float epilogue_value(float acc, float bias) {
    if constexpr (MODE == 0) return acc;
    else if constexpr (MODE == 1) return acc + bias;
    else return gelu_erf(acc + bias);
}

// One epilogue chunk: 32 accumulator columns col0 .. col0+31 of one row, bias and
// activation in fp32, rounded to bf16 (nearest-even) and stored as 16-byte
// vectors; columns past N and rows past M are not stored.
template <int MODE>
__device__ __forceinline__ void store_chunk(const uint32_t (&r)[32], int row, int col0, const Params& p) {
    if (col0 >= p.N) return;
    uint32_t bw[16];
    if constexpr (MODE > 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (col0 + 8 * i < p.N) v = ld_global_nc_v4(p.bias + col0 + 8 * i);
            bw[4 * i] = v.x;
            bw[4 * i + 1] = v.y;
            bw[4 * i + 2] = v.z;
            bw[4 * i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) bw[i] = 0u;
    }
    uint32_t o[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const float b0 = __uint_as_float(bw[j] << 16);
        const float b1 = __uint_as_float(bw[j] & 0xffff0000u);
        o[j] = pack_bf16x2(epilogue_value<MODE>(__uint_as_float(r[2 * j]), b0),
                           epilogue_value<MODE>(__uint_as_float(r[2 * j + 1]), b1));
    }
    if (row < p.M) {
        uint16_t* dst = p.c + static_cast<int64_t>(row) * p.N + col0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (col0 + 8 * i < p.N)
                *reinterpret_cast<uint4*>(dst + 8 * i) = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    const uint32_t bars = base + kBarOff;
    const auto full = [&](int s) { return bars + 8u * s; };
    const auto empty = [&](int s) { return bars + 8u * (kStages + s); };
    const auto acc_full = [&](int b) { return bars + 8u * (2 * kStages + b); };
    const auto acc_empty = [&](int b) { return bars + 8u * (2 * kStages + 2 + b); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBarOff + 8 * (2 * kStages + 4));
    volatile uint32_t* abort_flag = tmem_slot + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), kEpiWarps);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && p.num_kb > 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            int s = 0;
            uint32_t ph = 0;
            for (int t = blockIdx.x; t < p.tiles; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p, mb, nb);
                const int m0 = mb * kBM, n0 = nb * kBN;
                // B boxes wholly past column N are not loaded; their
                // accumulator columns are never stored.
                const int nbox = min(4, (p.N - n0 + 63) / 64);
                const uint32_t bytes = kABytes + nbox * kBBoxBytes;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    wait_bar(empty(s), ph ^ 1u, abort_flag, p.status);
                    mbar_arrive_expect_tx(full(s), bytes);
                    const uint32_t st = base + s * kStageBytes;
                    tma_load_2d(st, &tm_a, kb * kBK, m0, full(s));
                    for (int i = 0; i < nbox; ++i)
                        tma_load_2d(st + kABytes + i * kBBoxBytes, &tm_b, n0 + 64 * i, kb * kBK, full(s));
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, true);
            int s = 0, tl = 0;
            uint32_t ph = 0;
            for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tl) {
                const int buf = tl & 1;
                const uint32_t use = (tl >> 1) & 1;
                wait_bar(acc_empty(buf), use ^ 1u, abort_flag, p.status);
                tc_fence_after();
                const uint32_t d = tmem + buf * kBN;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    wait_bar(full(s), ph, abort_flag, p.status);
                    tc_fence_after();
                    const uint32_t a_st = base + s * kStageBytes;
                    const uint32_t b_st = a_st + kABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_ss(d, smem_desc_sw128(a_st + 32 * kk, 16, 1024),
                               smem_desc_sw128(b_st + 2048 * kk, kBBoxBytes, 1024), idesc,
                               (kb | kk) != 0 ? 1u : 0u);
                    mma_commit(empty(s));
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (p.num_kb > 0)
                    mma_commit(acc_full(buf));
                else
                    mbar_arrive(acc_full(buf));
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        int tl = 0;
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tl) {
            int mb, nb;
            tile_coords(t, p, mb, nb);
            const int buf = tl & 1;
            const uint32_t use = (tl >> 1) & 1;
            wait_bar(acc_full(buf), use, abort_flag, p.status);
            tc_fence_after();
            const int row = mb * kBM + quarter * 32 + lane;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kBN + half * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                if (p.num_kb > 0) {
                    tmem_ld32(taddr + 32 * c, r);
                    tmem_wait_ld();
                    reg_fence32(r);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) r[j] = 0u;
                }
                if (c == 3) {
                    // every TMEM read of this accumulator is done: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(acc_empty(buf));
                }
                store_chunk<MODE>(r, row, nb * kBN + half * 128 + 32 * c, p);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- two-SM tiles
// A CTA pair (cluster of 2, one CTA per SM of an SM pair) computes a 256 x 256
// tile with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): each CTA stages
// its 128 rows of A and its 128 columns of B (at the same shared-memory
// offsets), the even CTA issues every product, and each CTA receives its 128
// rows of the accumulator (all 256 columns) in its own TMEM.  Per SM that is
// half of B's shared-memory traffic and TMA bytes of the one-SM tile for the
// same tensor work: 64 B per cycle of operand reads and 64 B per cycle of TMA
// writes at the full tensor rate, against 96 + 96 for the one-SM 128 x 256
// tile, which needs more than the 128 B per cycle shared memory delivers.
//
// Pair protocol (every wait bounded):
//   full[s]      of the even CTA: its producer arms it with both CTAs' bytes;
//                both CTAs' TMA loads complete on it.
//   empty[s]     of both CTAs: one multicast commit after the products that
//                read stage s frees the stage in both.
//   acc_full[b]  of both CTAs: multicast commit after the tile's last product.
//   acc_empty[b] of the even CTA: the epilogue warps of both CTAs arrive
//                (the odd CTA's remotely) once they have read accumulator b.
// Before exit each CTA waits for the last arrivals addressed to it, then the
// pair meets at a cluster barrier and frees its TMEM.
constexpr int k2BM = 256, k2Stages = 7;
constexpr int k2ABytes = 128 * kBK * 2;           // 16 KiB: this CTA's 128 rows of A
constexpr int k2BBoxes = 2;                       // this CTA's 128 columns of B: 2 boxes of 64
constexpr int k2StageBytes = k2ABytes + k2BBoxes * kBBoxBytes;   // 32 KiB
constexpr int k2BarOff = k2Stages * k2StageBytes;
constexpr int k2SmemBytes = 1024 + k2BarOff + 256;
static_assert(k2SmemBytes <= 232448, "shared memory per CTA");

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    const uint32_t bars = base + k2BarOff;
    const auto full = [&](int s) { return bars + 8u * s; };
    const auto empty = [&](int s) { return bars + 8u * (k2Stages + s); };
    const auto acc_full = [&](int b) { return bars + 8u * (2 * k2Stages + b); };
    const auto acc_empty = [&](int b) { return bars + 8u * (2 * k2Stages + 2 + b); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + k2BarOff + 8 * (2 * k2Stages + 4));
    volatile uint32_t* abort_flag = tmem_slot + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();      // 0: issues the pair's products
    const int pair = static_cast<int>(blockIdx.x >> 1), pairs = static_cast<int>(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < k2Stages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 2 * kEpiWarps);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish_pair();
    }
    // barriers initialised and TMEM allocated in both CTAs before any CTA of the
    // pair signals the other
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            int s = 0;
            uint32_t ph = 0;
            for (int t = pair; t < p.tiles; t += pairs) {
                int mb, nb;
                tile_coords(t, p, mb, nb);
                const int m0 = mb * k2BM + 128 * static_cast<int>(rank);
                const int n0 = nb * kBN + 128 * static_cast<int>(rank);
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    wait_bar(empty(s), ph ^ 1u, abort_flag, p.status);
                    const uint32_t bar0 = mapa_shared(full(s), 0);
                    if (rank == 0) mbar_arrive_expect_tx(full(s), 2 * k2StageBytes);
                    const uint32_t st = base + s * k2StageBytes;
                    tma_load_2d_pair(st, &tm_a, kb * kBK, m0, bar0);
                    for (int i = 0; i < k2BBoxes; ++i)
                        tma_load_2d_pair(st + k2ABytes + i * kBBoxBytes, &tm_b, n0 + 64 * i, kb * kBK, bar0);
                    if (++s == k2Stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // the last stage releases (multicast commits from the even CTA) have
            // landed in this CTA's barriers before it may exit
            for (int k = 0; k < k2Stages; ++k) {
                wait_bar(empty(s), ph ^ 1u, abort_flag, p.status);
                if (++s == k2Stages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        // The whole warp runs the loop (converged, waits included); one elected
        // lane issues each product and commit.
        if (rank == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(k2BM, kBN, true);
            int s = 0, tl = 0;
            uint32_t ph = 0;
            for (int t = pair; t < p.tiles; t += pairs, ++tl) {
                const int buf = tl & 1;
                const uint32_t use = (tl >> 1) & 1;
                wait_bar(acc_empty(buf), use ^ 1u, abort_flag, p.status);
                tc_fence_after();
                const uint32_t d = tmem + buf * kBN;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    wait_bar(full(s), ph, abort_flag, p.status);
                    tc_fence_after();
                    const uint32_t a_st = base + s * k2StageBytes;
                    const uint32_t b_st = a_st + k2ABytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_ss_pair_elect(d, smem_desc_sw128(a_st + 32 * kk, 16, 1024),
                                    smem_desc_sw128(b_st + 2048 * kk, kBBoxBytes, 1024), idesc,
                                    (kb | kk) != 0 ? 1u : 0u);
                    mma_commit_pair_elect(empty(s), 0x3);
                    if (++s == k2Stages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                mma_commit_pair_elect(acc_full(buf), 0x3);
            }
            // both CTAs' epilogues have released every accumulator (their remote
            // arrivals have landed) before this CTA may exit: wait as if for the
            // next two tiles (a buffer never used passes at once)
            for (int k = 0; k < 2; ++k, ++tl)
                wait_bar(acc_empty(tl & 1), ((tl >> 1) & 1) ^ 1u, abort_flag, p.status);
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        const uint32_t acc_empty0 = mapa_shared(acc_empty(0), 0);
        int tl = 0;
        for (int t = pair; t < p.tiles; t += pairs, ++tl) {
            int mb, nb;
            tile_coords(t, p, mb, nb);
            const int buf = tl & 1;
            const uint32_t use = (tl >> 1) & 1;
            wait_bar(acc_full(buf), use, abort_flag, p.status);
            tc_fence_after();
            const int row = mb * k2BM + 128 * static_cast<int>(rank) + quarter * 32 + lane;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * kBN + half * 128;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(taddr + 32 * c, r);
                tmem_wait_ld();
                reg_fence32(r);
                if (c == 3) {
                    // every TMEM read of this accumulator is done: hand it back to
                    // the even CTA's issuer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * buf);
                }
                store_chunk<MODE>(r, row, nb * kBN + half * 128 + 32 * c, p);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
constexpr int kMaxDevices = 64;
struct DeviceState {
    std::once_flag once;
    int status = FA_OK;
    int sms = 0;
};
DeviceState g_dev[kMaxDevices];

template <int MODE>
int opt_in() {
    return cudaFuncSetAttribute(gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemBytes) == cudaSuccess &&
                   cudaFuncSetAttribute(gemm2_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        k2SmemBytes) == cudaSuccess
               ? FA_OK
               : FA_ERR_CUDA;
}

int device_ready(int& sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    DeviceState& st = g_dev[dev];
    std::call_once(st.once, [&] {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            st.status = FA_ERR_CUDA;
            return;
        }
        if (major != 10 || minor != 0) {
            st.status = FA_ERR_ARCH;
            return;
        }
        int rc;
        if ((rc = opt_in<0>()) != FA_OK || (rc = opt_in<1>()) != FA_OK || (rc = opt_in<2>()) != FA_OK)
            st.status = rc;
    });
    sms = st.sms;
    return st.status;
}

// Row-major bf16 [rows][cols] viewed 2-D with boxes of box_cols x box_rows.
int encode_2d(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, uint32_t box_cols,
              uint32_t box_rows) {
    auto enc = host::tensor_map_encoder();
    if (!enc) return FA_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t elem[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                     box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 256;

// The pair kernel needs a K loop (its even CTA arms every stage), more than one
// 128-row block of A, and at least one SM pair.
bool use_pairs(int64_t M, int64_t K, int sms) { return K > 0 && M > kBM && sms >= 2; }

int run(const void* a, const void* b, const void* bias, void* c, int64_t M, int64_t N, int64_t K,
        int epilogue, int* dev_status, void* stream) {
    if (epilogue < FA_GEMM_PLAIN || epilogue > FA_GEMM_BIAS_GELU) return FA_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return FA_ERR_SHAPE;
    if (M == 0 || N == 0) return FA_OK;
    if (!c || (K > 0 && (!a || !b)) || (epilogue != FA_GEMM_PLAIN && !bias)) return FA_ERR_NULL;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim || N % 8 != 0 || K % 8 != 0) return FA_ERR_SHAPE;
    if ((K > 0 && (!host::aligned(a, 16) || !host::aligned(b, 16))) || !host::aligned(c, 16) ||
        (epilogue != FA_GEMM_PLAIN && !host::aligned(bias, 16)))
        return FA_ERR_ALIGN;
    int sms = 0;
    int rc = device_ready(sms);
    if (rc != FA_OK) return rc;
    alignas(64) CUtensorMap ta{}, tb{};
    if (K > 0) {
        if (encode_2d(&ta, a, M, K, 64, kBM) != FA_OK || encode_2d(&tb, b, K, N, 64, kBK) != FA_OK)
            return FA_ERR_CUDA;
    }
    // 256-row tiles over SM pairs when there is more than one 128-row block of
    // work and a K loop; one-SM 128-row tiles otherwise
    const bool pairs = use_pairs(M, K, sms);
    const int bm = pairs ? k2BM : kBM;
    Params p;
    p.bias = static_cast<const uint16_t*>(bias);
    p.c = static_cast<uint16_t*>(c);
    p.status = dev_status;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.num_kb = static_cast<int>((K + kBK - 1) / kBK);
    p.m_blocks = static_cast<int>((M + bm - 1) / bm);
    p.n_blocks = static_cast<int>((N + kBN - 1) / kBN);
    const int64_t tiles = static_cast<int64_t>(p.m_blocks) * p.n_blocks;
    if (tiles > 0x7fffffffLL) return FA_ERR_SHAPE;
    p.tiles = static_cast<int>(tiles);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pairs) {
        const int64_t npairs = tiles < sms / 2 ? tiles : sms / 2;
        const unsigned grid2 = static_cast<unsigned>(2 * npairs);
        if (epilogue == FA_GEMM_PLAIN)
            gemm2_kernel<0><<<grid2, kThreads, k2SmemBytes, s>>>(ta, tb, p);
        else if (epilogue == FA_GEMM_BIAS)
            gemm2_kernel<1><<<grid2, kThreads, k2SmemBytes, s>>>(ta, tb, p);
        else
            gemm2_kernel<2><<<grid2, kThreads, k2SmemBytes, s>>>(ta, tb, p);
        return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
    if (epilogue == FA_GEMM_PLAIN)
        gemm_kernel<0><<<grid, kThreads, kSmemBytes, s>>>(ta, tb, p);
    else if (epilogue == FA_GEMM_BIAS)
        gemm_kernel<1><<<grid, kThreads, kSmemBytes, s>>>(ta, tb, p);
    else
        gemm_kernel<2><<<grid, kThreads, kSmemBytes, s>>>(ta, tb, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace gemm
}  // namespace fa

extern "C" int fa_gemm(const void* a, const void* b, const void* bias, void* c, int64_t M, int64_t N,
                       int64_t K, int epilogue, int* dev_status, void* stream) {
    return fa::gemm::run(a, b, bias, c, M, N, K, epilogue, dev_status, stream);
}

extern "C" int fa_gemm_launches(int64_t M, int64_t N, int64_t K) {
    (void)K;
    return (M > 0 && N > 0) ? 1 : 0;
}
