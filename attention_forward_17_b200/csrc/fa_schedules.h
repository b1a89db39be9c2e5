// Registry of the compiled schedules of the attention kernel.  A schedule is
// one instantiation of fa_fwd_kernel<D, CAUSAL, EMU, SLOTS, PERSIST> for both
// masking modes; the host picks one per problem from the table the schedule search
// writes (fa_schedule_table.h) or as the caller asks (fa_fwd_schedule).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_fwd_kernel.cuh"
#include "fa_fwd_pp_kernel.cuh"
#include "fa_fwd_2q_kernel.cuh"

namespace fa {

// tq, tk, tv: the Q, K, V maps; to: the same view of O (used by the kernels
// that store O with TMA).
using FwdLaunchFn = cudaError_t (*)(const CUtensorMap& tq, const CUtensorMap& tk,
                                    const CUtensorMap& tv, const CUtensorMap& to, const FwdParams& p,
                                    unsigned grid, cudaStream_t stream);

struct Schedule {
    int d;             // head dimension
    int emu;           // every emu-th exponential pair on the FMA pipe (0 = none)
    int slots;         // K/V ring depth
    int persist;       // launch form: 0 one tile per CTA, 1 persistent (static), 2 persistent by
                       // cluster launch control (tiles taken over from unlaunched CTAs)
    int alg;           // 0: one softmax pass over every key tile; 1: split-KV ping-pong
                       // (two softmax groups take alternate key tiles, merged at the end);
                       // 2: two query tiles per CTA, P over S in TMEM, one score buffer per
                       // tile; 3: the same with two score buffers per tile (scores of
                       // the next key tile computed while the softmax works); 4, 5: as
                       // 2, 3 with the sum of the bf16 weights on the tensor core; 6 to 9:
                       // as 2 to 5 with P released as 3/4 and then 1/4 of the keys; + 8:
                       // three query tiles per CTA instead of two
    int smem_bytes;    // dynamic shared memory per CTA
    int bn;            // rows of a key/value tile (128 except for the two-query-tile algorithms)
    FwdLaunchFn launch[2];   // [causal]
    int (*setup)();          // shared-memory opt-in and register check, both modes
};

// Defined in fa_fwd_sched_d128.cu and fa_fwd_sched_d64.cu; the first entry of
// each list is that head dimension's default.
const Schedule* schedules_d128(int* count);
const Schedule* schedules_d64(int* count);

// Shared by both definition files.
template <int D, bool CAUSAL, int EMU, int SLOTS>
cudaError_t launch_pp(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      const CUtensorMap&, const FwdParams& p, unsigned grid, cudaStream_t stream) {
    fa_fwd_pp_kernel<D, CAUSAL, EMU, SLOTS>
        <<<grid, kThreads, PPCfg<D, SLOTS>::kSmemBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <int D, bool CAUSAL, int EMU, int SLOTS>
int setup_pp_one() {
    auto* k = fa_fwd_pp_kernel<D, CAUSAL, EMU, SLOTS>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PPCfg<D, SLOTS>::kSmemBytes) != cudaSuccess)
        return -6;
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, k) != cudaSuccess) return -6;
    if (attr.numRegs * kThreads < kRegSplitTotal) return -6;
    return 0;
}

template <int D, int EMU, int SLOTS>
int setup_pp_both() {
    const int rc = setup_pp_one<D, false, EMU, SLOTS>();
    return rc ? rc : setup_pp_one<D, true, EMU, SLOTS>();
}

template <int D, int EMU, int SLOTS>
constexpr Schedule make_pp_schedule() {
    return Schedule{D,
                    EMU,
                    SLOTS,
                    0,
                    1,
                    PPCfg<D, SLOTS>::kSmemBytes,
                    128,
                    {&launch_pp<D, false, EMU, SLOTS>, &launch_pp<D, true, EMU, SLOTS>},
                    &setup_pp_both<D, EMU, SLOTS>};
}

template <int D, bool CAUSAL, int EMU, int SLOTS, int BN, bool DB, bool LT, bool P34, int NT>
cudaError_t launch_2q(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      const CUtensorMap& to, const FwdParams& p, unsigned grid, cudaStream_t stream) {
    fa_fwd_2q_kernel<D, CAUSAL, EMU, SLOTS, BN, DB, LT, P34, NT>
        <<<grid, Q2Roles<NT>::kThreads, Q2Cfg<D, SLOTS, BN, DB, LT, NT>::kSmemBytes, stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError();
}

template <int D, bool CAUSAL, int EMU, int SLOTS, int BN, bool DB, bool LT, bool P34, int NT>
int setup_2q_one() {
    auto* k = fa_fwd_2q_kernel<D, CAUSAL, EMU, SLOTS, BN, DB, LT, P34, NT>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Q2Cfg<D, SLOTS, BN, DB, LT, NT>::kSmemBytes) != cudaSuccess)
        return -6;
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, k) != cudaSuccess) return -6;
    if (attr.numRegs * Q2Roles<NT>::kThreads < Q2Roles<NT>::kRegTotal) return -6;
    return 0;
}

template <int D, int EMU, int SLOTS, int BN, bool DB, bool LT, bool P34, int NT>
int setup_2q_both() {
    const int rc = setup_2q_one<D, false, EMU, SLOTS, BN, DB, LT, P34, NT>();
    return rc ? rc : setup_2q_one<D, true, EMU, SLOTS, BN, DB, LT, P34, NT>();
}

// Several query tiles per CTA (fa_fwd_2q_kernel), key tiles of BN rows:
// algorithm 2 (two query tiles, one score buffer per tile), + 1 with two score
// buffers per tile (DB), + 2 with the sum of the bf16 weights accumulated by the
// tensor core (LT), + 4 with P released as three quarters and one quarter of the
// keys (P34), + 8 with three query tiles per CTA (NT = 3).
template <int D, int EMU, int SLOTS, int BN = 128, bool DB = false, bool LT = false, bool P34 = false,
          int NT = 2>
constexpr Schedule make_2q_schedule() {
    return Schedule{D,
                    EMU,
                    SLOTS,
                    0,
                    2 + (DB ? 1 : 0) + (LT ? 2 : 0) + (P34 ? 4 : 0) + (NT == 3 ? 8 : 0),
                    Q2Cfg<D, SLOTS, BN, DB, LT, NT>::kSmemBytes,
                    BN,
                    {&launch_2q<D, false, EMU, SLOTS, BN, DB, LT, P34, NT>,
                     &launch_2q<D, true, EMU, SLOTS, BN, DB, LT, P34, NT>},
                    &setup_2q_both<D, EMU, SLOTS, BN, DB, LT, P34, NT>};
}

// Query tiles per CTA of a schedule's algorithm.
constexpr int tiles_per_cta(int alg) { return alg < 2 ? 1 : (((alg - 2) & 8) ? 3 : 2); }

template <int D, bool CAUSAL, int EMU, int SLOTS, int PERSIST>
cudaError_t launch_schedule(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap&, const FwdParams& p, unsigned grid,
                            cudaStream_t stream) {
    fa_fwd_kernel<D, CAUSAL, EMU, SLOTS, PERSIST>
        <<<grid, kThreads, TileCfg<D, SLOTS>::kSmemBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

// Opts the instantiation into its dynamic shared memory and checks that it
// was compiled with enough registers for the in-kernel warpgroup rebalance (a
// setmaxnreg.inc asking for more than the launch allocated would never
// return).  Returns 0 (FA_OK), -6 (FA_ERR_CUDA).
template <int D, bool CAUSAL, int EMU, int SLOTS, int PERSIST>
int setup_one() {
    auto* k = fa_fwd_kernel<D, CAUSAL, EMU, SLOTS, PERSIST>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             TileCfg<D, SLOTS>::kSmemBytes) != cudaSuccess)
        return -6;
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, k) != cudaSuccess) return -6;
    if (attr.numRegs * kThreads < kRegSplitTotal) return -6;
    return 0;
}

template <int D, int EMU, int SLOTS, int PERSIST>
int setup_both() {
    const int rc = setup_one<D, false, EMU, SLOTS, PERSIST>();
    return rc ? rc : setup_one<D, true, EMU, SLOTS, PERSIST>();
}

template <int D, int EMU, int SLOTS, int PERSIST = 0>
constexpr Schedule make_schedule() {
    static_assert(TileCfg<D, SLOTS>::kSmemBytes <= 232448, "shared memory per CTA (227 KiB)");
    static_assert(TileCfg<D, SLOTS>::kTmemCols <= 512, "tensor memory columns");
    return Schedule{D,
                    EMU,
                    SLOTS,
                    PERSIST,
                    0,
                    TileCfg<D, SLOTS>::kSmemBytes,
                    128,
                    {&launch_schedule<D, false, EMU, SLOTS, PERSIST>,
                     &launch_schedule<D, true, EMU, SLOTS, PERSIST>},
                    &setup_both<D, EMU, SLOTS, PERSIST>};
}

}  // namespace fa
