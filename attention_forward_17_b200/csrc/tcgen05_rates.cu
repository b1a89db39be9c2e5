// Standalone measurement of the tcgen05.mma properties the attention kernel's
// schedule is built on (not part of libfa_b200.so):
//   1. streaming rate of M=128 K=16 bf16 products for N = 64 / 128 / 256, with
//      both operands in shared memory (SS) or A in tensor memory (TS);
//   2. the time one thread needs to issue k products into an idle pipe;
//   3. the latency of a dependent burst (issue 8 products, commit, wait);
//   4. one versus two issuing threads when the products are short (N = 64).
// One CTA per SM on every SM; cycles from clock64, averaged over the SMs.
//
// Build and run:  nvcc -gencode arch=compute_100a,code=sm_100a -O2 -std=c++17 \
//                      tcgen05_rates.cu -o tcgen05_rates && ./tcgen05_rates
#include <cuda_runtime.h>

#include <cstdio>

#include "ptx.cuh"

using namespace fa;

namespace {

constexpr int kSms = 148;
constexpr int kSmemBytes = 16384 + 256 * 128 + 2048;

struct Shared {
    uint32_t base;
    uint32_t tmem;
    uint32_t bar;
};

__device__ Shared setup(uint8_t* smem_raw, int nthreads) {
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw);
    for (int i = threadIdx.x; i < (16384 + 256 * 128) / 16; i += nthreads)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3f803f80u, 0x3f003f00u, 0xbf803f80u, 0x3f80bf00u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 16384 + 256 * 128);
    uint32_t* tb = reinterpret_cast<uint32_t*>(smem + 16384 + 256 * 128 + 64);
    if (threadIdx.x == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars[i]), 1);
        fence_barrier_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x < 32) {
        tmem_alloc(smem_u32(tb), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    return Shared{base, *tb, smem_u32(&bars[0])};
}

__device__ void teardown(uint32_t tmem) {
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

__device__ void wait_bounded(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_timer_ns() - t0 > 1000000000ull) break;
}

__device__ __forceinline__ void issue(bool ts, uint32_t tmem, uint32_t base, uint32_t idesc, int kk,
                                      uint32_t d_col) {
    const uint64_t b = smem_desc_sw128(base + 16384 + (kk & 3) * 32, 16, 1024);
    if (ts)
        mma_ts(tmem + d_col, tmem + (kk & 7) * 8, b, idesc, 1);
    else
        mma_ss(tmem + d_col, smem_desc_sw128(base + (kk & 3) * 32, 16, 1024), b, idesc, 1);
}

// 1. streaming: 4000 x 4 products back to back
template <int N, bool TS>
__global__ void __launch_bounds__(128, 1) k_stream(unsigned long long* out) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Shared sh = setup(smem_raw, 128);
    if (threadIdx.x == 0) {
        constexpr uint32_t id = idesc_bf16_f32(128, N, false);
        unsigned long long t0 = 0;
        for (int it = 0; it < 4008; ++it) {
            if (it == 8) t0 = clock64();
            for (int kk = 0; kk < 4; ++kk) issue(TS, sh.tmem, sh.base, id, kk, 256);
        }
        mma_commit(sh.bar);
        wait_bounded(sh.bar, 0);
        out[blockIdx.x] = (clock64() - t0) / (4000ull * 4ull);
    }
    __syncwarp();
    teardown(sh.tmem);
}

// 2 + 3. k products into an idle pipe: issue time, and issue + commit + wait
template <int K>
__global__ void __launch_bounds__(128, 1) k_burst(unsigned long long* out) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Shared sh = setup(smem_raw, 128);
    if (threadIdx.x == 0) {
        constexpr uint32_t id = idesc_bf16_f32(128, 128, true);
        unsigned long long ti = 0, tc = 0;
        for (int b = 0; b < 104; ++b) {
            const unsigned long long g = clock64();
            while (clock64() - g < 2000ull) {
            }
            const unsigned long long t0 = clock64();
            for (int kk = 0; kk < K; ++kk) issue(true, sh.tmem, sh.base, id, kk, 256);
            const unsigned long long t1 = clock64();
            mma_commit(sh.bar);
            wait_bounded(sh.bar, b & 1);
            const unsigned long long t2 = clock64();
            if (b >= 4) {
                ti += t1 - t0;
                tc += t2 - t0;
            }
        }
        out[2 * blockIdx.x] = ti / 100;
        out[2 * blockIdx.x + 1] = tc / 100;
    }
    __syncwarp();
    teardown(sh.tmem);
}

// 4. NW issuing threads (warps 0..NW-1), N = 64 products into separate accumulators
template <int NW>
__global__ void __launch_bounds__(128, 1) k_issuers(unsigned long long* out) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const Shared sh = setup(smem_raw, 128);
    const int w = threadIdx.x / 32;
    if (w < NW && (threadIdx.x & 31) == 0) {
        constexpr uint32_t id = idesc_bf16_f32(128, 64, true);
        unsigned long long t0 = 0;
        for (int it = 0; it < 1004; ++it) {
            if (it == 4) t0 = clock64();
            for (int kk = 0; kk < 4; ++kk) issue(true, sh.tmem, sh.base, id, kk, 256 + 64 * w);
        }
        mma_commit(sh.bar + 8 * w);
        wait_bounded(sh.bar + 8 * w, 0);
        out[4 * blockIdx.x + w] = clock64() - t0;
    }
    __syncwarp();
    teardown(sh.tmem);
}

template <class F>
double run(F kern, unsigned long long* d, int stride, int field) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    cudaMemset(d, 0, kSms * 4 * sizeof(unsigned long long));
    kern<<<kSms, 128, kSmemBytes>>>(d);
    if (cudaDeviceSynchronize() != cudaSuccess) return -1.0;
    unsigned long long h[kSms * 4];
    cudaMemcpy(h, d, sizeof(h), cudaMemcpyDeviceToHost);
    double s = 0;
    for (int i = 0; i < kSms; ++i) s += h[i * stride + field];
    return s / kSms;
}

}  // namespace

int main() {
    unsigned long long* d = nullptr;
    if (cudaMalloc(&d, kSms * 4 * sizeof(unsigned long long)) != cudaSuccess) return 1;
    std::printf("1. streaming, cycles per product (M=128, K=16, bf16 -> fp32)\n");
    std::printf("   SS N=64 %6.1f   N=128 %6.1f   N=256 %6.1f\n", run(k_stream<64, false>, d, 1, 0),
                run(k_stream<128, false>, d, 1, 0), run(k_stream<256, false>, d, 1, 0));
    std::printf("   TS N=64 %6.1f   N=128 %6.1f   N=256 %6.1f\n", run(k_stream<64, true>, d, 1, 0),
                run(k_stream<128, true>, d, 1, 0), run(k_stream<256, true>, d, 1, 0));
    std::printf("2./3. k TS products (N=128) into an idle pipe: issue cycles | issue+commit+wait cycles\n");
    std::printf("   k=1  %6.0f | %6.0f\n", run(k_burst<1>, d, 2, 0), run(k_burst<1>, d, 2, 1));
    std::printf("   k=2  %6.0f | %6.0f\n", run(k_burst<2>, d, 2, 0), run(k_burst<2>, d, 2, 1));
    std::printf("   k=4  %6.0f | %6.0f\n", run(k_burst<4>, d, 2, 0), run(k_burst<4>, d, 2, 1));
    std::printf("   k=8  %6.0f | %6.0f\n", run(k_burst<8>, d, 2, 0), run(k_burst<8>, d, 2, 1));
    std::printf("   k=16 %6.0f | %6.0f\n", run(k_burst<16>, d, 2, 0), run(k_burst<16>, d, 2, 1));
    const double one = run(k_issuers<1>, d, 4, 0) / 4000.0;
    const double two = run(k_issuers<2>, d, 4, 0) / 8000.0;
    std::printf("4. N=64 TS products, cycles per product over all issuers: 1 issuer %5.1f, 2 issuers %5.1f\n",
                one, two);
    cudaFree(d);
    return 0;
}
