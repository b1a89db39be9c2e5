// Row-wise softmax for sm_100a: y[r, :] = softmax(scale * x[r, :]) over bf16
// rows, fp32 arithmetic, bf16 output (round to nearest even).  The row's
// maximum and sum are reduced from register-resident fragments and the
// normalisation stays in registers ("TileLang tutorial", softmax section).
// The operation is bandwidth-bound: the fast path reads each element once and
// writes it once.
//
// Fast path (16-byte aligned rows, cols % 8 == 0, cols <= 16384): a row is held
// by TPR threads (a warp or a group of warps), each keeping VPT 16-byte vectors
// (8 bf16) of packed data in registers; 256 threads per CTA, 256 / TPR rows
// per CTA.  General path (anything else): one CTA per row, an online max/sum
// pass and a normalising pass (two reads, one write).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/fa.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr int kRsThreads = 256;

__device__ __forceinline__ void st_global_cs_v4(void* p, const uint4& v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Reduction over the TPR threads of one row (TPR = 32 * warps, aligned
// groups of warps; scratch: one float per warp of the CTA).
template <int TPR, bool kMax>
__device__ __forceinline__ float row_reduce(float v, float* scratch) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float w = __shfl_xor_sync(0xffffffffu, v, o);
        v = kMax ? fmaxf(v, w) : v + w;
    }
    if constexpr (TPR > 32) {
        constexpr int kWarps = TPR / 32;
        const int warp = threadIdx.x >> 5;
        const int first = warp & ~(kWarps - 1);
        __syncthreads();
        if ((threadIdx.x & 31) == 0) scratch[warp] = v;
        __syncthreads();
        v = scratch[first];
#pragma unroll
        for (int i = 1; i < kWarps; ++i) v = kMax ? fmaxf(v, scratch[first + i]) : v + scratch[first + i];
    }
    return v;
}

template <int TPR, int VPT>
__global__ void __launch_bounds__(kRsThreads) row_softmax_fast(const uint16_t* __restrict__ x,
                                                               uint16_t* __restrict__ y,
                                                               int64_t rows, int cols, float c) {
    __shared__ float scratch[kRsThreads / 32];
    constexpr int kRowsPerCta = kRsThreads / TPR;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + threadIdx.x / TPR;
    const int t = threadIdx.x % TPR;
    const bool row_ok = row < rows;
    const uint16_t* xr = x + (row_ok ? row : 0) * cols;
    uint16_t* yr = y + (row_ok ? row : 0) * cols;

    uint4 v[VPT];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int col = (i * TPR + t) * 8;
        if (row_ok && col < cols) {
            v[i] = ld_global_nc_v4(xr + col);
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) mx = max3f(mx, bf16_lo(w[k]), bf16_hi(w[k]));
        }
    }
    // softmax(c * x) with c = scale * log2(e): the max of c*x is c*max(x) for
    // c >= 0 and c*min(x) otherwise; track both extremes only when needed
    float mn = INFINITY;
    if (c < 0.f) {
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int col = (i * TPR + t) * 8;
            if (row_ok && col < cols) {
                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) mn = fminf(mn, fminf(bf16_lo(w[k]), bf16_hi(w[k])));
            }
        }
    }
    mx = row_reduce<TPR, true>(mx, scratch);
    if (c < 0.f) mn = -row_reduce<TPR, true>(-mn, scratch);
    const float m = (c < 0.f) ? c * mn : c * mx;
    const float neg_m = (m == -INFINITY || m == INFINITY) ? 0.f : -m;

    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int col = (i * TPR + t) * 8;
        if (row_ok && col < cols) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k)
                sum += ex2_approx(fmaf(bf16_lo(w[k]), c, neg_m)) + ex2_approx(fmaf(bf16_hi(w[k]), c, neg_m));
        }
    }
    sum = row_reduce<TPR, false>(sum, scratch);
    const float inv = 1.f / sum;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int col = (i * TPR + t) * 8;
        if (row_ok && col < cols) {
            const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                o[k] = pack_bf16x2(ex2_approx(fmaf(bf16_lo(w[k]), c, neg_m)) * inv,
                                   ex2_approx(fmaf(bf16_hi(w[k]), c, neg_m)) * inv);
            st_global_cs_v4(yr + col, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
}

// Any length and alignment: one CTA per row; online (max, sum) per thread,
// merged across the CTA, then a normalising pass.
__global__ void __launch_bounds__(kRsThreads) row_softmax_general(const uint16_t* __restrict__ x,
                                                                  uint16_t* __restrict__ y,
                                                                  int64_t cols, float c) {
    __shared__ float sm_m[kRsThreads / 32], sm_l[kRsThreads / 32];
    const int64_t row = blockIdx.x;
    const uint16_t* xr = x + row * cols;
    uint16_t* yr = y + row * cols;
    float m = -INFINITY, l = 0.f;
    for (int64_t col = threadIdx.x; col < cols; col += kRsThreads) {
        const float t = c * __uint_as_float(static_cast<uint32_t>(xr[col]) << 16);
        if (t > m) {
            l = (m == -INFINITY) ? 0.f : l * ex2_approx(m - t);
            m = t;
        }
        l += ex2_approx(t - m);
    }
    // merge (m, l) pairs: warp, then CTA
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
        const float mm = fmaxf(m, m2);
        l = (mm == -INFINITY) ? 0.f : l * ex2_approx(m - mm) + l2 * ex2_approx(m2 - mm);
        m = mm;
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        sm_m[warp] = m;
        sm_l[warp] = l;
    }
    __syncthreads();
    m = sm_m[0];
    l = sm_l[0];
#pragma unroll
    for (int i = 1; i < kRsThreads / 32; ++i) {
        const float mm = fmaxf(m, sm_m[i]);
        l = (mm == -INFINITY) ? 0.f : l * ex2_approx(m - mm) + sm_l[i] * ex2_approx(sm_m[i] - mm);
        m = mm;
    }
    const float inv = 1.f / l;
    const float neg_m = (m == -INFINITY || m == INFINITY) ? 0.f : -m;
    for (int64_t col = threadIdx.x; col < cols; col += kRsThreads) {
        const float t = __uint_as_float(static_cast<uint32_t>(xr[col]) << 16);
        const float p = ex2_approx(fmaf(t, c, neg_m)) * inv;
        yr[col] = static_cast<uint16_t>(pack_bf16x2(p, 0.f) & 0xffffu);
    }
}

template <int TPR, int VPT>
cudaError_t launch_fast(const void* x, void* y, int64_t rows, int64_t cols, float c, cudaStream_t s) {
    constexpr int kRowsPerCta = kRsThreads / TPR;
    const int64_t grid = (rows + kRowsPerCta - 1) / kRowsPerCta;
    row_softmax_fast<TPR, VPT><<<static_cast<unsigned>(grid), kRsThreads, 0, s>>>(
        static_cast<const uint16_t*>(x), static_cast<uint16_t*>(y), rows, static_cast<int>(cols), c);
    return cudaGetLastError();
}

}  // namespace
}  // namespace fa

extern "C" int fa_row_softmax(const void* x, void* y, int64_t rows, int64_t cols, float scale,
                              void* stream) {
    if (rows < 0 || cols < 0) return FA_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FA_OK;
    if (!x || !y) return FA_ERR_NULL;
    if (rows > 0x7fffffffLL || cols > (int64_t(1) << 31) - 1 || rows * cols > (int64_t(1) << 62))
        return FA_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(x) & 1) || (reinterpret_cast<uintptr_t>(y) & 1)) return FA_ERR_ALIGN;
    if (!std::isfinite(scale)) return FA_ERR_SCALE;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return FA_ERR_CUDA;
    if (major != 10) return FA_ERR_ARCH;
    const float c = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool vec = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (reinterpret_cast<uintptr_t>(y) % 16 == 0) &&
                     (cols % 8 == 0);
    cudaError_t e;
    if (vec && cols <= 256)
        e = fa::launch_fast<32, 1>(x, y, rows, cols, c, s);
    else if (vec && cols <= 512)
        e = fa::launch_fast<32, 2>(x, y, rows, cols, c, s);
    else if (vec && cols <= 1024)
        e = fa::launch_fast<32, 4>(x, y, rows, cols, c, s);
    else if (vec && cols <= 2048)
        e = fa::launch_fast<64, 4>(x, y, rows, cols, c, s);
    else if (vec && cols <= 4096)
        e = fa::launch_fast<128, 4>(x, y, rows, cols, c, s);
    else if (vec && cols <= 8192)
        e = fa::launch_fast<256, 4>(x, y, rows, cols, c, s);
    else if (vec && cols <= 16384)
        e = fa::launch_fast<256, 8>(x, y, rows, cols, c, s);
    else {
        fa::row_softmax_general<<<static_cast<unsigned>(rows), fa::kRsThreads, 0, s>>>(
            static_cast<const uint16_t*>(x), static_cast<uint16_t*>(y), cols, c);
        e = cudaGetLastError();
    }
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" int fa_row_softmax_launches(int64_t rows, int64_t cols) {
    return (rows > 0 && cols > 0) ? 1 : 0;
}
