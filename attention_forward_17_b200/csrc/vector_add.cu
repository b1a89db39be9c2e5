// Elementwise vector addition z = x + y over fp32 ("TileLang tutorial", the
// vector-add kernel its first section uses as a memory-bandwidth probe).
//
// Pure streaming: 12 bytes of HBM traffic per element, no reuse, so the kernel
// is sized for bytes in flight rather than arithmetic.  A grid of 8 CTAs of
// 256 threads per SM strides over the arrays in 16-byte vectors, four vectors
// per operand per iteration (loads that bypass L1, streaming stores).  When a
// pointer is not 16-byte aligned a scalar grid-stride loop does the whole job.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "host_common.h"
#include "ptx.cuh"

namespace fa {
namespace vadd {

constexpr int kThreads = 256;
constexpr int kCtasPerSm = 8;
constexpr int kUnroll = 4;

__device__ __forceinline__ void st_cs_v4(void* p, const uint4& v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 add4(const uint4& a, const uint4& b) {
    return make_uint4(__float_as_uint(__uint_as_float(a.x) + __uint_as_float(b.x)),
                      __float_as_uint(__uint_as_float(a.y) + __uint_as_float(b.y)),
                      __float_as_uint(__uint_as_float(a.z) + __uint_as_float(b.z)),
                      __float_as_uint(__uint_as_float(a.w) + __uint_as_float(b.w)));
}

// n4 = number of whole 4-float vectors; the n % 4 tail is added by the first
// threads of CTA 0.
__global__ void __launch_bounds__(kThreads) vector_add_v4(const float* __restrict__ x,
                                                          const float* __restrict__ y,
                                                          float* __restrict__ z, int64_t n) {
    const int64_t n4 = n >> 2;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
    for (; i + (kUnroll - 1) * stride < n4; i += kUnroll * stride) {
        uint4 a[kUnroll], b[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            a[u] = ld_global_nc_v4(x + 4 * (i + u * stride));
            b[u] = ld_global_nc_v4(y + 4 * (i + u * stride));
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) st_cs_v4(z + 4 * (i + u * stride), add4(a[u], b[u]));
    }
    for (; i < n4; i += stride)
        st_cs_v4(z + 4 * i, add4(ld_global_nc_v4(x + 4 * i), ld_global_nc_v4(y + 4 * i)));
    if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
        const int64_t j = 4 * n4 + threadIdx.x;
        z[j] = x[j] + y[j];
    }
}

__global__ void __launch_bounds__(kThreads) vector_add_scalar(const float* __restrict__ x,
                                                              const float* __restrict__ y,
                                                              float* __restrict__ z, int64_t n) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride)
        z[i] = x[i] + y[i];
}

constexpr int kMaxDevices = 64;
struct DeviceState {
    std::once_flag once;
    int status = FA_OK;
    int sms = 0;
};
DeviceState g_dev[kMaxDevices];

int device_ready(int& sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    DeviceState& st = g_dev[dev];
    std::call_once(st.once, [&] {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            st.status = FA_ERR_CUDA;
        else if (major != 10)
            st.status = FA_ERR_ARCH;
    });
    sms = st.sms;
    return st.status;
}

}  // namespace vadd
}  // namespace fa

extern "C" int fa_vector_add(const float* x, const float* y, float* z, int64_t n, void* stream) {
    if (n < 0) return FA_ERR_SHAPE;
    if (n == 0) return FA_OK;
    if (!x || !y || !z) return FA_ERR_NULL;
    if (n > (int64_t(1) << 40)) return FA_ERR_SHAPE;
    using fa::host::aligned;
    if (!aligned(x, 4) || !aligned(y, 4) || !aligned(z, 4)) return FA_ERR_ALIGN;
    int sms = 0;
    const int rc = fa::vadd::device_ready(sms);
    if (rc != FA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t want = (n + 4LL * fa::vadd::kThreads - 1) / (4LL * fa::vadd::kThreads);
    const int64_t cap = static_cast<int64_t>(sms) * fa::vadd::kCtasPerSm;
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    if (aligned(x, 16) && aligned(y, 16) && aligned(z, 16))
        fa::vadd::vector_add_v4<<<grid, fa::vadd::kThreads, 0, s>>>(x, y, z, n);
    else
        fa::vadd::vector_add_scalar<<<grid, fa::vadd::kThreads, 0, s>>>(x, y, z, n);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

extern "C" int fa_vector_add_launches(int64_t n) { return n > 0 ? 1 : 0; }
