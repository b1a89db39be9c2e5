// Host side of the fused attention forward library: argument checks, TMA
// descriptor encoding, kernel selection and launch.  Implements include/fa.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "fa_fwd_kernel.cuh"
#include "host_common.h"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    std::once_flag once;
    int status = FA_OK;   // outcome of the one-time set-up for this device
};
DeviceState g_devices[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Opts the instantiation into its dynamic shared memory and checks that it was
// compiled with enough registers for the in-kernel warpgroup rebalance (a
// setmaxnreg.inc asking for more than the launch allocated would never
// return).
template <int D, bool CAUSAL>
int set_smem_attr() {
    if (cudaFuncSetAttribute(fa::fa_fwd_kernel<D, CAUSAL>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::TileCfg<D>::kSmemBytes) != cudaSuccess)
        return FA_ERR_CUDA;
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, fa::fa_fwd_kernel<D, CAUSAL>) != cudaSuccess) return FA_ERR_CUDA;
    if (attr.numRegs * fa::kThreads < fa::kRegSplitTotal) return FA_ERR_CUDA;
    return FA_OK;
}

// One-time per-device set-up: architecture check and the shared-memory opt-in
// of every kernel instantiation.
int device_setup(int dev) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return FA_ERR_CUDA;
    if (major != 10 || minor != 0) return FA_ERR_ARCH;
    int rc;
    if ((rc = set_smem_attr<64, false>()) != FA_OK || (rc = set_smem_attr<64, true>()) != FA_OK ||
        (rc = set_smem_attr<128, false>()) != FA_OK || (rc = set_smem_attr<128, true>()) != FA_OK)
        return rc;
    return FA_OK;
}

int current_device_ready() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    DeviceState& st = g_devices[dev];
    std::call_once(st.once, [&] { st.status = device_setup(dev); });
    return st.status;
}

int encoder_ready() {
    g_encode = fa::host::tensor_map_encoder();
    return g_encode ? FA_OK : FA_ERR_CUDA;
}

// 3-D view [BH][N][d] of a bf16 tensor; boxes of 128 rows x 64 columns
// (128 bytes, matching the 128-byte swizzle); rows past N read as zero.
int encode_qkv_map(CUtensorMap* map, const void* ptr, int64_t BH, int64_t N, int64_t d) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(N * d * 2)};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t elem[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                          strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

using fa::host::aligned;

constexpr int64_t kMaxN = (int64_t(1) << 31) - 512;
constexpr int64_t kMaxBH = (int64_t(1) << 31) - 1;

// Checks that need no device, in the documented order.  Returns 1 for an
// empty problem (nothing to do), 0 to proceed, or a negative status.
int check_args(const void* q, const void* k, const void* v, const void* o, const void* lse,
               int64_t B, int64_t H, int64_t N, int64_t d, float scale) {
    if (B < 0 || H < 0 || N < 0) return FA_ERR_SHAPE;
    if (B == 0 || H == 0 || N == 0) return 1;
    if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
    if (N > kMaxN || B > kMaxBH || H > kMaxBH || B * H > kMaxBH) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_ALIGN;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_SCALE;
    return 0;
}

template <int D, bool CAUSAL>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const fa::FwdParams& p, int64_t grid, cudaStream_t stream) {
    fa::fa_fwd_kernel<D, CAUSAL><<<static_cast<unsigned>(grid), fa::kThreads,
                                   fa::TileCfg<D>::kSmemBytes, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

int run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
            int64_t N, int64_t d, int causal, float scale, int* dev_status, void* stream) {
    int rc = check_args(q, k, v, o, lse, B, H, N, d, scale);
    if (rc == 1) return FA_OK;
    if (rc != 0) return rc;
    if ((rc = current_device_ready()) != FA_OK) return rc;
    if ((rc = encoder_ready()) != FA_OK) return rc;
    const int64_t BH = B * H;
    alignas(64) CUtensorMap tq, tk, tv;
    if (encode_qkv_map(&tq, q, BH, N, d) || encode_qkv_map(&tk, k, BH, N, d) ||
        encode_qkv_map(&tv, v, BH, N, d))
        return FA_ERR_CUDA;
    fa::FwdParams p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.status = dev_status;
    p.N = static_cast<int>(N);
    p.BH = static_cast<int>(BH);
    p.n_qtile = static_cast<int>((N + fa::kBlockM - 1) / fa::kBlockM);
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    const int64_t grid = BH * p.n_qtile;
    if (grid > 0x7fffffffLL) return FA_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (d == 64)
        e = causal ? launch<64, true>(tq, tk, tv, p, grid, s) : launch<64, false>(tq, tk, tv, p, grid, s);
    else
        e = causal ? launch<128, true>(tq, tk, tv, p, grid, s)
                   : launch<128, false>(tq, tk, tv, p, grid, s);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
           int64_t N, int64_t d, int causal, float scale, void* stream) {
    return run_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, nullptr, stream);
}

int fa_fwd_status(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                  int64_t H, int64_t N, int64_t d, int causal, float scale, int* dev_status,
                  void* stream) {
    return run_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, dev_status, stream);
}

int fa_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h, float* lse_h,
                void* q_d, void* k_d, void* v_d, void* o_d, float* lse_d, int64_t B, int64_t H,
                int64_t N, int64_t d, int causal, float scale, void* stream) {
    int rc = check_args(q_d, k_d, v_d, o_d, lse_d, B, H, N, d, scale);
    if (rc == 1) return FA_OK;
    if (rc != 0) return rc;
    if (!q_h || !k_h || !v_h || !o_h || !lse_h) return FA_ERR_NULL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t tensor_bytes = static_cast<size_t>(B * H * N * d) * 2;
    const size_t lse_bytes = static_cast<size_t>(B * H * N) * 4;
    if (cudaMemcpyAsync(q_d, q_h, tensor_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(k_d, k_h, tensor_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaMemcpyAsync(v_d, v_h, tensor_bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return FA_ERR_CUDA;
    rc = run_fwd(q_d, k_d, v_d, o_d, lse_d, B, H, N, d, causal, scale, nullptr, stream);
    if (rc != FA_OK) return rc;
    if (cudaMemcpyAsync(o_h, o_d, tensor_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyAsync(lse_h, lse_d, lse_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return FA_ERR_CUDA;
    return FA_OK;
}

int fa_selftest_wait_timeout(int* dev_status, int64_t limit_us, int arrive, void* stream) {
    if (!dev_status) return FA_ERR_NULL;
    if (limit_us < 1 || limit_us > 10000000) return FA_ERR_SHAPE;
    int rc = current_device_ready();
    if (rc != FA_OK) return rc;
    fa::fa_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        dev_status, static_cast<uint64_t>(limit_us) * 1000ull, arrive ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fwd_launches(int64_t B, int64_t H, int64_t N, int64_t d) {
    (void)d;
    return (B > 0 && H > 0 && N > 0) ? 1 : 0;
}

const char* fa_strerror(int status) {
    switch (status) {
        case FA_OK: return "ok";
        case FA_ERR_NULL: return "a required pointer is NULL";
        case FA_ERR_SHAPE: return "B, H or N is negative or beyond the supported range";
        case FA_ERR_HEADDIM: return "head dimension d must be 64 or 128";
        case FA_ERR_ALIGN: return "q, k, v, o must be 16-byte aligned and lse 4-byte aligned";
        case FA_ERR_SCALE: return "scale must be finite and greater than zero";
        case FA_ERR_CUDA: return "a CUDA runtime or driver call failed";
        case FA_ERR_TIMEOUT: return "a device-side pipeline wait ran out of time";
        case FA_ERR_ARCH: return "the current device is not an sm_100 (B200-class) GPU";
        case FA_ERR_ARG: return "an enumerated argument is out of range";
        default: return "unknown status";
    }
}

int fa_version(void) { return (1 << 16) | 0; }

}  // extern "C"
