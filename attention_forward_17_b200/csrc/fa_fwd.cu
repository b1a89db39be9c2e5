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
#include "fa_schedule_table.h"
#include "fa_schedules.h"
#include "host_common.h"

namespace fa {
// Exercises the bounded wait on an mbarrier that nothing ever arrives at: the
// wait must give up after `limit_ns` and leave FA_ERR_TIMEOUT in *status.
// With `arrive` set, one thread completes the phase first and the wait must
// return at once with *status untouched.  One CTA of 32 threads.
__global__ void fa_wait_selftest_kernel(int* status, uint64_t limit_ns, int arrive) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0u;
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0 && arrive) mbar_arrive(smem_u32(&bar));
    __syncwarp();
    if (!mbar_try_wait(smem_u32(&bar), 0))
        wait_slow(smem_u32(&bar), 0, &abort_flag, status, limit_ns, limit_ns);
}
}  // namespace fa

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    std::once_flag once;
    int status = FA_OK;   // outcome of the one-time set-up for this device
    int sms = 0;          // streaming multiprocessors (persistent grid size)
};
DeviceState g_devices[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// The copy streams and events of fa_fwd_host's pipelined path, one set per
// device, created on first use and kept for the life of the process.
constexpr int kHostChunks = 8;
struct HostPipe {
    std::mutex mu;
    std::once_flag once;
    int status = FA_OK;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t ev[2 * kHostChunks + 2] = {};
};
HostPipe g_pipes[kMaxDevices];

int host_pipe(HostPipe** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    HostPipe& hp = g_pipes[dev];
    std::call_once(hp.once, [&] {
        bool ok = cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) == cudaSuccess;
        for (int i = 0; ok && i < 2 * kHostChunks + 2; ++i)
            ok = cudaEventCreateWithFlags(&hp.ev[i], cudaEventDisableTiming) == cudaSuccess;
        hp.status = ok ? FA_OK : FA_ERR_CUDA;
    });
    *out = &hp;
    return hp.status;
}

// Every compiled schedule, head dimension 128 first, then 64.  Ids are
// positions in this list.
struct ScheduleList {
    const fa::Schedule* items[64];
    int count = 0;
    ScheduleList() {
        int n = 0;
        const fa::Schedule* a = fa::schedules_d128(&n);
        for (int i = 0; i < n && count < 64; ++i) items[count++] = &a[i];
        const fa::Schedule* b = fa::schedules_d64(&n);
        for (int i = 0; i < n && count < 64; ++i) items[count++] = &b[i];
    }
};
const ScheduleList& schedules() {
    static const ScheduleList list;
    return list;
}

// One-time per-device set-up: architecture check and the shared-memory opt-in
// of every kernel instantiation.
int device_setup(int dev) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return FA_ERR_CUDA;
    if (major != 10 || minor != 0) return FA_ERR_ARCH;
    const ScheduleList& list = schedules();
    for (int i = 0; i < list.count; ++i) {
        const int rc = list.items[i]->setup();
        if (rc != FA_OK) return rc;
    }
    return FA_OK;
}

// The schedule id fa_fwd uses for (N, d, causal), and the causal launch group.
void pick_schedule(int64_t N, int64_t d, int causal, int* id, int* group) {
    const ScheduleList& list = schedules();
    int emu = -1, slots = -1, grp = 1, persist = 0, alg = 0, bn = 128;
    for (const auto& e : fa::kScheduleTable)
        if (e.d == d && e.causal == (causal ? 1 : 0) && N <= e.n_max) {
            emu = e.emu;
            slots = e.slots;
            grp = e.group;
            persist = e.persist;
            alg = e.alg;
            bn = e.bn;
            break;
        }
    int match = -1;
    for (int i = 0; i < list.count; ++i) {
        const fa::Schedule* s = list.items[i];
        if (s->d == d && s->emu == emu && s->slots == slots && s->persist == persist &&
            s->alg == alg && s->bn == bn) {
            match = i;
            break;
        }
    }
    // -1 when the table names a schedule that is not compiled (a build
    // inconsistency that the tests rule out; run_fwd then refuses to launch)
    *id = match;
    *group = grp > 0 ? grp : 1;
}

int current_device_ready(int* sms = nullptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
    DeviceState& st = g_devices[dev];
    std::call_once(st.once, [&] {
        st.status = device_setup(dev);
        if (st.status == FA_OK &&
            cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            st.status = FA_ERR_CUDA;
    });
    if (sms) *sms = st.sms;
    return st.status;
}

int encoder_ready() {
    g_encode = fa::host::tensor_map_encoder();
    return g_encode ? FA_OK : FA_ERR_CUDA;
}

// 3-D view [BH][N][d] of a bf16 tensor; boxes of `rows` rows x 64 columns
// (128 bytes, matching the 128-byte swizzle); rows past N read as zero and
// are not written by stores.
int encode_qkv_map(CUtensorMap* map, const void* ptr, int64_t BH, int64_t N, int64_t d,
                   uint32_t rows = 128) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d * 2), static_cast<cuuint64_t>(N * d * 2)};
    cuuint32_t box[3] = {64, rows, 1};
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

// schedule_id < 0 and group < 1 take the table's choice.
int run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
            int64_t N, int64_t d, int causal, float scale, int schedule_id, int group,
            int* dev_status, void* stream, unsigned long long* rescale_stats = nullptr) {
    int rc = check_args(q, k, v, o, lse, B, H, N, d, scale);
    if (rc == 1) return FA_OK;
    if (rc != 0) return rc;
    const ScheduleList& list = schedules();
    if (schedule_id >= list.count || (schedule_id >= 0 && list.items[schedule_id]->d != d))
        return FA_ERR_ARG;
    int table_id = 0, table_group = 1;
    pick_schedule(N, d, causal, &table_id, &table_group);
    if (schedule_id < 0) schedule_id = table_id;
    if (schedule_id < 0) return FA_ERR_ARG;
    if (group < 1) group = table_group;
    int sms = 0;
    if ((rc = current_device_ready(&sms)) != FA_OK) return rc;
    if ((rc = encoder_ready()) != FA_OK) return rc;
    const int64_t BH = B * H;
    const fa::Schedule* sch = list.items[schedule_id];
    // K and V boxes are one key tile (sch->bn rows); Q and O boxes one 128-row query tile
    alignas(64) CUtensorMap tq, tk, tv, to;
    const uint32_t bn = static_cast<uint32_t>(sch->bn);
    if (encode_qkv_map(&tq, q, BH, N, d) || encode_qkv_map(&tk, k, BH, N, d, bn) ||
        encode_qkv_map(&tv, v, BH, N, d, bn) || encode_qkv_map(&to, o, BH, N, d))
        return FA_ERR_CUDA;
    fa::FwdParams p;
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.status = dev_status;
    p.N = static_cast<int>(N);
    p.BH = static_cast<int>(BH);
    p.n_qtile = static_cast<int>((N + fa::kBlockM - 1) / fa::kBlockM);
    p.group = static_cast<int>(group < BH ? group : BH);
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    p.rescale_stats = rescale_stats;
    int64_t grid = BH * p.n_qtile;
    if (grid > 0x7fffffffLL) return FA_ERR_SHAPE;
    if (sch->alg >= 2) {
        // two or three query tiles per CTA
        const int nt = fa::tiles_per_cta(sch->alg);
        grid = BH * ((p.n_qtile + nt - 1) / nt);
    } else if (sch->persist == 1) {
        // one CTA per SM; causal work comes in units of two query tiles
        const int64_t units = causal ? BH * ((p.n_qtile + 1) / 2) : grid;
        grid = units < sms ? units : sms;
    }
    const cudaError_t e = sch->launch[causal ? 1 : 0](tq, tk, tv, to, p, static_cast<unsigned>(grid),
                                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
           int64_t N, int64_t d, int causal, float scale, void* stream) {
    return run_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, -1, 0, nullptr, stream);
}

int fa_fwd_status(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                  int64_t H, int64_t N, int64_t d, int causal, float scale, int* dev_status,
                  void* stream) {
    return run_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, -1, 0, dev_status, stream);
}

int fa_fwd_schedule(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                    int64_t H, int64_t N, int64_t d, int causal, float scale, int schedule_id,
                    int causal_group, int* dev_status, void* stream) {
    if (schedule_id < -1 || causal_group < 0) {
        const int rc = check_args(q, k, v, o, lse, B, H, N, d, scale);
        return rc == 0 ? FA_ERR_ARG : (rc == 1 ? FA_OK : rc);
    }
    return run_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, schedule_id, causal_group,
                   dev_status, stream);
}

int fa_fwd_rescale_stats(const void* q, const void* k, const void* v, void* o, float* lse,
                         int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                         int schedule_id, unsigned long long* dev_counts, void* stream) {
    const int rc = check_args(q, k, v, o, lse, B, H, N, d, scale);
    if (rc == 1) return FA_OK;
    if (rc != 0) return rc;
    if (!dev_counts) return FA_ERR_NULL;
    if (schedule_id < -1) return FA_ERR_ARG;
    return run_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, schedule_id, 0, nullptr, stream,
                   dev_counts);
}

int fa_schedule_count(void) { return schedules().count; }

int fa_schedule_info(int id, int* d, int* emu_every, int* kv_slots, int* persistent,
                     int* algorithm, int* smem_bytes, int* key_tile) {
    const ScheduleList& list = schedules();
    if (id < 0 || id >= list.count) return FA_ERR_ARG;
    const fa::Schedule* s = list.items[id];
    if (d) *d = s->d;
    if (emu_every) *emu_every = s->emu;
    if (kv_slots) *kv_slots = s->slots;
    if (persistent) *persistent = s->persist;
    if (algorithm) *algorithm = s->alg;
    if (smem_bytes) *smem_bytes = s->smem_bytes;
    if (key_tile) *key_tile = s->bn;
    return FA_OK;
}

int fa_fwd_pick_schedule(int64_t N, int64_t d, int causal, int* schedule_id, int* causal_group) {
    if (!schedule_id || !causal_group) return FA_ERR_NULL;
    if (N < 0) return FA_ERR_SHAPE;
    if (d != 64 && d != 128) return FA_ERR_HEADDIM;
    pick_schedule(N, d, causal, schedule_id, causal_group);
    return FA_OK;
}

int fa_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h, float* lse_h,
                void* q_d, void* k_d, void* v_d, void* o_d, float* lse_d, int64_t B, int64_t H,
                int64_t N, int64_t d, int causal, float scale, void* stream) {
    int rc = check_args(q_d, k_d, v_d, o_d, lse_d, B, H, N, d, scale);
    if (rc == 1) return FA_OK;
    if (rc != 0) return rc;
    if (!q_h || !k_h || !v_h || !o_h || !lse_h) return FA_ERR_NULL;
    int sms = 0;
    if ((rc = current_device_ready(&sms)) != FA_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t BH = B * H;
    const size_t slice = static_cast<size_t>(N * d);      // elements of one (b, h) slice
    // Chunks of (b, h) slices, each large enough for about four waves of
    // query tiles, at most kHostChunks: chunk c uploads while chunk c-1
    // computes and chunk c-2 downloads.
    const int64_t n_qtile = (N + fa::kBlockM - 1) / fa::kBlockM;
    int64_t per = (4 * static_cast<int64_t>(sms) + n_qtile - 1) / n_qtile;
    if (per < 1) per = 1;
    int64_t chunks = (BH + per - 1) / per;
    if (chunks > kHostChunks) chunks = kHostChunks;
    per = (BH + chunks - 1) / chunks;
    chunks = (BH + per - 1) / per;
    auto h2d = [&](int64_t c0, int64_t n, cudaStream_t st) {
        const size_t off = static_cast<size_t>(c0) * slice * 2, bytes = static_cast<size_t>(n) * slice * 2;
        return cudaMemcpyAsync(static_cast<char*>(q_d) + off, static_cast<const char*>(q_h) + off, bytes,
                               cudaMemcpyHostToDevice, st) == cudaSuccess &&
               cudaMemcpyAsync(static_cast<char*>(k_d) + off, static_cast<const char*>(k_h) + off, bytes,
                               cudaMemcpyHostToDevice, st) == cudaSuccess &&
               cudaMemcpyAsync(static_cast<char*>(v_d) + off, static_cast<const char*>(v_h) + off, bytes,
                               cudaMemcpyHostToDevice, st) == cudaSuccess;
    };
    auto d2h = [&](int64_t c0, int64_t n, cudaStream_t st) {
        const size_t off = static_cast<size_t>(c0) * slice * 2, bytes = static_cast<size_t>(n) * slice * 2;
        return cudaMemcpyAsync(static_cast<char*>(o_h) + off, static_cast<const char*>(o_d) + off, bytes,
                               cudaMemcpyDeviceToHost, st) == cudaSuccess &&
               cudaMemcpyAsync(lse_h + c0 * N, lse_d + c0 * N, static_cast<size_t>(n * N) * 4,
                               cudaMemcpyDeviceToHost, st) == cudaSuccess;
    };
    auto run_chunk = [&](int64_t c0, int64_t n) {
        const size_t off = static_cast<size_t>(c0) * slice * 2;
        return run_fwd(static_cast<const char*>(q_d) + off, static_cast<const char*>(k_d) + off,
                       static_cast<const char*>(v_d) + off, static_cast<char*>(o_d) + off, lse_d + c0 * N,
                       1, n, N, d, causal, scale, -1, 0, nullptr, stream);
    };
    if (chunks <= 1) {
        if (!h2d(0, BH, s)) return FA_ERR_CUDA;
        if (run_chunk(0, BH) != FA_OK) return FA_ERR_CUDA;
        return d2h(0, BH, s) ? FA_OK : FA_ERR_CUDA;
    }
    // Copies run on the device's two library-owned copy streams, ordered
    // against `stream` by events; `stream` waits for the last download, so its
    // completion means the whole call is done.  The streams and events are
    // created on the first pipelined call on a device and kept; the lock makes
    // concurrent calls take turns enqueueing (it is never held while waiting
    // for the GPU).
    HostPipe* pipe = nullptr;
    if ((rc = host_pipe(&pipe)) != FA_OK) return rc;
    std::lock_guard<std::mutex> lock(pipe->mu);
    cudaEvent_t* ev = pipe->ev;
    cudaEvent_t ev_start = ev[0], ev_done = ev[1];
    bool ok = cudaEventRecord(ev_start, s) == cudaSuccess &&
              cudaStreamWaitEvent(pipe->s_in, ev_start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(pipe->s_out, ev_start, 0) == cudaSuccess;
    for (int64_t c = 0; ok && c < chunks; ++c) {
        const int64_t c0 = c * per, n = (c0 + per <= BH) ? per : BH - c0;
        cudaEvent_t ev_in = ev[2 + 2 * c], ev_k = ev[3 + 2 * c];
        ok = h2d(c0, n, pipe->s_in) && cudaEventRecord(ev_in, pipe->s_in) == cudaSuccess &&
             cudaStreamWaitEvent(s, ev_in, 0) == cudaSuccess;
        ok = ok && run_chunk(c0, n) == FA_OK;
        ok = ok && cudaEventRecord(ev_k, s) == cudaSuccess &&
             cudaStreamWaitEvent(pipe->s_out, ev_k, 0) == cudaSuccess && d2h(c0, n, pipe->s_out);
    }
    if (ok) {
        ok = cudaEventRecord(ev_done, pipe->s_out) == cudaSuccess &&
             cudaStreamWaitEvent(s, ev_done, 0) == cudaSuccess;
        if (ok) return FA_OK;
    }
    // Something failed after work was enqueued: make `stream` wait for every
    // copy already queued on the copy streams (their host buffers must stay
    // valid until then), then report the failure.
    for (cudaStream_t cs : {pipe->s_in, pipe->s_out})
        if (cudaEventRecord(ev_done, cs) == cudaSuccess) cudaStreamWaitEvent(s, ev_done, 0);
    return FA_ERR_CUDA;
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

int fa_version(void) { return (1 << 16) | 2; }

}  // extern "C"
