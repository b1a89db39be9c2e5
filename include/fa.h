/*
 * fa.h - C ABI of the B200 (sm_100a) fused attention forward library
 * (libfa_b200.so).
 *
 * The main operation is the fused FlashAttention forward pass of the "TileLang
 * tutorial" (FlashAttention section): query, key and value tiles are processed
 * without materialising the attention-score matrix in global memory, using an
 * online softmax (running row maxima, running normalisation sums, rescaling
 * factors) and tensor-core products, for causal and non-causal attention.  For
 * every (b, h) slice and query row i it returns
 *
 *     O[b,h,i,:] = sum_j softmax_j( scale * Q[b,h,i,:] . K[b,h,j,:] ) * V[b,h,j,:]
 *     LSE[b,h,i] = ln sum_j exp( scale * Q[b,h,i,:] . K[b,h,j,:] )
 *
 * where, when `causal` is nonzero, only keys j <= i take part (top-left
 * alignment; query and key lengths are equal).  The pages validate this
 * against scaled-dot-product attention; LSE is the natural-log logsumexp of the
 * scaled scores.
 *
 * The library also carries the tutorial's other kernels, each behind its own
 * entry point below: the row-wise softmax, the tiled tensor-core GEMM with
 * its fused bias + GELU epilogue, and the vector addition.
 *
 * Layout: Q, K, V and O are bf16 [B, H, N, d], dense row-major (d fastest), in
 * device memory.  LSE is fp32 [B, H, N].  d must be 64 or 128.  Arithmetic:
 * bf16 tensor-core products with fp32 accumulation, fp32 softmax, P rounded to
 * bf16 (nearest-even) before the P.V product, O rounded to bf16 (nearest-even).
 *
 * Ownership: the caller owns every buffer.  The library never allocates device
 * memory and keeps no per-call state.
 *
 * Errors: the argument checks below run on the host in the listed order and
 * return before anything is launched.  Launches are asynchronous on `stream`
 * (a cudaStream_t; NULL = the legacy default stream); a launch failure returns
 * FA_ERR_CUDA.  The calls never synchronise the stream.
 *
 * Threading: every entry point is reentrant and may be called from several
 * host threads at once.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_NULL = -1,     /* a required pointer is NULL                              */
    FA_ERR_SHAPE = -2,    /* B, H or N negative, or beyond the supported range       */
    FA_ERR_HEADDIM = -3,  /* d is not 64 or 128                                      */
    FA_ERR_ALIGN = -4,    /* a device pointer is not 16-byte aligned (LSE: 4-byte)   */
    FA_ERR_SCALE = -5,    /* scale is not finite and > 0                             */
    FA_ERR_CUDA = -6,     /* a CUDA runtime/driver call failed                       */
    FA_ERR_TIMEOUT = -7,  /* a device-side pipeline wait ran out of time             */
    FA_ERR_ARCH = -8,     /* the current device is not compute capability 10.0       */
    FA_ERR_ARG = -9       /* an enumerated argument is out of range                  */
} fa_status;

/*
 * fa_fwd - fused attention forward.
 *
 *   q, k, v  device, bf16 [B,H,N,d], read only, 16-byte aligned.
 *   o        device, bf16 [B,H,N,d], written, 16-byte aligned.
 *   lse      device, fp32 [B,H,N], written, 4-byte aligned.
 *   B, H, N  >= 0; a zero makes the call a no-op that returns FA_OK (pointers
 *            are then not examined).  N <= 2^31 - 512 and B*H <= 2^31 - 1.
 *   d        64 or 128.
 *   causal   0 = full attention, nonzero = key j visible to query i iff j <= i.
 *   scale    multiplier of q.k inside the softmax (usually 1/sqrt(d)); finite, > 0.
 *   stream   cudaStream_t or NULL.
 *
 * o and lse must not overlap q, k or v (not checked).  Should a device-side
 * pipeline wait ever exceed about two seconds (it cannot in correct
 * operation), the CTA involved gives up: the rows of the query tile it is on
 * receive LSE = NaN, tiles a persistent CTA had not reached yet are left
 * unwritten, and the kernel still terminates (in-flight copies and products
 * are drained first).  The outputs are then undefined; use fa_fwd_status to
 * receive FA_ERR_TIMEOUT in a status word, the reliable signal.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t H,
           int64_t N, int64_t d, int causal, float scale, void* stream);

/*
 * fa_fwd_status - fa_fwd that also reports device-side failures.
 *
 *   dev_status  device int, caller-owned.  The kernel never clears it; it
 *               writes FA_ERR_TIMEOUT into it if a pipeline wait runs out of
 *               time.  Read it after the stream has completed.  NULL behaves
 *               like fa_fwd.
 * Other arguments and checks are those of fa_fwd.
 */
int fa_fwd_status(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                  int64_t H, int64_t N, int64_t d, int causal, float scale, int* dev_status,
                  void* stream);

/*
 * Schedules.  The kernel is compiled in several schedules: the share of
 * exponentials evaluated by polynomial on the FMA pipe instead of the
 * special-function unit, the depth of the K/V shared-memory ring, and the
 * launch form (one CTA per query tile; one persistent CTA per SM walking
 * several tiles so that one tile's epilogue overlaps the next tile's start,
 * under the causal mask in pairs of tiles of equal total work; or one CTA per
 * tile where a running CTA takes over the tiles of CTAs that have not launched
 * yet).  Under
 * the causal mask the launch order is a further runtime knob: (b, h) slices
 * are taken `causal_group` at a time, longest query tiles first within a
 * group.  fa_fwd and fa_fwd_status use, per (d, causal, N), the schedule and
 * group that a schedule search on a B200 measured fastest (the tutorial's
 * autotuning step: benchmark, validate, cache); fa_fwd_schedule lets the
 * caller choose.  Every schedule computes the same function within the same
 * tolerances.
 *
 * fa_schedule_count - number of compiled schedules (ids 0 .. count-1).
 * fa_schedule_info  - the head dimension, exponential split (every emu_every-th
 *                     pair by polynomial; 0 = none), K/V ring depth, launch
 *                     form (0 = one CTA per query tile, 1 = persistent with a
 *                     static tile assignment, 2 = one CTA per tile whose
 *                     running CTAs take over the tiles of CTAs not launched
 *                     yet, through cluster launch control), algorithm (0 =
 *                     one softmax pass over every key tile, 1 = split-KV
 *                     ping-pong: two softmax warp groups take alternate key
 *                     tiles with their own running statistics and output
 *                     accumulators, merged per row at the end; 2 = two
 *                     128-row query tiles per CTA sharing every key/value
 *                     tile, P kept over the scores in tensor memory, one
 *                     tensor-core issuing thread for both tiles in a fixed
 *                     alternating order, O stored through shared memory with
 *                     TMA; 3 = as 2 with two score buffers per query tile, so
 *                     the scores of the next key tile are computed while the
 *                     softmax works on the current one; 4, 5 = as 2, 3 with
 *                     the sum of the bf16 weights accumulated by the tensor
 *                     core, d = 64 only; 6 to 9 = as 2 to 5 with P released
 *                     to the tensor core as the first three quarters and then
 *                     the last quarter of a 128-key tile; + 8 = three query
 *                     tiles per CTA instead of two, d = 64 only), shared memory
 *                     per CTA
 *                     and rows of a key/value tile (128, or 64 / 192 for some
 *                     two-tile schedules) of schedule `id`; FA_ERR_ARG for an
 *                     unknown id.  Output pointers may be NULL.
 * fa_fwd_pick_schedule - the schedule id and causal group fa_fwd uses for
 *                     (N, d, causal).  FA_ERR_NULL, FA_ERR_SHAPE (N < 0),
 *                     FA_ERR_HEADDIM.
 * fa_fwd_schedule   - fa_fwd_status with an explicit schedule: schedule_id in
 *                     0 .. count-1 with the same d as the call, or -1 for the
 *                     table's choice; causal_group >= 1 (clamped to B*H), or 0
 *                     for the table's choice (the static persistent launch
 *                     ignores the group).  The arguments of fa_fwd are
 *                     checked first (same order and codes), then FA_ERR_ARG
 *                     for a bad schedule_id or causal_group.
 */
int fa_schedule_count(void);
int fa_schedule_info(int id, int* d, int* emu_every, int* kv_slots, int* persistent,
                     int* algorithm, int* smem_bytes, int* key_tile);
int fa_fwd_pick_schedule(int64_t N, int64_t d, int causal, int* schedule_id, int* causal_group);
int fa_fwd_schedule(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                    int64_t H, int64_t N, int64_t d, int causal, float scale, int schedule_id,
                    int causal_group, int* dev_status, void* stream);

/*
 * fa_fwd_rescale_stats - fa_fwd_schedule (causal_group from the table) that
 * also counts the lazy rescales of the output accumulator ("rescaling
 * factors" of the FlashAttention section: a row's O is rescaled only when its
 * running maximum grew by more than 2^8 since the last rescale).
 *
 *   schedule_id  as for fa_fwd_schedule (-1: the table's choice).
 *   dev_counts   device, two unsigned 64-bit counters, caller-owned, never
 *                cleared: [0] += (warp, key tile) steps at which at least one
 *                of the warp's 32 rows rescaled, [1] += (row, key tile)
 *                rescales.  Only the multi-tile kernel (algorithms 2
 *                and above) counts; other schedules leave the counters unchanged.
 *                NULL -> FA_ERR_NULL (after the checks of fa_fwd).
 * A diagnostic entry point: the atomics cost a little time.
 */
int fa_fwd_rescale_stats(const void* q, const void* k, const void* v, void* o, float* lse,
                         int64_t B, int64_t H, int64_t N, int64_t d, int causal, float scale,
                         int schedule_id, unsigned long long* dev_counts, void* stream);

/*
 * fa_fwd_host - the same computation starting from and ending in host memory.
 *
 * Copies q_h, k_h, v_h (host, bf16 [B,H,N,d]; pinned memory makes the copies
 * asynchronous) into the caller's device buffers q_d, k_d, v_d; runs the
 * forward pass on them into o_d and lse_d; copies o_d and lse_d back into o_h
 * and lse_h (host).  The (b, h) slices are processed in up to eight chunks so
 * that uploads, kernels and downloads of consecutive chunks overlap: the
 * kernels run on `stream`, the copies on two copy streams the library creates
 * once per device (with a few events) and keeps for the life of the process,
 * ordered by events so that the copies start after all earlier work on
 * `stream` and `stream` completes only after the last download.  Concurrent
 * calls on one device take turns enqueueing their copies on those streams.
 * Nothing is allocated on the device; the call returns without synchronising,
 * so the host buffers must stay valid until `stream` has completed.  Argument
 * checks are those of fa_fwd applied to the device buffers, plus FA_ERR_NULL
 * for a NULL host pointer.  A failure after some work was enqueued returns
 * FA_ERR_CUDA, and `stream` is still made to wait for every copy that was
 * queued, so its completion still means no copy touches the host buffers.
 */
int fa_fwd_host(const void* q_h, const void* k_h, const void* v_h, void* o_h, float* lse_h,
                void* q_d, void* k_d, void* v_d, void* o_d, float* lse_d, int64_t B, int64_t H,
                int64_t N, int64_t d, int causal, float scale, void* stream);

/*
 * fa_selftest_wait_timeout - exercises the device-side failure path.
 *
 * Launches one small kernel that waits, with the same bounded-wait routine
 * the attention kernel uses for every pipeline wait, on an mbarrier that
 * nothing arrives at.  The wait gives up after `limit_us` microseconds and
 * writes FA_ERR_TIMEOUT into the caller-owned device int `dev_status`; the
 * kernel then exits normally and the CUDA context stays usable.  With
 * `arrive` nonzero the barrier is completed first and `dev_status` is left
 * untouched (the control case).  Nothing faults, traps or hangs.
 *
 *   dev_status  device int, caller-owned, not cleared by the call (NULL -> FA_ERR_NULL)
 *   limit_us    1 .. 10,000,000 (else FA_ERR_SHAPE)
 */
int fa_selftest_wait_timeout(int* dev_status, int64_t limit_us, int arrive, void* stream);

/*
 * fa_row_softmax - row-wise softmax (the tutorial's softmax section: fragment
 * maximum and sum reductions, normalisation kept in registers).
 *
 *     y[r, c] = exp(scale * x[r, c] - max_c' scale * x[r, c']) / sum_c' exp(...)
 *
 *   x      device, bf16 [rows, cols], dense row-major, finite values, read only.
 *   y      device, bf16 [rows, cols], written (may not overlap x unless equal to it).
 *   rows   0 .. 2^31 - 1; cols 0 .. 2^31 - 1 (a zero is a no-op returning FA_OK).
 *   scale  any finite value (FA_ERR_SCALE otherwise).
 * x and y must be 2-byte aligned (FA_ERR_ALIGN).  fp32 arithmetic, output
 * rounded to nearest even.  Rows with cols % 8 == 0, 16-byte aligned
 * pointers and cols <= 16384 are read once and written once; other shapes
 * read the row twice.  Asynchronous on `stream`; FA_ERR_ARCH on a non-sm_100
 * device; nothing is allocated.
 */
int fa_row_softmax(const void* x, void* y, int64_t rows, int64_t cols, float scale, void* stream);

/* Number of kernel launches one fa_row_softmax call makes (0 or 1). */
int fa_row_softmax_launches(int64_t rows, int64_t cols);

/* Epilogues of fa_gemm. */
typedef enum {
    FA_GEMM_PLAIN = 0,     /* C = A B                              */
    FA_GEMM_BIAS = 1,      /* C = A B + bias                       */
    FA_GEMM_BIAS_GELU = 2  /* C = GELU(A B + bias), exact erf form */
} fa_gemm_epilogue;

/*
 * fa_gemm - tiled tensor-core matrix product with a fused epilogue (the
 * tutorial's tiled GEMM section, and its fused-epilogue section: bias and
 * GELU applied to the accumulator before the only store of C).
 *
 *     C[i, j] = epi( sum_k A[i, k] B[k, j] )
 *        FA_GEMM_PLAIN      epi(x) = x
 *        FA_GEMM_BIAS       epi(x) = x + bias[j]
 *        FA_GEMM_BIAS_GELU  epi(x) = GELU(x + bias[j]),  GELU(u) = u/2 (1 + erf(u / sqrt 2))
 *
 *   a         device, bf16 [M, K] row-major, 16-byte aligned, read only (may be NULL if K = 0).
 *   b         device, bf16 [K, N] row-major, 16-byte aligned, read only (may be NULL if K = 0).
 *   bias      device, bf16 [N], 16-byte aligned, read only; unused (may be NULL) with
 *             FA_GEMM_PLAIN.
 *   c         device, bf16 [M, N] row-major, 16-byte aligned, written; must not overlap a, b
 *             or bias (not checked).
 *   M, N, K   >= 0 and <= 2^31 - 256; N and K multiples of 8 (rows of whole 16-byte units).
 *             M = 0 or N = 0 is a no-op returning FA_OK; K = 0 gives C = epi(0).
 *   epilogue  a fa_gemm_epilogue value (FA_ERR_ARG otherwise).
 *   dev_status  optional caller-owned device int, never cleared: receives FA_ERR_TIMEOUT if a
 *             device-side pipeline wait ran out of time (about two seconds; C is then
 *             undefined).  NULL to ignore.
 *   stream    cudaStream_t or NULL.
 * Checks, in order: epilogue (FA_ERR_ARG), negative sizes (FA_ERR_SHAPE), empty (FA_OK),
 * pointers (FA_ERR_NULL), size limits and multiples of 8 (FA_ERR_SHAPE), alignment
 * (FA_ERR_ALIGN), device (FA_ERR_ARCH / FA_ERR_CUDA).  Arithmetic: bf16 products with fp32
 * accumulation in tensor memory, the epilogue in fp32, C rounded to bf16 (nearest-even).
 * Problems of more than 128 rows with K > 0 run 256 x 256 tiles on pairs of SMs (a cluster
 * of two CTAs, tcgen05.mma.cta_group::2); others run 128 x 256 tiles on single SMs.
 * One launch, asynchronous on `stream`; nothing is allocated.
 */
int fa_gemm(const void* a, const void* b, const void* bias, void* c, int64_t M, int64_t N,
            int64_t K, int epilogue, int* dev_status, void* stream);

/* Number of kernel launches one fa_gemm call makes (0 or 1). */
int fa_gemm_launches(int64_t M, int64_t N, int64_t K);

/*
 * fa_vector_add - z[i] = x[i] + y[i] over fp32 (the tutorial's vector-add
 * kernel, a memory-bandwidth probe).
 *
 *   x, y  device, fp32 [n], read only, 4-byte aligned.
 *   z     device, fp32 [n], written, 4-byte aligned; may be x or y itself (in place) but may
 *         not overlap them otherwise.
 *   n     0 .. 2^40 (0 is a no-op returning FA_OK; negative or larger: FA_ERR_SHAPE).
 * IEEE fp32 addition, round-to-nearest-even, so the result is exact to the bit.  When all
 * three pointers are 16-byte aligned the kernel moves 16-byte vectors, else single floats.
 * Checks: size, pointers (FA_ERR_NULL), alignment (FA_ERR_ALIGN), device.  One launch,
 * asynchronous on `stream`; nothing is allocated.
 */
int fa_vector_add(const float* x, const float* y, float* z, int64_t n, void* stream);

/* Number of kernel launches one fa_vector_add call makes (0 or 1). */
int fa_vector_add_launches(int64_t n);

/* Number of kernel launches one fa_fwd call makes for these sizes (0 or 1). */
int fa_fwd_launches(int64_t B, int64_t H, int64_t N, int64_t d);

/* Static description of a status code; never NULL. */
const char* fa_strerror(int status);

/* Library ABI version, (major << 16) | minor. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
