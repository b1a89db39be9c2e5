"""B200 (sm_100a) fused attention forward: O = softmax(scale * Q K^T [+ causal mask]) V and
the per-row logsumexp, computed by hand-written tcgen05/TMA kernels behind the C ABI in
include/fa.h.  This package is the thin Python binding of that library."""
from ._binding import (FA_ERR_ALIGN, FA_ERR_ARCH, FA_ERR_ARG, FA_ERR_CUDA, FA_ERR_HEADDIM,
                       FA_ERR_NULL, FA_ERR_SCALE, FA_ERR_SHAPE, FA_ERR_TIMEOUT, FA_GEMM_BIAS,
                       FA_GEMM_BIAS_GELU, FA_GEMM_PLAIN, FA_OK, FaError, LIB_PATH, fa_fwd,
                       fa_fwd_host, gemm, header_functions, launches_per_call, lib, pick_schedule,
                       rescale_stats, row_softmax, schedules, selftest_wait_timeout, strerror, vector_add,
                       version)

__all__ = ["fa_fwd", "fa_fwd_host", "rescale_stats", "row_softmax", "gemm", "vector_add", "schedules",
           "pick_schedule", "selftest_wait_timeout",
           "FaError", "strerror", "version", "launches_per_call", "header_functions", "lib",
           "LIB_PATH", "FA_OK", "FA_ERR_NULL", "FA_ERR_SHAPE", "FA_ERR_HEADDIM", "FA_ERR_ALIGN",
           "FA_ERR_SCALE", "FA_ERR_CUDA", "FA_ERR_TIMEOUT", "FA_ERR_ARCH", "FA_ERR_ARG",
           "FA_GEMM_PLAIN", "FA_GEMM_BIAS", "FA_GEMM_BIAS_GELU"]
