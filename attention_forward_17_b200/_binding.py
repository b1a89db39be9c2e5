"""ctypes binding of libfa_b200.so (include/fa.h).

Argument marshalling only: every step of the attention forward pass (and of
the row softmax, GEMM and vector-add entry points) runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or the device is not
sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
HEADER = os.path.join(ROOT, "include", "fa.h")
LIB_PATH = os.path.join(HERE, "libfa_b200.so")

FA_OK = 0
FA_ERR_NULL = -1
FA_ERR_SHAPE = -2
FA_ERR_HEADDIM = -3
FA_ERR_ALIGN = -4
FA_ERR_SCALE = -5
FA_ERR_CUDA = -6
FA_ERR_TIMEOUT = -7
FA_ERR_ARCH = -8
FA_ERR_ARG = -9

FA_GEMM_PLAIN, FA_GEMM_BIAS, FA_GEMM_BIAS_GELU = 0, 1, 2

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


class FaError(RuntimeError):
    def __init__(self, status: int, where: str = "fa_fwd"):
        self.status = status
        super().__init__(f"{where} failed with status {status}: {strerror(status)}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python attention_forward_17_b200/build.py` "
            "(there is no non-CUDA fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.fa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.c_int,
                           ctypes.c_float, _vp]
    lib.fa_fwd.restype = ctypes.c_int
    lib.fa_fwd_status.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.c_int,
                                  ctypes.c_float, _vp, _vp]
    lib.fa_fwd_status.restype = ctypes.c_int
    lib.fa_fwd_host.argtypes = [_vp] * 10 + [_i64, _i64, _i64, _i64, ctypes.c_int, ctypes.c_float,
                                            _vp]
    lib.fa_fwd_host.restype = ctypes.c_int
    lib.fa_selftest_wait_timeout.argtypes = [_vp, _i64, ctypes.c_int, _vp]
    lib.fa_selftest_wait_timeout.restype = ctypes.c_int
    lib.fa_row_softmax.argtypes = [_vp, _vp, _i64, _i64, ctypes.c_float, _vp]
    lib.fa_row_softmax.restype = ctypes.c_int
    lib.fa_row_softmax_launches.argtypes = [_i64, _i64]
    lib.fa_row_softmax_launches.restype = ctypes.c_int
    lib.fa_fwd_schedule.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.c_int,
                                    ctypes.c_float, ctypes.c_int, ctypes.c_int, _vp, _vp]
    lib.fa_fwd_schedule.restype = ctypes.c_int
    lib.fa_fwd_rescale_stats.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                         ctypes.c_int, ctypes.c_float, ctypes.c_int, _vp, _vp]
    lib.fa_fwd_rescale_stats.restype = ctypes.c_int
    lib.fa_schedule_count.argtypes = []
    lib.fa_schedule_count.restype = ctypes.c_int
    lib.fa_schedule_info.argtypes = [ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
    lib.fa_schedule_info.restype = ctypes.c_int
    lib.fa_fwd_pick_schedule.argtypes = [_i64, _i64, ctypes.c_int, _vp, _vp]
    lib.fa_fwd_pick_schedule.restype = ctypes.c_int
    lib.fa_gemm.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_int, _vp, _vp]
    lib.fa_gemm.restype = ctypes.c_int
    lib.fa_gemm_launches.argtypes = [_i64, _i64, _i64]
    lib.fa_gemm_launches.restype = ctypes.c_int
    lib.fa_vector_add.argtypes = [_vp, _vp, _vp, _i64, _vp]
    lib.fa_vector_add.restype = ctypes.c_int
    lib.fa_vector_add_launches.argtypes = [_i64]
    lib.fa_vector_add_launches.restype = ctypes.c_int
    lib.fa_fwd_launches.argtypes = [_i64, _i64, _i64, _i64]
    lib.fa_fwd_launches.restype = ctypes.c_int
    lib.fa_strerror.argtypes = [ctypes.c_int]
    lib.fa_strerror.restype = ctypes.c_char_p
    lib.fa_version.argtypes = []
    lib.fa_version.restype = ctypes.c_int
    return lib


lib = _load()


def header_functions() -> list[str]:
    """Names of the functions include/fa.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(", text, flags=re.M)


def strerror(status: int) -> str:
    return lib.fa_strerror(int(status)).decode()


def version() -> tuple[int, int]:
    v = lib.fa_version()
    return v >> 16, v & 0xFFFF


def launches_per_call(B: int, H: int, N: int, d: int) -> int:
    return int(lib.fa_fwd_launches(B, H, N, d))


def _check_qkv(q, k, v):
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [B, H, N, d], got shape {tuple(t.shape)}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.shape == k.shape == v.shape):
        raise ValueError(f"q, k, v shapes differ: {tuple(q.shape)} {tuple(k.shape)} {tuple(v.shape)}")
    if not (q.device == k.device == v.device) or q.device.type != "cuda":
        raise ValueError("q, k, v must be on the same CUDA device")


def schedules() -> list[dict]:
    """Every compiled schedule of the attention kernel: id, d, emu_every, kv_slots,
    persistent, algorithm, smem_bytes, key_tile."""
    out = []
    for i in range(lib.fa_schedule_count()):
        vals = [ctypes.c_int() for _ in range(7)]
        rc = lib.fa_schedule_info(i, *[ctypes.byref(x) for x in vals])
        if rc != FA_OK:
            raise FaError(rc, "fa_schedule_info")
        out.append(dict(id=i, d=vals[0].value, emu_every=vals[1].value, kv_slots=vals[2].value,
                        persistent=vals[3].value, algorithm=vals[4].value,
                        smem_bytes=vals[5].value, key_tile=vals[6].value))
    return out


def pick_schedule(N: int, d: int, causal: bool) -> tuple[int, int]:
    """(schedule id, causal group) that fa_fwd uses for this problem."""
    sid, grp = ctypes.c_int(), ctypes.c_int()
    rc = lib.fa_fwd_pick_schedule(N, d, int(bool(causal)), ctypes.byref(sid), ctypes.byref(grp))
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_pick_schedule")
    return sid.value, grp.value


def fa_fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None,
           stream=None, status=None, schedule: int | None = None, causal_group: int | None = None):
    """O, LSE = attention forward of bf16 [B, H, N, d] CUDA tensors.

    ``out`` (bf16 [B,H,N,d]) and ``lse`` (fp32 [B,H,N]) are allocated when not
    given.  Runs on ``stream`` (a torch.cuda.Stream) or the current stream.
    ``status`` may be an int32 CUDA tensor with one element; it then receives
    FA_ERR_TIMEOUT should a device-side wait run out of time.  ``schedule``
    (an id from ``schedules()``) and ``causal_group`` override the table's
    choice.
    """
    import torch
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if out.dtype != torch.bfloat16 or out.shape != q.shape or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [B, H, N] tensor")
    s = (stream if stream is not None else torch.cuda.current_stream(q.device)).cuda_stream
    with torch.cuda.device(q.device):
        if schedule is not None or causal_group is not None:
            rc = lib.fa_fwd_schedule(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                     -1 if schedule is None else int(schedule),
                                     0 if causal_group is None else int(causal_group),
                                     status.data_ptr() if status is not None else None, s)
        elif status is None:
            rc = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale), s)
        else:
            rc = lib.fa_fwd_status(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                   status.data_ptr(), s)
    if rc != FA_OK:
        raise FaError(rc)
    return out, lse


def rescale_stats(q, k, v, causal: bool = False, scale: float | None = None,
                  schedule: int | None = None):
    """Runs the forward pass once with the rescale counters on; returns
    (O, LSE, warp_steps_rescaled, row_steps_rescaled, warp_steps_total): how many
    (warp, key tile) steps and (row, key tile) steps rescaled the output
    accumulator, and the number of (warp, key tile) steps the two-query-tile
    kernel executed.  Only that kernel counts (other schedules report zeros)."""
    import torch
    _check_qkv(q, k, v)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    counts = torch.zeros(2, dtype=torch.int64, device=q.device)
    s = torch.cuda.current_stream(q.device).cuda_stream
    with torch.cuda.device(q.device):
        rc = lib.fa_fwd_rescale_stats(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      lse.data_ptr(), B, H, N, d, int(bool(causal)), float(scale),
                                      -1 if schedule is None else int(schedule),
                                      counts.data_ptr(), s)
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_rescale_stats")
    torch.cuda.synchronize(q.device)
    # (warp, key tile) steps of the two-query-tile kernel: 4 warps per query tile,
    # key tiles up to the diagonal under the mask
    nq, nk = (N + 127) // 128, (N + 127) // 128
    steps = sum(min(nk, t + 1) if causal else nk for t in range(nq))
    return out, lse, int(counts[0].item()), int(counts[1].item()), 4 * B * H * steps


def fa_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, causal: bool = False,
                scale: float | None = None, stream=None):
    """Host-to-host attention forward through caller-provided device buffers.

    All arguments are torch tensors: the ``*_h`` ones on the CPU (pinned for
    asynchronous copies), the ``*_d`` ones on the GPU.  Enqueues H2D copies,
    the kernel and D2H copies on ``stream`` and returns without waiting.
    """
    import torch
    _check_qkv(q_d, k_d, v_d)
    B, H, N, d = q_d.shape
    for t in (q_h, k_h, v_h, o_h):
        if t.shape != q_d.shape or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("host q/k/v/o must be contiguous bf16 tensors shaped like q_d")
    if tuple(lse_h.shape) != (B, H, N) or lse_h.dtype != torch.float32:
        raise ValueError("lse_h must be fp32 [B, H, N]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    s = (stream if stream is not None else torch.cuda.current_stream(q_d.device)).cuda_stream
    with torch.cuda.device(q_d.device):
        rc = lib.fa_fwd_host(q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), o_h.data_ptr(),
                             lse_h.data_ptr(), q_d.data_ptr(), k_d.data_ptr(), v_d.data_ptr(),
                             o_d.data_ptr(), lse_d.data_ptr(), B, H, N, d, int(bool(causal)),
                             float(scale), s)
    if rc != FA_OK:
        raise FaError(rc, "fa_fwd_host")


def selftest_wait_timeout(status, limit_us: int, arrive: bool = False, stream=None):
    """Run the bounded-wait self-test kernel; `status` is an int32 CUDA tensor (one element)."""
    import torch
    s = (stream if stream is not None else torch.cuda.current_stream(status.device)).cuda_stream
    with torch.cuda.device(status.device):
        rc = lib.fa_selftest_wait_timeout(status.data_ptr(), int(limit_us), int(bool(arrive)), s)
    if rc != FA_OK:
        raise FaError(rc, "fa_selftest_wait_timeout")


def row_softmax(x, scale: float = 1.0, out=None, stream=None):
    """y = softmax(scale * x) over the last dimension of a contiguous bf16 CUDA tensor."""
    import torch
    if not isinstance(x, torch.Tensor) or x.dtype != torch.bfloat16 or x.device.type != "cuda":
        raise TypeError("x must be a bfloat16 CUDA tensor")
    if not x.is_contiguous() or x.dim() < 1:
        raise ValueError("x must be contiguous with at least one dimension")
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    if out is None:
        out = torch.empty_like(x)
    if out.shape != x.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like x")
    s = (stream if stream is not None else torch.cuda.current_stream(x.device)).cuda_stream
    with torch.cuda.device(x.device):
        rc = lib.fa_row_softmax(x.data_ptr(), out.data_ptr(), rows, cols, float(scale), s)
    if rc != FA_OK:
        raise FaError(rc, "fa_row_softmax")
    return out


def gemm(a, b, bias=None, epilogue: int = FA_GEMM_BIAS_GELU, out=None, stream=None, status=None):
    """C = epilogue(A @ B) for contiguous bf16 CUDA tensors A [M, K], B [K, N], bias [N].

    ``epilogue`` is FA_GEMM_PLAIN, FA_GEMM_BIAS or FA_GEMM_BIAS_GELU (exact erf
    GELU).  ``out`` (bf16 [M, N]) is allocated when not given.  ``status`` may
    be an int32 CUDA tensor with one element (receives FA_ERR_TIMEOUT).
    """
    import torch
    for name, t in (("a", a), ("b", b)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.device.type != "cuda":
            raise TypeError(f"{name} must be a bfloat16 CUDA tensor")
        if t.dim() != 2 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous 2-D tensor")
    M, K = a.shape
    K2, N = b.shape
    if K != K2:
        raise ValueError(f"inner dimensions differ: {tuple(a.shape)} @ {tuple(b.shape)}")
    if bias is not None and (bias.dtype != torch.bfloat16 or tuple(bias.shape) != (N,)
                             or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous bf16 [N] tensor")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    if out.dtype != torch.bfloat16 or tuple(out.shape) != (M, N) or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [M, N] tensor")
    s = (stream if stream is not None else torch.cuda.current_stream(a.device)).cuda_stream
    with torch.cuda.device(a.device):
        rc = lib.fa_gemm(a.data_ptr() if K else None, b.data_ptr() if K else None,
                         bias.data_ptr() if bias is not None else None, out.data_ptr(), M, N, K,
                         int(epilogue), status.data_ptr() if status is not None else None, s)
    if rc != FA_OK:
        raise FaError(rc, "fa_gemm")
    return out


def vector_add(x, y, out=None, stream=None):
    """z = x + y for contiguous fp32 CUDA tensors of equal shape."""
    import torch
    for name, t in (("x", x), ("y", y)):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.float32 or t.device.type != "cuda":
            raise TypeError(f"{name} must be a float32 CUDA tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if x.shape != y.shape:
        raise ValueError("x and y shapes differ")
    if out is None:
        out = torch.empty_like(x)
    if out.shape != x.shape or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be a contiguous float32 tensor shaped like x")
    s = (stream if stream is not None else torch.cuda.current_stream(x.device)).cuda_stream
    with torch.cuda.device(x.device):
        rc = lib.fa_vector_add(x.data_ptr(), y.data_ptr(), out.data_ptr(), x.numel(), s)
    if rc != FA_OK:
        raise FaError(rc, "fa_vector_add")
    return out
