"""Layerwise Query-Key RMSNorm (QK-Norm) on NVIDIA B200: Python binding.

A thin ctypes layer over ``libqknorm.so`` (C ABI in ``include/qknorm.h``).
It only checks tensor metadata and passes pointers, sizes and the current
CUDA stream; every step of the computation runs in the library's CUDA
kernels. There is no CPU fallback: importing this package fails loudly if the
library has not been built (``python qk_norm_attention_b200/csrc/build_lib.py``).

Entry points (same names as the C ABI):

* ``qknorm_fwd(q, k, gamma_q, gamma_k, P, eps, out_q=None, out_k=None)``:
  the fused single-pass QK-Norm of Q [T, Dq] and K [T, Dk].
* ``qknorm_partial_sumsq(x, P, stats=None)``: per-shard fp32 sums of squares,
  stats [T, P].
* ``qknorm_apply(x, gamma, stats, eps, out=None)``: the factor from stats and
  (x * gamma) * r.

Tensors are CUDA tensors, row-major contiguous, fp32, bf16 or FP8 E4M3
(torch.float8_e4m3fn) for x/y and fp32 for gamma and stats. Calls are asynchronous on ``torch.cuda.current_stream()``
(or the ``stream`` argument).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libqknorm.so")

QKNORM_F32, QKNORM_BF16, QKNORM_E4M3 = 0, 1, 2
QKNORM_OK = 0
QKNORM_ERR_INVALID_ARG = 1
QKNORM_ERR_MISALIGNED = 2
QKNORM_ERR_UNSUPPORTED = 3
QKNORM_ERR_CUDA = 4

VARIANT_AUTO, VARIANT_CTA, VARIANT_WARP, VARIANT_GENERIC, VARIANT_BULK, VARIANT_ROWS, VARIANT_PAIR, \
    VARIANT_GPAIR = -1, 0, 1, 2, 3, 4, 5, 6
VARIANT_NAMES = {VARIANT_CTA: "cta", VARIANT_WARP: "warp", VARIANT_GENERIC: "generic",
                 VARIANT_BULK: "bulk", VARIANT_ROWS: "rows", VARIANT_PAIR: "pair",
                 VARIANT_GPAIR: "gpair"}

_DTYPE = {torch.float32: QKNORM_F32, torch.bfloat16: QKNORM_BF16,
          torch.float8_e4m3fn: QKNORM_E4M3}


class QKNormError(RuntimeError):
    """A libqknorm call returned a non-OK status."""

    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{fn}: {qknorm_status_string(status)} (status {status})"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)


class QKNormPlan(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int32), ("block", ctypes.c_int32),
                ("grid", ctypes.c_int64), ("vmax", ctypes.c_int32),
                ("prefetch", ctypes.c_int32), ("groups_q", ctypes.c_int32),
                ("groups_k", ctypes.c_int32), ("stages", ctypes.c_int32),
                ("tokens_per_stage", ctypes.c_int32), ("gamma_regs", ctypes.c_int32),
                ("full_lanes", ctypes.c_int32), ("smem_bytes", ctypes.c_int64),
                ("q_warps", ctypes.c_int32), ("gamma_smem", ctypes.c_int32),
                ("k_pairs", ctypes.c_int32), ("vmax_k", ctypes.c_int32),
                ("half_slots", ctypes.c_int32), ("mixed", ctypes.c_int32)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIBRARY):
        raise ImportError(
            f"libqknorm.so not found at {LIBRARY}; build it with "
            "`python qk_norm_attention_b200/csrc/build_lib.py` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIBRARY)
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    lib.qknorm_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, i32, vp]
    lib.qknorm_partial_sumsq.argtypes = [vp, vp, i64, i32, i32, i32, vp]
    lib.qknorm_apply.argtypes = [vp, vp, vp, vp, i64, i32, i32, f32, i32, vp]
    for fn in (lib.qknorm_fwd, lib.qknorm_partial_sumsq, lib.qknorm_apply):
        fn.restype = ctypes.c_int
    lib.qknorm_fwd_strided.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, i32,
                                       i64, i64, i64, i64, vp]
    lib.qknorm_fwd_strided.restype = ctypes.c_int
    lib.qknorm_headwise_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, i32,
                                        i64, i64, i64, i64, vp]
    lib.qknorm_headwise_fwd.restype = ctypes.c_int
    lib.qknorm_fwd_host.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, f32, i32, vp, i64,
                                    i64, vp]
    lib.qknorm_fwd_host.restype = ctypes.c_int
    lib.qknorm_fwd_host_workspace.argtypes = [i64, i32, i32, i32]
    lib.qknorm_fwd_host_workspace.restype = ctypes.c_int64
    lib.qknorm_apply_tp.argtypes = [vp, vp, vp, i64, vp, i64, i32, i32, i32, f32, i32, vp]
    lib.qknorm_apply_tp.restype = ctypes.c_int
    lib.qknorm_partial_sumsq_qk.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, vp]
    lib.qknorm_partial_sumsq_qk.restype = ctypes.c_int
    lib.qknorm_apply_tp_qk.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, vp, i64, i32, i32, i32, i32,
                                       f32, i32, vp]
    lib.qknorm_apply_tp_qk.restype = ctypes.c_int
    lib.qknorm_xgamma.argtypes = [vp, vp, vp, i64, i32, i32, vp]
    lib.qknorm_xgamma.restype = ctypes.c_int
    lib.qknorm_inv_rms.argtypes = [vp, vp, i64, i32, i32, f32, i32, vp]
    lib.qknorm_inv_rms.restype = ctypes.c_int
    lib.qknorm_split_noalloc.argtypes = [vp, vp, vp, i64, i32, i32, f32, i32, vp]
    lib.qknorm_split_noalloc.restype = ctypes.c_int
    lib.qknorm_split_noalloc_max_stats.argtypes = []
    lib.qknorm_split_noalloc_max_stats.restype = ctypes.c_int64
    lib.qknorm_status_string.argtypes = [ctypes.c_int]
    lib.qknorm_status_string.restype = ctypes.c_char_p
    lib.qknorm_last_error.argtypes = []
    lib.qknorm_last_error.restype = ctypes.c_char_p
    lib.qknorm_plan_fwd.argtypes = [i64, i32, i32, i32, i32, i32, i32, ctypes.POINTER(QKNormPlan)]
    lib.qknorm_plan_fwd.restype = ctypes.c_int
    lib.qknorm_launch_plan.argtypes = [i64, i32, i32, i32, i32, ctypes.POINTER(QKNormPlan)]
    lib.qknorm_launch_plan.restype = ctypes.c_int
    lib.qknorm_force_variant.argtypes = [i32, i64]
    lib.qknorm_force_variant.restype = ctypes.c_int
    lib.qknorm_version.restype = ctypes.c_int
    lib.qknorm_set_tuning.argtypes = [i32, i32, i32, i32]
    lib.qknorm_set_tuning.restype = ctypes.c_int
    lib.qknorm_set_pdl.argtypes = [i32]
    lib.qknorm_set_pdl.restype = ctypes.c_int
    lib.qknorm_set_rows_tuning.argtypes = [i32, i32, i32, i32]
    lib.qknorm_set_rows_tuning.restype = ctypes.c_int
    lib.qknorm_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    lib.qknorm_device_errors.restype = ctypes.c_int
    lib.qknorm_selftest_bounded_wait.argtypes = [ctypes.c_uint64, vp]
    lib.qknorm_selftest_bounded_wait.restype = ctypes.c_int
    return lib


lib = _load()


def qknorm_status_string(status: int) -> str:
    return lib.qknorm_status_string(int(status)).decode()


def qknorm_last_error() -> str:
    return lib.qknorm_last_error().decode()


def _check(fn: str, status: int) -> None:
    if status != QKNORM_OK:
        raise QKNormError(fn, status, qknorm_last_error() if status == QKNORM_ERR_CUDA else "")


def _stream_handle(device: torch.device, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPE:
        raise TypeError(f"unsupported dtype {t.dtype}; use torch.float32, torch.bfloat16 "
                        "or torch.float8_e4m3fn")
    return _DTYPE[t.dtype]


def _need_cuda_contig(name: str, t: torch.Tensor) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def qknorm_fwd(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor,
               P: int, eps: float, out_q: Optional[torch.Tensor] = None,
               out_k: Optional[torch.Tensor] = None, stream=None):
    """Fused layerwise QK-Norm of q [T, Dq] and k [T, Dk]; returns (out_q, out_k)."""
    if q.dim() != 2 or k.dim() != 2 or q.shape[0] != k.shape[0]:
        raise ValueError("q and k must be [T, Dq] and [T, Dk] with the same T")
    if q.dtype != k.dtype:
        raise TypeError("q and k must have the same dtype")
    out_q = torch.empty_like(q) if out_q is None else out_q
    out_k = torch.empty_like(k) if out_k is None else out_k
    for name, t in (("q", q), ("k", k), ("gamma_q", gamma_q), ("gamma_k", gamma_k),
                    ("out_q", out_q), ("out_k", out_k)):
        _need_cuda_contig(name, t)
    if gamma_q.dtype != torch.float32 or gamma_k.dtype != torch.float32:
        raise TypeError("gamma must be float32")
    if out_q.shape != q.shape or out_k.shape != k.shape or out_q.dtype != q.dtype or out_k.dtype != k.dtype:
        raise ValueError("outputs must match the inputs' shape and dtype")
    if gamma_q.numel() != q.shape[1] or gamma_k.numel() != k.shape[1]:
        raise ValueError("gamma_q/gamma_k must have Dq/Dk elements")
    T, Dq = q.shape
    Dk = k.shape[1]
    st = lib.qknorm_fwd(q.data_ptr(), k.data_ptr(), gamma_q.data_ptr(), gamma_k.data_ptr(),
                        out_q.data_ptr(), out_k.data_ptr(), T, Dq, Dk, int(P), float(eps),
                        _dtype_code(q), _stream_handle(q.device, stream))
    _check("qknorm_fwd", st)
    return out_q, out_k


def _rows_view(name: str, t: torch.Tensor):
    """(T, D, row stride) of a 2-D CUDA tensor whose rows are dense (stride 1
    along a row), e.g. a column slice of a fused QKV buffer."""
    if not t.is_cuda or t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be a 2-D CUDA tensor with unit stride along rows")
    return t.shape[0], t.shape[1], t.stride(0)


def qknorm_fwd_strided(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor,
                       gamma_k: torch.Tensor, P: int, eps: float,
                       out_q: Optional[torch.Tensor] = None, out_k: Optional[torch.Tensor] = None,
                       stream=None):
    """qknorm_fwd on row-strided q and k (e.g. slices of a fused QKV buffer);
    the outputs may be the inputs themselves (in place) or dense tensors."""
    T, Dq, ldq = _rows_view("q", q)
    Tk, Dk, ldk = _rows_view("k", k)
    if T != Tk or q.dtype != k.dtype:
        raise ValueError("q and k must share T and dtype")
    out_q = torch.empty((T, Dq), dtype=q.dtype, device=q.device) if out_q is None else out_q
    out_k = torch.empty((T, Dk), dtype=k.dtype, device=k.device) if out_k is None else out_k
    _, Doq, ldoq = _rows_view("out_q", out_q)
    _, Dok, ldok = _rows_view("out_k", out_k)
    if (Doq, Dok) != (Dq, Dk) or out_q.dtype != q.dtype or out_k.dtype != k.dtype:
        raise ValueError("outputs must match the inputs' widths and dtype")
    for name, g, D in (("gamma_q", gamma_q, Dq), ("gamma_k", gamma_k, Dk)):
        _need_cuda_contig(name, g)
        if g.dtype != torch.float32 or g.numel() != D:
            raise ValueError(f"{name} must be float32 with {D} elements")
    st = lib.qknorm_fwd_strided(q.data_ptr(), k.data_ptr(), gamma_q.data_ptr(), gamma_k.data_ptr(),
                                out_q.data_ptr(), out_k.data_ptr(), T, Dq, Dk, int(P), float(eps),
                                _dtype_code(q), ldq, ldk, ldoq, ldok, _stream_handle(q.device, stream))
    _check("qknorm_fwd_strided", st)
    return out_q, out_k


def qknorm_headwise_fwd(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor,
                        gamma_k: torch.Tensor, head_dim: int, eps: float,
                        out_q: Optional[torch.Tensor] = None, out_k: Optional[torch.Tensor] = None,
                        stream=None):
    """Headwise QK-Norm: q [T, Hq*head_dim], k [T, Hk*head_dim] (rows may be
    strided), gamma [head_dim] per tensor; one factor per head."""
    T, Dq, ldq = _rows_view("q", q)
    Tk, Dk, ldk = _rows_view("k", k)
    if T != Tk or q.dtype != k.dtype or Dq % head_dim or Dk % head_dim:
        raise ValueError("q and k must share T and dtype; widths must be multiples of head_dim")
    out_q = torch.empty((T, Dq), dtype=q.dtype, device=q.device) if out_q is None else out_q
    out_k = torch.empty((T, Dk), dtype=k.dtype, device=k.device) if out_k is None else out_k
    _, Doq, ldoq = _rows_view("out_q", out_q)
    _, Dok, ldok = _rows_view("out_k", out_k)
    if (Doq, Dok) != (Dq, Dk) or out_q.dtype != q.dtype or out_k.dtype != k.dtype:
        raise ValueError("outputs must match the inputs' widths and dtype")
    for name, g in (("gamma_q", gamma_q), ("gamma_k", gamma_k)):
        _need_cuda_contig(name, g)
        if g.dtype != torch.float32 or g.numel() != head_dim:
            raise ValueError(f"{name} must be float32 with head_dim elements")
    st = lib.qknorm_headwise_fwd(q.data_ptr(), k.data_ptr(), gamma_q.data_ptr(), gamma_k.data_ptr(),
                                 out_q.data_ptr(), out_k.data_ptr(), T, Dq // head_dim,
                                 Dk // head_dim, int(head_dim), float(eps), _dtype_code(q),
                                 ldq, ldk, ldoq, ldok, _stream_handle(q.device, stream))
    _check("qknorm_headwise_fwd", st)
    return out_q, out_k


def qknorm_partial_sumsq(x: torch.Tensor, P: int, stats: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """stats[t, p] = fp32 sum of squares of shard p of row t; returns stats [T, P]."""
    if x.dim() != 2:
        raise ValueError("x must be [T, D]")
    T, D = x.shape
    stats = torch.empty((T, int(P)), dtype=torch.float32, device=x.device) if stats is None else stats
    _need_cuda_contig("x", x)
    _need_cuda_contig("stats", stats)
    if stats.dtype != torch.float32 or stats.numel() != T * int(P):
        raise ValueError("stats must be float32 with T*P elements")
    st = lib.qknorm_partial_sumsq(x.data_ptr(), stats.data_ptr(), T, D, int(P), _dtype_code(x),
                                  _stream_handle(x.device, stream))
    _check("qknorm_partial_sumsq", st)
    return stats


def qknorm_apply(x: torch.Tensor, gamma: torch.Tensor, stats: torch.Tensor, eps: float,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out = (x * gamma) * rsqrt(sum_p stats[t, p] / D + eps); P = stats.shape[1]."""
    if x.dim() != 2 or stats.dim() != 2 or stats.shape[0] != x.shape[0]:
        raise ValueError("x must be [T, D] and stats [T, P]")
    T, D = x.shape
    P = stats.shape[1]
    out = torch.empty_like(x) if out is None else out
    for name, t in (("x", x), ("gamma", gamma), ("stats", stats), ("out", out)):
        _need_cuda_contig(name, t)
    if gamma.dtype != torch.float32 or stats.dtype != torch.float32:
        raise TypeError("gamma and stats must be float32")
    if out.shape != x.shape or out.dtype != x.dtype or gamma.numel() != D:
        raise ValueError("out must match x; gamma must have D elements")
    st = lib.qknorm_apply(x.data_ptr(), gamma.data_ptr(), stats.data_ptr(), out.data_ptr(), T, D,
                          P, float(eps), _dtype_code(x), _stream_handle(x.device, stream))
    _check("qknorm_apply", st)
    return out


def qknorm_fwd_host_workspace(Dq: int, Dk: int, dtype: torch.dtype, chunk_tokens: int = 0) -> int:
    """Device workspace bytes qknorm_fwd_host needs."""
    n = lib.qknorm_fwd_host_workspace(int(chunk_tokens), int(Dq), int(Dk), _DTYPE[dtype])
    if n < 0:
        raise ValueError("invalid widths or dtype")
    return n


def qknorm_fwd_host(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor,
                    P: int, eps: float, workspace: torch.Tensor,
                    out_q: Optional[torch.Tensor] = None, out_k: Optional[torch.Tensor] = None,
                    chunk_tokens: int = 0, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """qknorm_fwd on CPU tensors q [T, Dq], k [T, Dk] (pinned for overlap),
    gamma on the GPU, `workspace` a uint8 CUDA tensor of at least
    qknorm_fwd_host_workspace bytes. Returns CPU outputs; they are complete
    once `stream` (default: the current stream of workspace's device) is
    synchronised."""
    if q.dim() != 2 or k.dim() != 2 or q.shape[0] != k.shape[0] or q.dtype != k.dtype:
        raise ValueError("q [T, Dq] and k [T, Dk] of one dtype")
    if q.is_cuda or k.is_cuda or not (q.is_contiguous() and k.is_contiguous()):
        raise ValueError("q and k must be contiguous host (CPU) tensors")
    T, Dq = q.shape
    Dk = k.shape[1]
    out_q = torch.empty_like(q, pin_memory=q.is_pinned()) if out_q is None else out_q
    out_k = torch.empty_like(k, pin_memory=k.is_pinned()) if out_k is None else out_k
    for name, t in (("gamma_q", gamma_q), ("gamma_k", gamma_k), ("workspace", workspace)):
        _need_cuda_contig(name, t)
    if out_q.shape != q.shape or out_k.shape != k.shape or out_q.is_cuda or out_k.is_cuda:
        raise ValueError("outputs must be host tensors shaped like q and k")
    st = lib.qknorm_fwd_host(q.data_ptr(), k.data_ptr(), gamma_q.data_ptr(), gamma_k.data_ptr(),
                             out_q.data_ptr(), out_k.data_ptr(), T, Dq, Dk, int(P), float(eps),
                             _dtype_code(q), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             int(chunk_tokens), _stream_handle(workspace.device, stream))
    _check("qknorm_fwd_host", st)
    return out_q, out_k


def qknorm_apply_tp(x: torch.Tensor, gamma: torch.Tensor, stats: torch.Tensor, eps: float,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One tensor-parallel rank's apply step: x [T, D_local] (this rank's
    slice), gamma [D_local], stats [ranks, T, P_local] (every rank's shard
    sums, rank-major, as an all-gather leaves them; a strided view with
    contiguous [T, P_local] blocks is accepted). The divisor is ranks * D_local."""
    if x.dim() != 2 or stats.dim() != 3 or stats.shape[1] != x.shape[0]:
        raise ValueError("x must be [T, D_local] and stats [ranks, T, P_local]")
    T, D = x.shape
    ranks, _, P = stats.shape
    out = torch.empty_like(x) if out is None else out
    for name, t in (("x", x), ("gamma", gamma), ("out", out)):
        _need_cuda_contig(name, t)
    if not stats.is_cuda or stats.stride(2) != 1 or stats.stride(1) != P:
        raise ValueError("stats blocks must be contiguous [T, P_local] on the GPU")
    if gamma.dtype != torch.float32 or stats.dtype != torch.float32:
        raise TypeError("gamma and stats must be float32")
    if out.shape != x.shape or out.dtype != x.dtype or gamma.numel() != D:
        raise ValueError("out must match x; gamma must have D_local elements")
    st = lib.qknorm_apply_tp(x.data_ptr(), gamma.data_ptr(), stats.data_ptr(), stats.stride(0),
                             out.data_ptr(), T, D, P, ranks, float(eps), _dtype_code(x),
                             _stream_handle(x.device, stream))
    _check("qknorm_apply_tp", st)
    return out


def qknorm_partial_sumsq_qk(q: torch.Tensor, k: torch.Tensor, P: int,
                            stats: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The shard sums of q [T, Dq] and k [T, Dk] in one launch: returns
    stats [2, T, P] (stats[0] Q's, stats[1] K's), each as qknorm_partial_sumsq."""
    if q.dim() != 2 or k.dim() != 2 or q.shape[0] != k.shape[0]:
        raise ValueError("q and k must be [T, Dq] and [T, Dk]")
    T, P = q.shape[0], int(P)
    stats = torch.empty((2, T, P), dtype=torch.float32, device=q.device) if stats is None else stats
    for name, t in (("q", q), ("k", k), ("stats", stats)):
        _need_cuda_contig(name, t)
    if stats.dtype != torch.float32 or tuple(stats.shape) != (2, T, P) or q.dtype != k.dtype:
        raise ValueError("stats must be float32 [2, T, P]; q and k of one dtype")
    st = lib.qknorm_partial_sumsq_qk(q.data_ptr(), k.data_ptr(), stats[0].data_ptr(), stats[1].data_ptr(),
                                     T, q.shape[1], k.shape[1], P, _dtype_code(q),
                                     _stream_handle(q.device, stream))
    _check("qknorm_partial_sumsq_qk", st)
    return stats


def qknorm_apply_tp_qk(q: torch.Tensor, k: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor,
                       stats: torch.Tensor, eps: float, out_q: Optional[torch.Tensor] = None,
                       out_k: Optional[torch.Tensor] = None,
                       stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """qknorm_apply_tp of one rank's q [T, Dq_local] and k [T, Dk_local] in one
    launch, from stats [ranks, 2, T, P_local] (every rank's Q and K shard sums,
    as an all-gather of each rank's [2, T, P_local] leaves them)."""
    if q.dim() != 2 or k.dim() != 2 or stats.dim() != 4 or stats.shape[1] != 2 or \
            stats.shape[2] != q.shape[0] or k.shape[0] != q.shape[0]:
        raise ValueError("q, k must be [T, D_local] and stats [ranks, 2, T, P_local]")
    T = q.shape[0]
    ranks, _, _, P = stats.shape
    out_q = torch.empty_like(q) if out_q is None else out_q
    out_k = torch.empty_like(k) if out_k is None else out_k
    for name, t in (("q", q), ("k", k), ("gamma_q", gamma_q), ("gamma_k", gamma_k), ("out_q", out_q),
                    ("out_k", out_k)):
        _need_cuda_contig(name, t)
    if not stats.is_cuda or stats.stride(3) != 1 or stats.stride(2) != P or stats.stride(1) != T * P:
        raise ValueError("stats must hold contiguous [2, T, P_local] blocks on the GPU")
    if gamma_q.dtype != torch.float32 or gamma_k.dtype != torch.float32 or stats.dtype != torch.float32:
        raise TypeError("gamma and stats must be float32")
    if out_q.shape != q.shape or out_k.shape != k.shape or out_q.dtype != q.dtype or \
            out_k.dtype != k.dtype or q.dtype != k.dtype or gamma_q.numel() != q.shape[1] or \
            gamma_k.numel() != k.shape[1]:
        raise ValueError("outputs must match their inputs; gamma_q, gamma_k of the local widths")
    st = lib.qknorm_apply_tp_qk(q.data_ptr(), k.data_ptr(), gamma_q.data_ptr(), gamma_k.data_ptr(),
                                stats[:, 0].data_ptr(), stats[:, 1].data_ptr(), stats.stride(0),
                                out_q.data_ptr(), out_k.data_ptr(), T, q.shape[1], k.shape[1], P, ranks,
                                float(eps), _dtype_code(q), _stream_handle(q.device, stream))
    _check("qknorm_apply_tp_qk", st)
    return out_q, out_k


def qknorm_xgamma(x: torch.Tensor, gamma: torch.Tensor, out: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    """out = x * gamma (the weight multiply alone, rounded to x's dtype)."""
    if x.dim() != 2:
        raise ValueError("x must be [T, D]")
    T, D = x.shape
    out = torch.empty_like(x) if out is None else out
    for name, t in (("x", x), ("gamma", gamma), ("out", out)):
        _need_cuda_contig(name, t)
    if gamma.dtype != torch.float32 or gamma.numel() != D or out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("gamma must be float32 [D]; out must match x")
    _check("qknorm_xgamma", lib.qknorm_xgamma(x.data_ptr(), gamma.data_ptr(), out.data_ptr(), T, D,
                                              _dtype_code(x), _stream_handle(x.device, stream)))
    return out


def qknorm_inv_rms(x: torch.Tensor, P: int, eps: float, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """inv_rms[t] = rsqrt(mean_j x[t, j]^2 + eps) (fp32, the per-token factor alone)."""
    if x.dim() != 2:
        raise ValueError("x must be [T, D]")
    T, D = x.shape
    out = torch.empty(T, dtype=torch.float32, device=x.device) if out is None else out
    _need_cuda_contig("x", x)
    _need_cuda_contig("out", out)
    if out.dtype != torch.float32 or out.numel() != T:
        raise ValueError("out must be float32 [T]")
    _check("qknorm_inv_rms", lib.qknorm_inv_rms(x.data_ptr(), out.data_ptr(), T, D, int(P), float(eps),
                                                _dtype_code(x), _stream_handle(x.device, stream)))
    return out


def qknorm_plan_fwd(T: int, Dq: int, Dk: int, P: int, dtype: int, num_sms: int,
                    blocks_per_sm: int = 0) -> dict:
    """The selector's plan for a device with ``num_sms`` SMs (host logic only)."""
    pl = QKNormPlan()
    _check("qknorm_plan_fwd", lib.qknorm_plan_fwd(T, Dq, Dk, P, dtype, num_sms, blocks_per_sm,
                                                  ctypes.byref(pl)))
    return pl.as_dict()


def qknorm_launch_plan(T: int, Dq: int, Dk: int, P: int, dtype: int) -> dict:
    """The plan qknorm_fwd uses on the current device."""
    pl = QKNormPlan()
    _check("qknorm_launch_plan", lib.qknorm_launch_plan(T, Dq, Dk, P, dtype, ctypes.byref(pl)))
    return pl.as_dict()


def qknorm_force_variant(variant: int = VARIANT_AUTO, grid: int = 0) -> None:
    """Override the selector process-wide (tests and benchmarks)."""
    _check("qknorm_force_variant", lib.qknorm_force_variant(int(variant), int(grid)))


def qknorm_version() -> int:
    return lib.qknorm_version()


def qknorm_set_tuning(stages: int = 0, tokens_per_stage: int = 0, gamma_regs: int = -1,
                      wait_limit_ms: int = 0) -> None:
    """Tune the bulk variant process-wide (the defaults restore automatic choice)."""
    _check("qknorm_set_tuning", lib.qknorm_set_tuning(int(stages), int(tokens_per_stage),
                                                      int(gamma_regs), int(wait_limit_ms)))


def qknorm_set_pdl(enable: bool = True) -> None:
    """Programmatic dependent launch on (default) or off, process-wide."""
    _check("qknorm_set_pdl", lib.qknorm_set_pdl(int(bool(enable))))


def qknorm_set_rows_tuning(q_warps: int = 0, k_warps: int = 0, stages: int = 0,
                           gamma_smem: int = -1) -> None:
    """Q-pool and K-pool warps per CTA, row stages per warp and gamma staging
    of the rows variant (0, 0, 0, -1 = automatic)."""
    _check("qknorm_set_rows_tuning", lib.qknorm_set_rows_tuning(int(q_warps), int(k_warps),
                                                                int(stages), int(gamma_smem)))


def qknorm_device_errors(clear: bool = True) -> int:
    """The device error word (bit 1: a bounded wait timed out; bit 2: copies
    were in flight when a CTA left). Synchronises with the device."""
    v = ctypes.c_uint32(0)
    _check("qknorm_device_errors", lib.qknorm_device_errors(ctypes.byref(v), int(bool(clear))))
    return v.value


def qknorm_selftest_bounded_wait(limit_ns: int, stream=None, device=None) -> None:
    """Launch the bounded-wait self-test kernel (it must time out and set bit 1)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _check("qknorm_selftest_bounded_wait",
           lib.qknorm_selftest_bounded_wait(int(limit_ns), _stream_handle(dev, stream)))


def qknorm_split_noalloc(x: torch.Tensor, gamma: torch.Tensor, P: int, eps: float,
                         out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The split path (statistics, then apply) in one call, with the statistics
    in the library's own device buffer: for callers that cannot allocate
    device memory. T * P must not exceed qknorm_split_noalloc_max_stats()."""
    if x.dim() != 2:
        raise ValueError("x must be [T, D]")
    T, D = x.shape
    code = _dtype_code(x)
    if gamma.dtype != torch.float32:
        raise TypeError("gamma must be float32")
    if gamma.numel() != D:
        raise ValueError(f"gamma must have D = {D} elements")
    out = torch.empty_like(x) if out is None else out
    if out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("out must have x's shape and dtype")
    for name, t in (("x", x), ("gamma", gamma), ("out", out)):
        _need_cuda_contig(name, t)
    st = lib.qknorm_split_noalloc(x.data_ptr(), gamma.data_ptr(), out.data_ptr(), T, D, int(P),
                                  float(eps), code, _stream_handle(x.device, stream))
    _check("qknorm_split_noalloc", st)
    return out
