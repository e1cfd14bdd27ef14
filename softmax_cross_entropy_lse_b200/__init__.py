"""Fused softmax cross-entropy for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/ce_b200.h``: it turns torch
tensors into pointers, strides and the current CUDA stream, allocates the
outputs with torch, and raises on a non-zero status. Every step of the
computation runs in the CUDA kernels of ``libce_b200.so``; there is no Python
or CPU fallback, and calling any op without the built library raises.

Row ops accept logits as a 2-D (N, V) tensor or a 3-D (B, L, V) tensor with
any strides (for instance the view ``x[:, :-1]``); they are read in place,
never copied. Targets are (N,) or (B, L) int32/int64 tensors with any strides.
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libce_b200.so")

CE_F32, CE_BF16, CE_F16 = 0, 1, 2
CE_I32, CE_I64 = 0, 1
STATUS = {0: "CE_OK", 1: "CE_EINVAL", 2: "CE_EALIAS", 3: "CE_EWORKSPACE", 4: "CE_ECUDA",
          5: "CE_ETARGET", 6: "CE_ENOTSUP", 7: "CE_ETIMEOUT"}
EXPORTED = ["ce_workspace_size", "ce_forward", "ce_backward", "linear_ce_workspace_size",
            "linear_ce_forward", "linear_ce_backward_workspace_size", "linear_ce_backward",
            "ce_get_error", "ce_status_string", "ce_forward_noalloc", "ce_forward_backward",
            "ce_soft_forward", "ce_soft_backward", "ce_kl_forward", "ce_kl_backward",
            "ce_testing_set_wait"]
NOALLOC_SCRATCH_BYTES = 64 << 10


class ce_layout(ctypes.Structure):
    _fields_ = [("inner", ctypes.c_int64), ("s_outer", ctypes.c_int64),
                ("s_inner", ctypes.c_int64), ("s_col", ctypes.c_int64)]


class CEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_status_string(status)})")


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m softmax_cross_entropy_lse_b200.build` "
                "(there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, f32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.ce_workspace_size.argtypes = [i64, i64, ctypes.c_int, ctypes.c_int]
        L.ce_workspace_size.restype = sz
        L.ce_forward.argtypes = [vp, ctypes.c_int, ce_layout, i64, i64, vp, ctypes.c_int, ce_layout,
                                 f32, i64, vp, vp, vp, vp, vp, sz, vp]
        L.ce_forward.restype = ctypes.c_int
        L.ce_backward.argtypes = [vp, i64, vp, ctypes.c_int, ce_layout, i64, i64, vp, ctypes.c_int,
                                  ce_layout, vp, vp, f32, i64, vp, ctypes.c_int, ce_layout, vp]
        L.ce_backward.restype = ctypes.c_int
        L.linear_ce_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int]
        L.linear_ce_workspace_size.restype = sz
        L.linear_ce_forward.argtypes = [vp, i64, vp, i64, vp, ctypes.c_int, i64, i64, i64, f32, i64,
                                        vp, vp, vp, sz, vp]
        L.linear_ce_forward.restype = ctypes.c_int
        L.linear_ce_backward_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int]
        L.linear_ce_backward_workspace_size.restype = sz
        L.linear_ce_backward.argtypes = [vp, i64, vp, i64, vp, i64, vp, ctypes.c_int, vp, i64, i64,
                                         i64, f32, i64, vp, ctypes.c_int, vp, ctypes.c_int, vp, sz, vp]
        L.linear_ce_backward.restype = ctypes.c_int
        L.ce_forward_noalloc.argtypes = [vp, ctypes.c_int, ce_layout, i64, i64, vp, ctypes.c_int,
                                         ce_layout, f32, i64, vp, vp, vp, vp, vp]
        L.ce_forward_noalloc.restype = ctypes.c_int
        L.ce_forward_backward.argtypes = [vp, ctypes.c_int, ce_layout, i64, i64, vp, ctypes.c_int,
                                          ce_layout, f32, i64, vp, i64, vp, vp, vp, vp, vp,
                                          ctypes.c_int, ce_layout, vp, sz, vp]
        L.ce_forward_backward.restype = ctypes.c_int
        L.ce_soft_forward.argtypes = [vp, ctypes.c_int, ce_layout, i64, i64, vp, ctypes.c_int, ce_layout,
                                      f32, vp, vp, vp, vp, vp]
        L.ce_soft_forward.restype = ctypes.c_int
        L.ce_soft_backward.argtypes = [vp, i64, vp, ctypes.c_int, ce_layout, i64, i64, vp, ctypes.c_int,
                                       ce_layout, vp, vp, vp, f32, vp, ctypes.c_int, ce_layout, vp]
        L.ce_soft_backward.restype = ctypes.c_int
        L.ce_kl_forward.argtypes = [vp, vp, ctypes.c_int, ce_layout, ce_layout, i64, i64, vp, vp, vp, vp,
                                    vp, vp]
        L.ce_kl_forward.restype = ctypes.c_int
        L.ce_kl_backward.argtypes = [vp, i64, vp, vp, ctypes.c_int, ce_layout, ce_layout, i64, i64, vp,
                                     vp, vp, vp, vp, ctypes.c_int, ce_layout, vp]
        L.ce_kl_backward.restype = ctypes.c_int
        L.ce_testing_set_wait.argtypes = [ctypes.c_uint64, ctypes.c_int]
        L.ce_testing_set_wait.restype = ctypes.c_int
        L.ce_get_error.argtypes = [vp]
        L.ce_get_error.restype = ctypes.c_int
        L.ce_status_string.argtypes = [ctypes.c_int]
        L.ce_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _status_string(s: int) -> str:
    try:
        return lib().ce_status_string(s).decode()
    except Exception:  # pragma: no cover - only when the library is absent
        return "?"


def _check(status: int, where: str) -> None:
    if status != 0:
        raise CEError(status, where)


# -- torch marshalling -------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    m = {torch.float32: CE_F32, torch.bfloat16: CE_BF16, torch.float16: CE_F16}
    if t.dtype not in m:
        raise TypeError(f"unsupported logits dtype {t.dtype}")
    return m[t.dtype]


def _index_code(t) -> int:
    torch = _torch()
    m = {torch.int32: CE_I32, torch.int64: CE_I64}
    if t.dtype not in m:
        raise TypeError(f"unsupported targets dtype {t.dtype}")
    return m[t.dtype]


def _merge_dims(sizes, strides):
    """Merge adjacent dims whose strides allow it (no copy); returns lists."""
    out_s, out_t = [], []
    for n, s in zip(sizes, strides):
        if out_s and out_t[-1] == s * n:
            out_s[-1] *= n
            out_t[-1] = s
        elif n == 1 and out_s:
            continue
        else:
            out_s.append(n)
            out_t.append(s)
    return out_s, out_t


def row_layout(t, has_cols: bool = True):
    """(N, ce_layout) for a tensor of rows (..., V) or of row scalars (...)."""
    sizes = list(t.shape[:-1]) if has_cols else list(t.shape)
    strides = list(t.stride()[:-1]) if has_cols else list(t.stride())
    s_col = t.stride()[-1] if has_cols else 0
    N = 1
    for n in sizes:
        N *= n
    if N == 0:
        return 0, ce_layout(1, 0, 0, s_col)
    ms, mt = _merge_dims(sizes, strides)
    if len(ms) == 0:
        return N, ce_layout(1, 0, 0, s_col)
    if len(ms) == 1:
        return N, ce_layout(ms[0], 0, mt[0], s_col)
    if len(ms) == 2:
        return N, ce_layout(ms[1], mt[0], mt[1], s_col)
    raise ValueError(f"rows of shape {tuple(t.shape)} with strides {t.stride()} need more than "
                     "two levels of row addressing; pass a view with at most two row levels")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("every tensor must live on the CUDA device (no CPU path)")


# -- row cross-entropy ------------------------------------------------------------------
class ForwardResult(NamedTuple):
    loss: "object"
    lse: "object"
    lse_lo: "object"
    argmax: "object"


def ce_workspace_size(N: int, V: int, dtype, num_sms: int = 0) -> int:
    code = dtype if isinstance(dtype, int) else _dtype_code(_torch().empty(0, dtype=dtype))
    return int(lib().ce_workspace_size(N, V, code, num_sms))


def _row_outputs(N: int, dev, return_argmax: bool, out):
    """Per-row output tensors: fresh ones, or the caller's `out` (a
    ForwardResult of contiguous float32 loss, lse, lse_lo and int32 argmax on
    the logits' device, N entries each), written in place."""
    torch = _torch()
    if out is None:
        return (torch.empty(N, dtype=torch.float32, device=dev),
                torch.empty(N, dtype=torch.float32, device=dev),
                torch.empty(N, dtype=torch.float32, device=dev),
                torch.empty(N, dtype=torch.int32, device=dev) if return_argmax else None)
    loss, lse, lse_lo, am = out
    want = [(loss, torch.float32), (lse, torch.float32), (lse_lo, torch.float32)]
    if return_argmax:
        if am is None:
            raise ValueError("return_argmax needs an argmax tensor in `out`")
        want.append((am, torch.int32))
    for t, dt in want:
        if t.dtype != dt or t.numel() != N or not t.is_contiguous() or t.device != dev:
            raise ValueError(f"`out` tensors must be contiguous {dt} with {N} entries on {dev}")
    return loss, lse, lse_lo, (am if return_argmax else None)


def ce_forward(logits, targets, label_smoothing: float = 0.0, ignore_index: int = -100, *,
               return_argmax: bool = False, workspace=None, stream=None, out=None) -> ForwardResult:
    """Per-row loss, lse (and its low-order float lse_lo, and optional argmax).
    `out` (a ForwardResult) receives them in place instead of new tensors."""
    torch = _torch()
    _require_cuda(logits, targets)
    N, lg = row_layout(logits, True)
    Nt, tg = row_layout(targets, False)
    if Nt != N:
        raise ValueError(f"targets hold {Nt} rows, logits {N}")
    V = logits.shape[-1]
    dev = logits.device
    loss, lse, lse_lo, am = _row_outputs(N, dev, return_argmax, out)
    dt = _dtype_code(logits)
    with torch.cuda.device(dev):
        need = int(lib().ce_workspace_size(N, V, dt, 0))
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib().ce_forward(_ptr(logits), dt, lg, N, V, _ptr(targets), _index_code(targets), tg,
                              float(label_smoothing), int(ignore_index), _ptr(loss), _ptr(lse),
                              _ptr(lse_lo), _ptr(am), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "ce_forward")
    return ForwardResult(loss, lse, lse_lo, am)


def ce_backward(grad_out, logits, targets, lse, lse_lo=None, label_smoothing: float = 0.0,
                ignore_index: int = -100, *, dlogits=None, out_dtype=None, stream=None):
    """dlogits = g (softmax - (1-eps) onehot - eps/V), zero on ignored rows.

    grad_out: a float32 tensor of N per-row values, or a 0-d / 1-element
    tensor broadcast to every row. dlogits may be `logits` itself (in place).
    """
    torch = _torch()
    _require_cuda(grad_out, logits, targets, lse, lse_lo, dlogits)
    N, lg = row_layout(logits, True)
    Nt, tg = row_layout(targets, False)
    if Nt != N:
        raise ValueError(f"targets hold {Nt} rows, logits {N}")
    V = logits.shape[-1]
    if grad_out.dtype != torch.float32:
        raise TypeError("grad_out must be float32")
    if grad_out.numel() == 1:
        g_stride = 0
    else:
        if grad_out.numel() != N:
            raise ValueError("grad_out must hold one value per row or a single value")
        gflat = grad_out.reshape(-1) if grad_out.dim() != 1 else grad_out
        if gflat.data_ptr() != grad_out.data_ptr():
            raise ValueError("grad_out must be a view over its storage")
        g_stride = gflat.stride(0)
        grad_out = gflat
    if dlogits is None:
        dt = out_dtype or logits.dtype
        dlogits = torch.empty(logits.shape, dtype=dt, device=logits.device)
    Nd, dl = row_layout(dlogits, True)
    if Nd != N or dlogits.shape[-1] != V:
        raise ValueError("dlogits must have the shape of logits")
    with torch.cuda.device(logits.device):
        st = lib().ce_backward(_ptr(grad_out), g_stride, _ptr(logits), _dtype_code(logits), lg, N, V,
                               _ptr(targets), _index_code(targets), tg, _ptr(lse), _ptr(lse_lo),
                               float(label_smoothing), int(ignore_index), _ptr(dlogits),
                               _dtype_code(dlogits), dl, _stream(stream))
    _check(st, "ce_backward")
    return dlogits


class SoftResult(NamedTuple):
    loss: object
    lse: object
    lse_lo: object
    target_sum: object


def _grad_view(torch, grad_out, N):
    if grad_out.dtype != torch.float32:
        raise TypeError("grad_out must be float32")
    if grad_out.numel() == 1:
        return grad_out, 0
    if grad_out.numel() != N:
        raise ValueError("grad_out must hold one value per row or a single value")
    gflat = grad_out.reshape(-1) if grad_out.dim() != 1 else grad_out
    if gflat.data_ptr() != grad_out.data_ptr():
        raise ValueError("grad_out must be a view over its storage")
    return gflat, gflat.stride(0)


def ce_soft_forward(logits, target_probs, label_smoothing: float = 0.0, *,
                    return_target_sum: bool = True, stream=None) -> SoftResult:
    """Cross-entropy against probability targets: loss_i = sum_j t'_ij
    (lse_i - z_ij) with t' = (1-eps) t + eps/V. target_probs has the shape of
    logits (any strides), dtype of the logits or float32. Also returns lse,
    lse_lo and (if asked) the per-row sums of target_probs for the backward."""
    torch = _torch()
    _require_cuda(logits, target_probs)
    N, lg = row_layout(logits, True)
    Nt, tl = row_layout(target_probs, True)
    if Nt != N or target_probs.shape[-1] != logits.shape[-1]:
        raise ValueError("target_probs must have the shape of logits")
    V = logits.shape[-1]
    dev = logits.device
    loss, lse, lse_lo = (torch.empty(N, dtype=torch.float32, device=dev) for _ in range(3))
    tsum = torch.empty(N, dtype=torch.float32, device=dev) if return_target_sum else None
    with torch.cuda.device(dev):
        st = lib().ce_soft_forward(_ptr(logits), _dtype_code(logits), lg, N, V, _ptr(target_probs),
                                   _dtype_code(target_probs), tl, float(label_smoothing), _ptr(loss),
                                   _ptr(lse), _ptr(lse_lo), _ptr(tsum), _stream(stream))
    _check(st, "ce_soft_forward")
    return SoftResult(loss, lse, lse_lo, tsum)


def ce_soft_backward(grad_out, logits, target_probs, lse, lse_lo=None, target_sum=None,
                     label_smoothing: float = 0.0, *, dlogits=None, out_dtype=None, stream=None):
    """dlogits = g (softmax T' - t'), T' = (1-eps) T + eps with T the row sums
    of target_probs (target_sum from ce_soft_forward; None: rows sum to 1)."""
    torch = _torch()
    _require_cuda(grad_out, logits, target_probs, lse, lse_lo, target_sum, dlogits)
    N, lg = row_layout(logits, True)
    Nt, tl = row_layout(target_probs, True)
    if Nt != N or target_probs.shape[-1] != logits.shape[-1]:
        raise ValueError("target_probs must have the shape of logits")
    V = logits.shape[-1]
    grad_out, g_stride = _grad_view(torch, grad_out, N)
    if dlogits is None:
        dlogits = torch.empty(logits.shape, dtype=out_dtype or logits.dtype, device=logits.device)
    Nd, dl = row_layout(dlogits, True)
    if Nd != N or dlogits.shape[-1] != V:
        raise ValueError("dlogits must have the shape of logits")
    with torch.cuda.device(logits.device):
        st = lib().ce_soft_backward(_ptr(grad_out), g_stride, _ptr(logits), _dtype_code(logits), lg, N, V,
                                    _ptr(target_probs), _dtype_code(target_probs), tl, _ptr(lse),
                                    _ptr(lse_lo), _ptr(target_sum), float(label_smoothing),
                                    _ptr(dlogits), _dtype_code(dlogits), dl, _stream(stream))
    _check(st, "ce_soft_backward")
    return dlogits


class KlResult(NamedTuple):
    loss: object
    lse_student: object
    lse_student_lo: object
    lse_teacher: object
    lse_teacher_lo: object


def _same_rows(a, b, what):
    Na, la = row_layout(a, True)
    Nb, lb = row_layout(b, True)
    if Na != Nb or a.shape[-1] != b.shape[-1]:
        raise ValueError(f"{what} must have the shape of the student logits")
    return Na, la, lb


def kl_forward(student, teacher, *, stream=None) -> KlResult:
    """KL(softmax(teacher) || softmax(student)) per row, with both lse pairs.
    student and teacher: same shape and dtype, any strides."""
    torch = _torch()
    _require_cuda(student, teacher)
    if teacher.dtype != student.dtype:
        raise TypeError("student and teacher logits must share a dtype")
    N, ls, lt = _same_rows(student, teacher, "teacher logits")
    V = student.shape[-1]
    dev = student.device
    outs = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(5)]
    with torch.cuda.device(dev):
        st = lib().ce_kl_forward(_ptr(student), _ptr(teacher), _dtype_code(student), ls, lt, N, V,
                                 *[_ptr(o) for o in outs], _stream(stream))
    _check(st, "ce_kl_forward")
    return KlResult(*outs)


def kl_backward(grad_out, student, teacher, r: KlResult, *, dstudent=None, out_dtype=None, stream=None):
    """g (softmax(student) - softmax(teacher)) from kl_forward's lse pairs."""
    torch = _torch()
    _require_cuda(grad_out, student, teacher, dstudent)
    N, ls, lt = _same_rows(student, teacher, "teacher logits")
    V = student.shape[-1]
    grad_out, g_stride = _grad_view(torch, grad_out, N)
    if dstudent is None:
        dstudent = torch.empty(student.shape, dtype=out_dtype or student.dtype, device=student.device)
    Nd, dl = row_layout(dstudent, True)
    if Nd != N or dstudent.shape[-1] != V:
        raise ValueError("dstudent must have the shape of the student logits")
    with torch.cuda.device(student.device):
        st = lib().ce_kl_backward(_ptr(grad_out), g_stride, _ptr(student), _ptr(teacher),
                                  _dtype_code(student), ls, lt, N, V, _ptr(r.lse_student),
                                  _ptr(r.lse_student_lo), _ptr(r.lse_teacher), _ptr(r.lse_teacher_lo),
                                  _ptr(dstudent), _dtype_code(dstudent), dl, _stream(stream))
    _check(st, "ce_kl_backward")
    return dstudent


def ce_forward_backward(logits, targets, grad_out, label_smoothing: float = 0.0,
                        ignore_index: int = -100, *, return_argmax: bool = False, dlogits=None,
                        out_dtype=None, workspace=None, stream=None, out=None):
    """Forward and VJP in one call (g known up front). Returns (ForwardResult,
    dlogits); rows that fit on chip are read from HBM once. `out` as for
    ce_forward."""
    torch = _torch()
    _require_cuda(logits, targets, grad_out, dlogits)
    N, lg = row_layout(logits, True)
    Nt, tg = row_layout(targets, False)
    if Nt != N:
        raise ValueError(f"targets hold {Nt} rows, logits {N}")
    V = logits.shape[-1]
    if grad_out.dtype != torch.float32:
        raise TypeError("grad_out must be float32")
    if grad_out.numel() == 1:
        g_stride = 0
    else:
        if grad_out.numel() != N or grad_out.dim() != 1:
            raise ValueError("grad_out must hold one value per row (1-D) or a single value")
        g_stride = grad_out.stride(0)
    dev = logits.device
    if dlogits is None:
        dlogits = torch.empty(logits.shape, dtype=out_dtype or logits.dtype, device=dev)
    Nd, dl = row_layout(dlogits, True)
    if Nd != N or dlogits.shape[-1] != V:
        raise ValueError("dlogits must have the shape of logits")
    loss, lse, lse_lo, am = _row_outputs(N, dev, return_argmax, out)
    dt = _dtype_code(logits)
    with torch.cuda.device(dev):
        need = int(lib().ce_workspace_size(N, V, dt, 0))
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib().ce_forward_backward(_ptr(logits), dt, lg, N, V, _ptr(targets),
                                       _index_code(targets), tg, float(label_smoothing),
                                       int(ignore_index), _ptr(grad_out), g_stride, _ptr(loss),
                                       _ptr(lse), _ptr(lse_lo), _ptr(am), _ptr(dlogits),
                                       _dtype_code(dlogits), dl, _ptr(workspace), ws_bytes,
                                       _stream(stream))
    _check(st, "ce_forward_backward")
    return ForwardResult(loss, lse, lse_lo, am), dlogits


def get_error(stream=None) -> int:
    """Waits for the stream and returns (and clears) the device error status."""
    return int(lib().ce_get_error(_stream(stream)))


def testing_set_wait(limit_ns: int = 0, starve: bool = False) -> None:
    """Testing hook of the bounded pipeline waits (ce_testing_set_wait): the
    wait limit for later launches (0 = the default) and whether they issue
    no copies, so that their waits run out. Not for production use."""
    _check(lib().ce_testing_set_wait(int(limit_ns), 1 if starve else 0), "ce_testing_set_wait")


# -- fused-linear cross-entropy ----------------------------------------------------------
def linear_ce_forward(H, W, targets, label_smoothing: float = 0.0, ignore_index: int = -100, *,
                      workspace=None, stream=None):
    """loss, lse of Z = H W^T (bf16 H (N, D), W (V, D)); Z is never stored."""
    torch = _torch()
    _require_cuda(H, W, targets)
    if H.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise TypeError("H and W must be bfloat16")
    if H.stride(1) != 1 or W.stride(1) != 1 or targets.dim() != 1 or targets.stride(0) != 1:
        raise ValueError("H, W need unit column stride and targets must be contiguous")
    N, D = H.shape
    V = W.shape[0]
    loss = torch.empty(N, dtype=torch.float32, device=H.device)
    lse = torch.empty(N, dtype=torch.float32, device=H.device)
    with torch.cuda.device(H.device):
        need = int(lib().linear_ce_workspace_size(N, V, D, 0))
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=H.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib().linear_ce_forward(_ptr(H), H.stride(0), _ptr(W), W.stride(0), _ptr(targets),
                                     _index_code(targets), N, V, D, float(label_smoothing),
                                     int(ignore_index), _ptr(loss), _ptr(lse), _ptr(workspace),
                                     ws_bytes, _stream(stream))
    _check(st, "linear_ce_forward")
    return loss, lse


def linear_ce_backward(grad_out, H, W, targets, lse, label_smoothing: float = 0.0,
                       ignore_index: int = -100, *, dH_dtype=None, dW_dtype=None,
                       workspace=None, stream=None):
    """dH (N, D) and dW (V, D) with the logits recomputed chunk by chunk."""
    torch = _torch()
    _require_cuda(grad_out, H, W, targets, lse)
    N, D = H.shape
    V = W.shape[0]
    g_stride = 0 if grad_out.numel() == 1 else grad_out.stride(0)
    dH = torch.empty((N, D), dtype=dH_dtype or torch.bfloat16, device=H.device)
    dW = torch.empty((V, D), dtype=dW_dtype or torch.bfloat16, device=H.device)
    with torch.cuda.device(H.device):
        need = int(lib().linear_ce_backward_workspace_size(N, V, D, 0))
        if workspace is None and need > 0:
            workspace = torch.empty(need, dtype=torch.uint8, device=H.device)
        ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        st = lib().linear_ce_backward(_ptr(grad_out), g_stride, _ptr(H), H.stride(0), _ptr(W),
                                      W.stride(0), _ptr(targets), _index_code(targets), _ptr(lse),
                                      N, V, D, float(label_smoothing), int(ignore_index), _ptr(dH),
                                      _dtype_code(dH), _ptr(dW), _dtype_code(dW), _ptr(workspace),
                                      ws_bytes, _stream(stream))
    _check(st, "linear_ce_backward")
    return dH, dW
