"""Python binding of libhaste.so: the C ABI of ``include/haste.h`` under the same
names, with argument marshalling only.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback path.  PyTorch supplies device
memory and streams.

Tensors are passed as torch CUDA tensors (contiguous, row-major); the plan's
index array is a host numpy int32 array.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhaste.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "haste.h")

HASTE_OK = 0
HASTE_ERR_INVALID_ARG = 1
HASTE_ERR_INDEX_UNSORTED_OR_DUP = 2
HASTE_ERR_INDEX_OUT_OF_RANGE = 3
HASTE_ERR_UNSUPPORTED_SHAPE = 4
HASTE_ERR_WORKSPACE = 5
HASTE_ERR_CUDA = 6
HASTE_ERR_TIMEOUT = 7
HASTE_F32 = 0
HASTE_BF16 = 1

_STATUS_NAMES = {v: k for k, v in globals().items() if k.startswith("HASTE_ERR_") or k == "HASTE_OK"}


class HasteError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class Targets(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("ids", ctypes.c_void_p)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_double)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhaste.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python {os.path.join(_HERE, 'csrc', 'build.py')}`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    S = ctypes.c_int
    sig = {
        "haste_abi_version": ([], ctypes.c_int),
        "haste_last_error": ([], ctypes.c_char_p),
        "haste_device_status": ([P], S),
        "haste_selftest_wait_timeout": ([P], S),
        "haste_set_wait_limit_ns": ([ctypes.c_uint64], S),
        "haste_profile_start": ([], S),
        "haste_profile_stop": ([P, I32], I32),
        "haste_plan_inverse_host": ([P, I64, I32, I32, P, P], S),
        "haste_plan": ([P, P, I64, I32, I32, I32, P], S),
        "haste_plan_destroy": ([P], S),
        "haste_plan_update": ([P, P, I64, P, P], S),
        "haste_plan_info": ([P, P, P], S),
        "haste_plan_export": ([P, P, P, P], S),
        "haste_workspace_size": ([P, I32, S], SZ),
        "haste_forward": ([P, I32, S, P, P, P, P, SZ, P], S),
        "haste_backward_dw": ([P, I32, S, P, P, P, P, SZ, P], S),
        "haste_backward_dx": ([P, I32, S, P, P, P, S, P, SZ, P], S),
        "haste_backward_dx_noalloc": ([P, I32, S, P, P, P, S, P], S),
        "haste_bce_step": ([P, I32, S, P, P, Targets, F, P, P, P, S, P, SZ, P], S),
        "haste_bce_step_sgd": ([P, I32, S, P, P, Targets, F, P, F, F, P, P, P, S, P, SZ, P], S),
        "haste_topk_workspace_size": ([P, I32, S, I32, I32], SZ),
        "haste_topk": ([P, I32, S, P, P, I32, I32, I32, P, P, P, SZ, P], S),
        "haste_head_workspace_size": ([I32, I32, I32, S], SZ),
        "haste_head_forward": ([I32, I32, I32, S, P, P, P, P, F, P, P, SZ, P], S),
        "haste_head_backward": ([I32, I32, I32, S, P, P, P, P, P, P, SZ, P], S),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _check(status: int, where: str) -> None:
    if status != HASTE_OK:
        raise HasteError(status, where, lib().haste_last_error().decode())


def _np_ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _tptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must be CUDA tensors (the library reads them on the GPU)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream) if not hasattr(stream, "cuda_stream") else stream.cuda_stream


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return HASTE_BF16
    if t.dtype == torch.float32:
        return HASTE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _torch_dtype(code: int):
    import torch
    return torch.bfloat16 if code == HASTE_BF16 else torch.float32


def _expect(t, name: str, shape, dtype=None):
    """Shape and dtype of one tensor argument (before any pointer is taken)."""
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _same_device(device, **tensors):
    """Every tensor on one CUDA device, the plan's when a plan is involved."""
    devs = {n: t.device for n, t in tensors.items() if t is not None}
    want = device if device is not None else next(iter(devs.values()))
    for n, dv in devs.items():
        if dv.type != "cuda":
            raise ValueError(f"{n} is on {dv}; tensors must be CUDA tensors (the library reads them on the GPU)")
        if want.type == "cuda" and (dv.index or 0) != (want.index or 0):
            raise ValueError(f"{n} is on {dv}, but the call's device is {want}")


def _plan_device(plan):
    import torch
    return torch.device("cuda", plan.device) if plan.device is not None else None


def _tail_tensors(plan, B: int, code: int, **named):
    """Shapes and dtypes of the sparse-tail arguments: X [B, d], W [L, k], dY and
    logits [B, L] in the input dtype; dW [L, k] like W; dX [B, d] fp32."""
    import torch
    dt = _torch_dtype(code)
    shapes = {"X": ((B, plan.d), dt), "W": ((plan.L, plan.k), dt), "dY": ((B, plan.L), dt),
              "logits": ((B, plan.L), dt), "dW": ((plan.L, plan.k), dt), "dX": ((B, plan.d), torch.float32)}
    for n, t in named.items():
        _expect(t, n, *shapes[n])
    _same_device(_plan_device(plan), **named)


def _targets(row_ptr, ids, B: int, name: str):
    import torch
    _expect(row_ptr, f"{name} row_ptr", (B + 1,), torch.int32)
    if ids is None or ids.dim() != 1 or ids.dtype != torch.int32:
        raise ValueError(f"{name} ids must be a 1-D int32 tensor")


def _scalar_out(t, name: str):
    import torch
    if t is not None and (t.dtype != torch.float32 or t.numel() < 1):
        raise ValueError(f"{name} must be a float32 tensor of at least one element")


# ---------------------------------------------------------------- the plan
def haste_plan_inverse_host(idx: np.ndarray, d: int) -> Tuple[np.ndarray, np.ndarray]:
    """Host-only validation and inverse map (no GPU needed)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    n_groups, k = idx.shape
    inv_off = np.empty(d + 1, dtype=np.int32)
    inv_ent = np.empty(n_groups * k, dtype=np.int32)
    _check(lib().haste_plan_inverse_host(_np_ptr(idx), n_groups, k, d, _np_ptr(inv_off), _np_ptr(inv_ent)),
           "haste_plan_inverse_host")
    return inv_off, inv_ent


class Plan:
    """Owner of a haste_plan_t (freed on close() or garbage collection)."""

    def __init__(self, handle: int, n_groups: int, G: int, k: int, d: int, device: Optional[int] = None):
        self.handle, self.n_groups, self.G, self.k, self.d = handle, n_groups, G, k, d
        self.device = device  # CUDA ordinal the plan's arrays live on

    @property
    def L(self) -> int:
        return self.n_groups * self.G

    def close(self) -> None:
        if self.handle:
            lib().haste_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def info(self) -> Tuple[int, int]:
        a, b = ctypes.c_int64(), ctypes.c_int64()
        _check(lib().haste_plan_info(self.handle, ctypes.byref(a), ctypes.byref(b)), "haste_plan_info")
        return a.value, b.value

    def export(self):
        idx = np.empty((self.n_groups, self.k), dtype=np.int32)
        off = np.empty(self.d + 1, dtype=np.int32)
        ent = np.empty(self.n_groups * self.k, dtype=np.int32)
        _check(lib().haste_plan_export(self.handle, _np_ptr(idx), _np_ptr(off), _np_ptr(ent)), "haste_plan_export")
        return idx, off, ent

    def update(self, groups: np.ndarray, rows: np.ndarray, stream=None) -> None:
        """Replace the index rows of `groups` (ascending group ids) by `rows`
        [len(groups), k] and rebuild the inverse map on the device."""
        groups = np.ascontiguousarray(groups, dtype=np.int32)
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        if rows.shape != (len(groups), self.k):
            raise ValueError(f"rows has shape {rows.shape}, expected {(len(groups), self.k)}")
        _check(lib().haste_plan_update(self.handle, _np_ptr(groups), len(groups), _np_ptr(rows), _stream(stream)),
               "haste_plan_update")

    def workspace_size(self, B: int, dtype: int) -> int:
        return int(lib().haste_workspace_size(self.handle, B, dtype))


def haste_plan(idx: np.ndarray, G: int, d: int, stream=None) -> Plan:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    n_groups, k = idx.shape
    h = ctypes.c_void_p()
    _check(lib().haste_plan(ctypes.byref(h), _np_ptr(idx), n_groups, G, k, d, _stream(stream)), "haste_plan")
    import torch
    return Plan(h.value, n_groups, G, k, d, torch.cuda.current_device())


def haste_device_status(stream=None) -> int:
    return lib().haste_device_status(_stream(stream))


def haste_set_wait_limit_ns(ns: int) -> None:
    """Limit of the pipelined kernels' inter-warp waits (0: the 2 s default)."""
    _check(lib().haste_set_wait_limit_ns(int(ns)), "haste_set_wait_limit_ns")


def haste_profile_start() -> None:
    _check(lib().haste_profile_start(), "haste_profile_start")


def haste_profile_stop():
    """{kernel name: (launches, total ms)} of the launches since haste_profile_start()."""
    buf = (KernelTime * 64)()
    n = lib().haste_profile_stop(buf, 64)
    if n < 0:
        raise HasteError(HASTE_ERR_CUDA, "haste_profile_stop", "event timing failed")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(min(n, 64))}


# ------------------------------------------------------------- sparse tail
def _ws(ws):
    return (_tptr(ws), ws.numel() * ws.element_size()) if ws is not None else (None, 0)


def haste_forward(plan: Plan, X, W, logits, ws, stream=None) -> None:
    _tail_tensors(plan, X.shape[0], dtype_code(X), X=X, W=W, logits=logits)
    p, n = _ws(ws)
    _check(lib().haste_forward(plan.handle, X.shape[0], dtype_code(X), _tptr(X), _tptr(W), _tptr(logits), p, n,
                               _stream(stream)), "haste_forward")


def haste_backward_dw(plan: Plan, X, dY, dW, ws, stream=None) -> None:
    _tail_tensors(plan, X.shape[0], dtype_code(X), X=X, dY=dY, dW=dW)
    p, n = _ws(ws)
    _check(lib().haste_backward_dw(plan.handle, X.shape[0], dtype_code(X), _tptr(X), _tptr(dY), _tptr(dW), p, n,
                                   _stream(stream)), "haste_backward_dw")


def haste_backward_dx(plan: Plan, W, dY, dX, ws, accumulate: bool = False, stream=None) -> None:
    _tail_tensors(plan, dY.shape[0], dtype_code(W), W=W, dY=dY, dX=dX)
    p, n = _ws(ws)
    _check(lib().haste_backward_dx(plan.handle, dY.shape[0], dtype_code(W), _tptr(W), _tptr(dY), _tptr(dX),
                                   int(accumulate), p, n, _stream(stream)), "haste_backward_dx")


def haste_backward_dx_noalloc(plan: Plan, W, dY, dX, accumulate: bool = False, stream=None) -> None:
    """dX with no workspace and no device allocation (library-owned static scratch)."""
    _tail_tensors(plan, dY.shape[0], dtype_code(W), W=W, dY=dY, dX=dX)
    _check(lib().haste_backward_dx_noalloc(plan.handle, dY.shape[0], dtype_code(W), _tptr(W), _tptr(dY), _tptr(dX),
                                           int(accumulate), _stream(stream)), "haste_backward_dx_noalloc")


def haste_bce_step(plan: Plan, X, W, pos_row_ptr, pos_ids, grad_scale: float, loss, dW, dX, ws,
                   accumulate: bool = False, stream=None) -> None:
    B = X.shape[0]
    _targets(pos_row_ptr, pos_ids, B, "tail positives")
    _scalar_out(loss, "loss")
    _tail_tensors(plan, B, dtype_code(X), X=X, W=W, dW=dW, dX=dX)
    _same_device(_plan_device(plan), X=X, pos_row_ptr=pos_row_ptr, pos_ids=pos_ids, loss=loss)
    p, n = _ws(ws)
    tg = Targets(_tptr(pos_row_ptr), _tptr(pos_ids))
    _check(lib().haste_bce_step(plan.handle, X.shape[0], dtype_code(X), _tptr(X), _tptr(W), tg, float(grad_scale),
                                _tptr(loss), _tptr(dW), _tptr(dX), int(accumulate), p, n, _stream(stream)),
           "haste_bce_step")


def haste_bce_step_sgd(plan: Plan, X, W, pos_row_ptr, pos_ids, grad_scale: float, loss, lr: float,
                       momentum: float, M, W_out, dX, ws, accumulate: bool = False, stream=None) -> None:
    """Fused step with an SGD (momentum) update in place of the dW output:
    M <- momentum*M + dW, W_out <- W - lr*M (W itself is not written)."""
    B = X.shape[0]
    _targets(pos_row_ptr, pos_ids, B, "tail positives")
    _scalar_out(loss, "loss")
    _tail_tensors(plan, B, dtype_code(X), X=X, W=W, dX=dX)
    _expect(W_out, "W_out", tuple(W.shape), W.dtype)
    if M is not None:
        _expect(M, "M", tuple(W.shape), W.dtype)
    elif momentum != 0.0:
        raise ValueError("momentum != 0 needs the momentum buffer M")
    _same_device(_plan_device(plan), X=X, W_out=W_out, M=M, pos_row_ptr=pos_row_ptr, pos_ids=pos_ids, loss=loss)
    p, n = _ws(ws)
    tg = Targets(_tptr(pos_row_ptr), _tptr(pos_ids))
    _check(lib().haste_bce_step_sgd(plan.handle, B, dtype_code(X), _tptr(X), _tptr(W), tg, float(grad_scale),
                                    _tptr(loss), float(lr), float(momentum), _tptr(M), _tptr(W_out), _tptr(dX),
                                    int(accumulate), p, n, _stream(stream)), "haste_bce_step_sgd")


# ------------------------------------------------------------ top-k scoring
def haste_topk_workspace_size(plan: Plan, B: int, dtype: int, n_buckets: int, kp: int) -> int:
    return int(lib().haste_topk_workspace_size(plan.handle, B, dtype, n_buckets, kp))


def haste_topk(plan: Plan, X, W, k: int, kp: int, n_buckets: int, out_val, out_id, ws, stream=None) -> None:
    """Two-stage top-k of the tail logits per sample (see include/haste.h):
    out_val [B, k] fp32 and out_id [B, k] int32, larger logit first."""
    import torch
    B = X.shape[0]
    _expect(out_val, "out_val", (B, k), torch.float32)
    _expect(out_id, "out_id", (B, k), torch.int32)
    _tail_tensors(plan, B, dtype_code(X), X=X, W=W)
    _same_device(_plan_device(plan), X=X, out_val=out_val, out_id=out_id)
    p, n = _ws(ws)
    _check(lib().haste_topk(plan.handle, X.shape[0], dtype_code(X), _tptr(X), _tptr(W), int(k), int(kp),
                            int(n_buckets), _tptr(out_val), _tptr(out_id), p, n, _stream(stream)), "haste_topk")


# ---------------------------------------------------------------- dense head
def _head_tensors(B: int, H: int, d: int, xdtype, **named):
    """Xh [B, d], Wh [H, d], logits / dY_h [B, H] and dWh [H, d] in Xh's dtype;
    dXh [B, d] fp32; all on Xh's device."""
    import torch
    if xdtype not in (torch.bfloat16, torch.float32):
        raise TypeError(f"unsupported dtype {xdtype}")
    dt = xdtype
    shapes = {"Xh": ((B, d), dt), "Wh": ((H, d), dt), "logits_or_dY": ((B, H), dt), "dYh": ((B, H), dt),
              "dWh": ((H, d), dt), "dXh": ((B, d), torch.float32)}
    for n, t in named.items():
        _expect(t, n, *shapes[n])
    _same_device(None, **named)


def haste_head_workspace_size(B: int, H: int, d: int, dtype: int) -> int:
    return int(lib().haste_head_workspace_size(B, H, d, dtype))


def haste_head_forward(Xh, Wh, out, ws, pos_row_ptr=None, pos_ids=None, grad_scale: float = 1.0, loss=None,
                       stream=None) -> None:
    B, d = Xh.shape
    H = Wh.shape[0]
    _head_tensors(B, H, d, Xh.dtype, Xh=Xh, Wh=Wh, logits_or_dY=out)
    if pos_row_ptr is not None:
        _targets(pos_row_ptr, pos_ids, B, "head positives")
        _same_device(Xh.device, pos_row_ptr=pos_row_ptr, pos_ids=pos_ids)
    _scalar_out(loss, "loss")
    _same_device(Xh.device, loss=loss)
    p, n = _ws(ws)
    tg = None
    if pos_row_ptr is not None:
        tg = ctypes.byref(Targets(_tptr(pos_row_ptr), _tptr(pos_ids)))
    _check(lib().haste_head_forward(B, H, d, dtype_code(Xh), _tptr(Xh), _tptr(Wh), _tptr(out), tg,
                                    float(grad_scale), _tptr(loss), p, n, _stream(stream)), "haste_head_forward")


def haste_head_backward(Xh, Wh, dYh, dWh, dXh, ws, stream=None) -> None:
    B, d = Xh.shape
    H = Wh.shape[0]
    _head_tensors(B, H, d, Xh.dtype, Xh=Xh, Wh=Wh, dYh=dYh, dWh=dWh, dXh=dXh)
    p, n = _ws(ws)
    _check(lib().haste_head_backward(B, H, d, dtype_code(Xh), _tptr(Xh), _tptr(Wh), _tptr(dYh), _tptr(dWh),
                                     _tptr(dXh), p, n, _stream(stream)), "haste_head_backward")
