"""Python face of the fp64 oracle (``haste_ref.c``) plus the dense-head oracle.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It never imports the
CUDA library and the CUDA library never imports it.

Source: "HASTE: Hardware-Aware Dynamic Sparse Training for Large Output Spaces"
(summary page), Methodology 1 (group-shared fixed fan-in sparsity: one shared
fan-in index set per group, an own weight vector per label, indices stored once
per group) and Methodology 2 (head-tail decomposition: a dense classifier over the
few frequent head labels).  The loss, binary cross-entropy with logits against
sparse positive lists, summed over labels and scaled by 1/B, is this project's
reading; the page names no loss.

Functions return float64 arrays.  bf16 inputs are uint16 bit patterns and widen
exactly.  Parity status: every function here is pinned by ``tests/test_oracle.py``
(dense masked products, brute-force loops, finite differences, closed forms).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "haste_ref.c")
_LIB = os.path.join(_HERE, "libhaste_ref.so")
_lib = None

OK, ERR_ARG, ERR_UNSORTED, ERR_RANGE = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, -O2, OpenMP) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c11", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.ref_validate.argtypes = [P, I64, I32, I32]
        lib.ref_plan.argtypes = [P, I64, I32, I32, P, P]
        C = ctypes.c_int
        lib.ref_forward.argtypes = [C, P, C, P, P, I32, I32, I64, I32, I32, P]
        lib.ref_backward_dw.argtypes = [C, P, C, P, P, I32, I32, I64, I32, I32, P]
        lib.ref_backward_dx.argtypes = [C, P, C, P, P, I32, I32, I64, I32, I32, P]
        lib.ref_bce.argtypes = [P, P, P, I32, I64, D, P]
        lib.ref_bce.restype = D
        lib.ref_logits_at.argtypes = [ctypes.c_int, P, P, P, I32, I32, I32, I64, P, P, P]
        lib.ref_dw_at.argtypes = [ctypes.c_int, P, P, P, P, I32, I32, I64, I32, I32, ctypes.c_int,
                                  P, P, D, I64, P, P, P]
        lib.ref_dx_at.argtypes = [ctypes.c_int, P, P, P, P, I32, I32, I64, I32, I32, ctypes.c_int,
                                  P, P, D, I64, P, P, P]
        lib.ref_topk.argtypes = [ctypes.c_int, P, P, P, I32, I64, I32, I32, I32, I32, I32, I64, P, P, P]
        lib.ref_bce_loss.argtypes = [ctypes.c_int, P, P, P, I32, I32, I64, I32, I32, P, P, D]
        lib.ref_bce_loss.restype = D
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    if a.dtype == np.float64:
        return 2
    raise TypeError(f"oracle takes fp32, bf16 bits (uint16) or fp64, got {a.dtype}")


def _c(a, dtype=None):
    return np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of fp32 or bf16-bit arrays to float64."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# --------------------------------------------------------------------- the plan
def plan(idx: np.ndarray, d: int) -> Tuple[int, np.ndarray, np.ndarray]:
    """(status, inv_off int32 [d+1], inv_ent int32 [n_groups*k])."""
    idx = _c(idx, np.int32)
    n_groups, k = idx.shape
    inv_off = np.zeros(d + 1, dtype=np.int32)
    inv_ent = np.zeros(n_groups * k, dtype=np.int32)
    st = _load().ref_plan(_ptr(idx), n_groups, k, d, _ptr(inv_off), _ptr(inv_ent))
    return st, inv_off, inv_ent


def validate(idx: np.ndarray, d: int) -> int:
    idx = _c(idx, np.int32)
    return _load().ref_validate(_ptr(idx), idx.shape[0], idx.shape[1], d)


def index_bytes(n_groups: int, k: int) -> int:
    """Bytes of the group-shared index store: one int32 per (group, slot)."""
    return 4 * n_groups * k


# ------------------------------------------------------------ the sparse tail
def forward(X, W, idx, G: int) -> np.ndarray:
    X, W, idx = _c(X), _c(W), _c(idx, np.int32)
    B, d = X.shape
    n_groups, k = idx.shape
    out = np.empty((B, n_groups * G), dtype=np.float64)
    _load().ref_forward(_dt(X), _ptr(X), _dt(W), _ptr(W), _ptr(idx), B, d, n_groups, G, k, _ptr(out))
    return out


def backward_dw(X, dY, idx, G: int) -> np.ndarray:
    X, dY, idx = _c(X), _c(dY), _c(idx, np.int32)
    B, d = X.shape
    n_groups, k = idx.shape
    out = np.empty((n_groups * G, k), dtype=np.float64)
    _load().ref_backward_dw(_dt(X), _ptr(X), _dt(dY), _ptr(dY), _ptr(idx), B, d, n_groups, G, k,
                            _ptr(out))
    return out


def backward_dx(W, dY, idx, G: int, d: int) -> np.ndarray:
    W, dY, idx = _c(W), _c(dY), _c(idx, np.int32)
    B = dY.shape[0]
    n_groups, k = idx.shape
    out = np.empty((B, d), dtype=np.float64)
    _load().ref_backward_dx(_dt(W), _ptr(W), _dt(dY), _ptr(dY), _ptr(idx), B, d, n_groups, G, k,
                            _ptr(out))
    return out


def bce(logits: np.ndarray, row_ptr, ids, scale: float, want_grad: bool = True):
    """(loss, dY or None) of BCE-with-logits against the CSR positives."""
    logits = _c(logits, np.float64)
    B, L = logits.shape
    row_ptr, ids = _c(row_ptr, np.int32), _c(ids, np.int32)
    dY = np.empty_like(logits) if want_grad else None
    loss = _load().ref_bce(_ptr(logits), _ptr(row_ptr), _ptr(ids), B, L, scale, _ptr(dY))
    return loss, dY


def bce_step(X, W, idx, G: int, row_ptr, ids, scale: float):
    """Fused tail step: forward, BCE loss and gradient, then dW and dX from the
    fp64 gradient (all in fp64)."""
    d = X.shape[1]
    z = forward(X, W, idx, G)
    loss, dY = bce(z, row_ptr, ids, scale)
    dW = backward_dw(X, dY, idx, G)
    dX = backward_dx(W, dY, idx, G, d)
    return loss, dY, dW, dX


def bce_loss(X, W, idx, G: int, row_ptr, ids, scale: float) -> float:
    """The fused step's tail loss alone (forward + BCE sum, no B x L logits kept),
    for full-size checks.  X and W share one dtype."""
    X, W, idx = _c(X), _c(W), _c(idx, np.int32)
    if _dt(X) != _dt(W):
        raise TypeError("bce_loss takes X and W of one dtype")
    row_ptr, ids = _c(row_ptr, np.int32), _c(ids, np.int32)
    B, d = X.shape
    n_groups, k = idx.shape
    return float(_load().ref_bce_loss(_dt(X), _ptr(X), _ptr(W), _ptr(idx), B, d, n_groups, G, k,
                                      _ptr(row_ptr), _ptr(ids), scale))


# ------------------------------------------------------- optimizer update
def sgd_update(W, M, dW64, lr: float, momentum: float):
    """One step of SGD with heavy-ball momentum on the tail weights, in fp64:
    M' = momentum * M + dW and W' = W - lr * M' (momentum = 0: M' = dW, W' =
    W - lr * dW).  W and M are fp32, bf16 bits or fp64 (M may be None when
    momentum is 0); returns (W', M') as float64.  This is the update the fused
    step applies to each group's weights while its dW is still on chip; the
    training loop it serves is the one of the HASTE summary page's experiments
    (the page names no optimizer: plain SGD with momentum is this library's
    choice)."""
    W64 = to_f64(np.asarray(W))
    M64 = np.zeros_like(W64) if M is None else to_f64(np.asarray(M))
    M_new = momentum * M64 + dW64
    return W64 - lr * M_new, M_new


def bce_step_sgd(X, W, M, idx, G: int, row_ptr, ids, scale: float, lr: float, momentum: float):
    """Fused tail step with the update: (loss, dX, W', M') in fp64; dX uses the
    weights before the update."""
    loss, _, dW, dX = bce_step(X, W, idx, G, row_ptr, ids, scale)
    W_new, M_new = sgd_update(W, M, dW, lr, momentum)
    return loss, dX, W_new, M_new


# ------------------------------------------------ sampled single-output checks
def logits_at(X, W, idx, G, bs, ls) -> np.ndarray:
    X, W, idx = _c(X), _c(W), _c(idx, np.int32)
    bs, ls = _c(bs, np.int32), _c(ls, np.int64)
    out = np.empty(len(bs))
    _load().ref_logits_at(_dt(X), _ptr(X), _ptr(W), _ptr(idx), X.shape[1], G, idx.shape[1],
                          len(bs), _ptr(bs), _ptr(ls), _ptr(out))
    return out


def dw_at(X, W, idx, G, ls, ss, *, dY=None, pos=None, scale=1.0) -> np.ndarray:
    X, W, idx = _c(X), _c(W), _c(idx, np.int32)
    ls, ss = _c(ls, np.int64), _c(ss, np.int32)
    fused = dY is None
    rp, ids = (None, None) if pos is None else (_c(pos[0], np.int32), _c(pos[1], np.int32))
    dY = None if dY is None else _c(dY)
    out = np.empty(len(ls))
    L = idx.shape[0] * G
    _load().ref_dw_at(_dt(X), _ptr(X), _ptr(W), _ptr(dY), _ptr(idx), X.shape[0], X.shape[1], L,
                      G, idx.shape[1], int(fused), _ptr(rp), _ptr(ids), scale, len(ls),
                      _ptr(ls), _ptr(ss), _ptr(out))
    return out


def dx_at(X, W, idx, G, bs, fs, *, dY=None, pos=None, scale=1.0) -> np.ndarray:
    X, W, idx = _c(X), _c(W), _c(idx, np.int32)
    bs, fs = _c(bs, np.int32), _c(fs, np.int32)
    fused = dY is None
    rp, ids = (None, None) if pos is None else (_c(pos[0], np.int32), _c(pos[1], np.int32))
    dY = None if dY is None else _c(dY)
    out = np.empty(len(bs))
    L = idx.shape[0] * G
    _load().ref_dx_at(_dt(X), _ptr(X), _ptr(W), _ptr(dY), _ptr(idx), X.shape[0], X.shape[1], L,
                      G, idx.shape[1], int(fused), _ptr(rp), _ptr(ids), scale, len(bs),
                      _ptr(bs), _ptr(fs), _ptr(out))
    return out


# ------------------------------------------------------- two-stage top-k scoring
def topk(X, W, idx, G, K, Kp, n_buckets, rows=None) -> Tuple[np.ndarray, np.ndarray]:
    """Two-stage top-K of the tail logits of the given sample rows ("A Faster
    Generalized Two-Stage Approximate Top-K", Methodology): stage 1 keeps the top
    Kp of each bucket, bucket j = the labels of groups [j*n_g/nb, (j+1)*n_g/nb);
    stage 2 returns the top K of the survivors.  Order: larger logit first, equal
    logits by smaller label id.  Returns (values float64 [n, K], ids int64 [n, K])."""
    X, W, idx = _c(X), _c(W), _c(idx, np.int32)
    B = X.shape[0]
    rows = np.arange(B, dtype=np.int32) if rows is None else _c(rows, np.int32)
    n_groups = idx.shape[0]
    vals = np.empty((len(rows), K))
    ids = np.empty((len(rows), K), dtype=np.int64)
    _load().ref_topk(_dt(X), _ptr(X), _ptr(W), _ptr(idx), X.shape[1], n_groups, G, idx.shape[1], K, Kp,
                     n_buckets, len(rows), _ptr(rows), _ptr(vals), _ptr(ids))
    return vals, ids


# ---------------------------------------------------------------- dense head
def head_forward(Xh, Wh) -> np.ndarray:
    """logits_h = Xh . Wh^T (dense classifier over the head labels)."""
    return to_f64(Xh) @ to_f64(Wh).T


def head_backward(Xh, Wh, dYh64) -> Tuple[np.ndarray, np.ndarray]:
    """(dWh = dY_h^T . Xh, dXh = dY_h . Wh)."""
    return dYh64.T @ to_f64(Xh), dYh64 @ to_f64(Wh)


def head_step(Xh, Wh, row_ptr, ids, scale: float):
    z = head_forward(Xh, Wh)
    loss, dY = bce(z, row_ptr, ids, scale)
    dWh, dXh = head_backward(Xh, Wh, dY)
    return loss, dY, dWh, dXh
