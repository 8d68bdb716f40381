"""Seeded synthetic inputs for the group-shared fixed fan-in output layer.

This module only draws random numbers and lays them out; it holds none of the
layer's arithmetic.  The oracle (under ``oracle/``) and the CUDA path both take
their inputs from here, so the two sides see bit-identical operands.

Recipe (numpy PCG64, one independent stream per tensor, seed = [base, tensor_id]):

* ``idx``     -- each group's fan-in set is k distinct features drawn uniformly
                 from [0, d) and sorted ascending (HASTE, method section 1
                 "structure": all labels of a group share one input-feature set).
* ``X``, ``Xh`` -- N(0, 1) drawn in fp32, then rounded to bf16 (round to nearest
                 even) when the workload is bf16.
* ``W``       -- N(0, 1/k) (variance 1/k, so logits are about N(0, 1)).
* ``Wh``      -- N(0, 1/d).
* ``dY``      -- N(0, 1) upstream gradient for the given-gradient calls.
* positives   -- p distinct label ids per sample from a finite Zipf law,
                 P(id) proportional to (id + 1) ** -alpha over [0, H + L), drawn by
                 inverse CDF; ids below H are head labels (the most frequent),
                 the rest are tail labels with local id = id - H (HASTE, method
                 section 2: frequent head labels, long tail in the sparse layer).

bf16 tensors are carried as ``uint16`` arrays holding the bf16 bit pattern.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import numpy as np

# tensor ids for the per-tensor seed streams
_T_IDX, _T_X, _T_W, _T_DY, _T_POS, _T_XH, _T_WH, _T_DYH = range(8)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the bit pattern."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor_id)])


def make_idx(n_groups: int, k: int, d: int, seed: int = 0, *, stream: int = _T_IDX) -> np.ndarray:
    """int32 [n_groups, k]: per group, k distinct uniform features of [0, d), sorted.

    A uniform k-subset is taken as the k smallest of d iid uniform keys; rows are
    produced in chunks so that the 8.6M-label pattern stays within memory.
    """
    if not (0 < k <= d):
        raise ValueError("need 0 < k <= d")
    rng = _rng(seed, stream)
    out = np.empty((n_groups, k), dtype=np.int32)
    chunk = max(1, (1 << 22) // d)
    for g0 in range(0, n_groups, chunk):
        g1 = min(n_groups, g0 + chunk)
        keys = rng.random((g1 - g0, d), dtype=np.float32)
        part = np.argpartition(keys, k - 1, axis=1)[:, :k] if k < d else np.tile(np.arange(d), (g1 - g0, 1))
        part.sort(axis=1)
        out[g0:g1] = part
    return out


def make_normal(shape, std: float, seed: int, tensor_id: int, dtype: str) -> np.ndarray:
    """N(0, std^2) in fp32, returned as fp32 or as bf16 bits (uint16)."""
    if dtype not in ("bf16", "f32"):
        raise ValueError(dtype)
    rng = _rng(seed, tensor_id)
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16 if dtype == "bf16" else np.float32)
    step = 1 << 24
    for i in range(0, n, step):   # one chunk at a time: no full-size fp32 temporaries
        j = min(n, i + step)
        v = rng.standard_normal(j - i, dtype=np.float32) * np.float32(std)
        out[i:j] = f32_to_bf16_bits(v) if dtype == "bf16" else v
    return out.reshape(shape)


def make_zipf_positives(B: int, n_ids: int, p: int, alpha: float, seed: int,
                        *, stream: int = _T_POS) -> Tuple[np.ndarray, np.ndarray]:
    """CSR (row_ptr int32 [B+1], ids int32 [B*p]) of p distinct Zipf ids per sample.

    Ids are drawn by inverse CDF of P(id) ~ (id+1)^-alpha over [0, n_ids) and
    redrawn until the row holds p distinct ids; each row is sorted ascending.
    """
    if p > n_ids:
        raise ValueError("p > n_ids")
    rng = _rng(seed, stream)
    w = np.arange(1, n_ids + 1, dtype=np.float64) ** (-float(alpha))
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    rows = []
    for _ in range(B):
        got = set()
        while len(got) < p:
            u = rng.random(p - len(got))
            for v in np.searchsorted(cdf, u, side="right"):
                got.add(int(min(v, n_ids - 1)))
        rows.append(sorted(got)[:p])
    ids = np.array(rows, dtype=np.int32).reshape(-1)
    row_ptr = (np.arange(B + 1, dtype=np.int64) * p).astype(np.int32)
    return row_ptr, ids


def split_head_tail(row_ptr: np.ndarray, ids: np.ndarray, H: int):
    """Split global ids into head CSR (ids < H) and tail CSR (ids - H)."""
    B = len(row_ptr) - 1
    hp, hi, tp, ti = [0], [], [0], []
    for b in range(B):
        r = ids[row_ptr[b]:row_ptr[b + 1]]
        h = r[r < H]
        t = r[r >= H] - H
        hi.extend(h.tolist()); ti.extend(t.tolist())
        hp.append(len(hi)); tp.append(len(ti))
    as32 = lambda v: np.array(v, dtype=np.int32)
    return (as32(hp), as32(hi)), (as32(tp), as32(ti))


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload shaped like a benchmark of the HASTE experiments."""
    name: str
    B: int
    d: int
    L: int
    G: int
    k: int
    dtype: str            # "bf16" or "f32"
    H: int = 0            # dense head labels (0: no head)
    positives: int = 0    # positives per sample (0: given-gradient workload)
    alpha: float = 1.0
    fused: bool = False   # fused BCE step (True) or forward/dW/dX with given dY

    @property
    def n_groups(self) -> int:
        return self.L // self.G


# The workloads of the HASTE evaluation (label counts of Amazon-670K, Amazon-3M and
# LF-Paper2Keywords-8.6M, section "experimental results"); synthetic stand-ins.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=32, d=256, L=4096, G=16, k=32, dtype="f32"),
    "670k": Workload("670k", B=256, d=768, L=670_208, G=32, k=128, dtype="bf16",
                     H=4096, positives=5, alpha=1.0, fused=True),
    "sweep16": Workload("sweep16", B=512, d=1024, L=1_048_576, G=16, k=128, dtype="bf16"),
    "sweep32": Workload("sweep32", B=512, d=1024, L=1_048_576, G=32, k=128, dtype="bf16"),
    "sweep64": Workload("sweep64", B=512, d=1024, L=1_048_576, G=64, k=128, dtype="bf16"),
    "3m": Workload("3m", B=256, d=768, L=3_000_000, G=64, k=64, dtype="bf16",
                   H=8192, positives=5, alpha=1.0, fused=True),
    "8.6m": Workload("8.6m", B=256, d=768, L=8_600_064, G=64, k=128, dtype="bf16",
                     H=16_384, positives=8, alpha=1.1, fused=True),
}


@dataclasses.dataclass
class Inputs:
    wl: Workload
    idx: np.ndarray
    X: np.ndarray
    W: np.ndarray
    dY: Optional[np.ndarray] = None
    tail_pos: Optional[Tuple[np.ndarray, np.ndarray]] = None
    head_pos: Optional[Tuple[np.ndarray, np.ndarray]] = None
    Xh: Optional[np.ndarray] = None
    Wh: Optional[np.ndarray] = None


def make_inputs(wl: Workload, seed: int = 0, *, with_dy: Optional[bool] = None,
                with_head: Optional[bool] = None) -> Inputs:
    """All seeded inputs of a workload (see the module docstring for the recipe)."""
    idx = make_idx(wl.n_groups, wl.k, wl.d, seed)
    X = make_normal((wl.B, wl.d), 1.0, seed, _T_X, wl.dtype)
    W = make_normal((wl.L, wl.k), 1.0 / np.sqrt(wl.k), seed, _T_W, wl.dtype)
    inp = Inputs(wl, idx, X, W)
    if with_dy is None:
        with_dy = not wl.fused
    if with_dy:
        inp.dY = make_normal((wl.B, wl.L), 1.0, seed, _T_DY, wl.dtype)
    if wl.positives:
        rp, ids = make_zipf_positives(wl.B, wl.H + wl.L, wl.positives, wl.alpha, seed)
        inp.head_pos, inp.tail_pos = split_head_tail(rp, ids, wl.H)
    if with_head is None:
        with_head = wl.H > 0
    if with_head and wl.H > 0:
        inp.Xh = make_normal((wl.B, wl.d), 1.0, seed, _T_XH, wl.dtype)
        inp.Wh = make_normal((wl.H, wl.d), 1.0 / np.sqrt(wl.d), seed, _T_WH, wl.dtype)
    return inp
