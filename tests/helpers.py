"""Test helpers: numpy <-> torch marshalling and the parity metrics.

Tolerances for floating point (fp32 accumulation on the tensor cores, bf16 or
tf32 operands): relative L2 error <= 5e-3 and elementwise max-abs relative error
<= 2e-2, the latter read as max_i |gpu_i - ref_i| / max(|ref_i|, rms(ref)).
"""
import numpy as np

REL_L2 = 5e-3
MAX_REL = 2e-2


def to_torch(a: np.ndarray, device="cuda"):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_np64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((got - ref).ravel()) / (den if den > 0 else 1.0))


def max_rel(got: np.ndarray, ref: np.ndarray) -> float:
    r = ref.ravel()
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    den = np.maximum(np.abs(r), rms if rms > 0 else 1.0)
    return float(np.max(np.abs(got.ravel() - r) / den)) if r.size else 0.0


def assert_close(got: np.ndarray, ref: np.ndarray, what: str, rel_l2_tol=REL_L2, max_rel_tol=MAX_REL):
    e1, e2 = rel_l2(got, ref), max_rel(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert e1 <= rel_l2_tol and e2 <= max_rel_tol, f"{what}: rel_l2={e1:.3e} max_rel={e2:.3e}"
    return e1, e2
