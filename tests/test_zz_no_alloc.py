"""The allocation-free dX entry point, called through the C ABI.

haste_backward_dx_noalloc serves callers that must not allocate device memory
(code under a framework's caching allocator, hooks inside another library's call
path, loops that may not allocate): it takes no workspace and keeps its scratch
in a 16 MiB static device array owned by the library.

Each case first runs a call of a different shape (more features, more group
chunks) so that the shared scratch holds nonzero partials where the checked calls
write theirs; the checked calls must not read any of them.  Then two calls in a
row must match the fp64 oracle and the workspace entry point haste_backward_dx
within the parity tolerance, a third call with accumulate = 1 must add onto the
caller's dX, and shapes whose scratch does not fit must be refused before any
launch.  This file is collected last so that a run stopping at the first failure
has already run every other test.
"""
import math

import numpy as np
import pytest

from oracle import oracle as O
from structured_sparse_output_b200 import haste as H
from structured_sparse_output_b200 import inputs as I
from tests.helpers import assert_close, to_np64, to_torch

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _inputs(B, d, n_groups, G, k, dtype, seed):
    idx = I.make_idx(n_groups, k, d, seed)
    W = I.make_normal((n_groups * G, k), 1.0 / math.sqrt(k), seed, 2, dtype)
    dY = I.make_normal((B, n_groups * G), 1.0, seed, 3, dtype)
    return idx, W, dY


def _dirty_scratch(B, dtype):
    """A call of another plan with d = 2048 and many chunks: its partials cover
    more of the scratch than any checked case's."""
    d, n_groups, G, k = 2048, 600, 32, 64 if dtype == "bf16" else 32
    idx, W, dY = _inputs(B, d, n_groups, G, k, dtype, 9)
    plan = H.haste_plan(idx, G, d)
    out = torch.empty((B, d), dtype=torch.float32, device="cuda")
    H.haste_backward_dx_noalloc(plan, to_torch(W), to_torch(dY), out)
    torch.cuda.synchronize()
    assert H.haste_device_status() == H.HASTE_OK
    assert float(out.abs().max().item()) > 0.0


@pytest.mark.parametrize("B,d,n_groups,G,k,dtype", [
    (256, 768, 500, 64, 128, "bf16"),
    (200, 320, 333, 32, 64, "bf16"),
    (32, 256, 256, 16, 32, "f32"),
])
def test_noalloc_dx_matches_oracle_and_workspace_dx(B, d, n_groups, G, k, dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    idx, W_np, dY_np = _inputs(B, d, n_groups, G, k, dtype, 2)
    r_dx = O.backward_dx(W_np, dY_np, idx, G, d)
    W, dY = to_torch(W_np), to_torch(dY_np)
    plan = H.haste_plan(idx, G, d)
    ws = torch.empty(plan.workspace_size(B, H.dtype_code(W)), dtype=torch.uint8, device="cuda")
    ref = torch.empty((B, d), dtype=torch.float32, device="cuda")
    H.haste_backward_dx(plan, W, dY, ref, ws)
    torch.cuda.synchronize()
    ref64 = to_np64(ref)
    _dirty_scratch(B, dtype)
    for call in range(2):
        out = torch.full((B, d), float("nan"), dtype=torch.float32, device="cuda")
        H.haste_backward_dx_noalloc(plan, W, dY, out)
        torch.cuda.synchronize()
        assert H.haste_device_status() == H.HASTE_OK
        got = to_np64(out)
        assert_close(got, r_dx, f"noalloc dX vs oracle, call {call + 1}")
        assert_close(got, ref64, f"noalloc dX vs haste_backward_dx, call {call + 1}")
    # accumulate = 1 adds onto what the caller's dX holds
    dX0 = I.make_normal((B, d), 1.0, 2, 7, "f32")
    out = to_torch(dX0)
    H.haste_backward_dx_noalloc(plan, W, dY, out, accumulate=True)
    torch.cuda.synchronize()
    assert H.haste_device_status() == H.HASTE_OK
    assert_close(to_np64(out), r_dx + dX0.astype(np.float64), "noalloc dX, accumulate")


def test_noalloc_dx_refuses_oversized_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    B, d, n_groups, G, k = 512, 8200, 4, 16, 64          # 8200 * 512 * 4 bytes > 16 MiB
    plan = H.haste_plan(I.make_idx(n_groups, k, d, 1), G, d)
    W = torch.zeros((n_groups * G, k), dtype=torch.bfloat16, device="cuda")
    dY = torch.zeros((B, n_groups * G), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((B, d), dtype=torch.float32, device="cuda")
    with pytest.raises(H.HasteError) as e:
        H.haste_backward_dx_noalloc(plan, W, dY, out)
    assert e.value.status == H.HASTE_ERR_UNSUPPORTED_SHAPE
    assert "16777216" in str(e.value)
