"""The allocation-free dX entry point, called through the C ABI.

haste_backward_dx_noalloc serves callers that must not allocate device memory
(code under a framework's caching allocator, hooks inside another library's call
path, loops that may not allocate): it takes no workspace and keeps its scratch
in a 16 MiB static device array owned by the library.  Its output must match
haste_backward_dx within the parity tolerance on two calls in a row (the second
call runs on the scratch contents the first one left behind), and shapes whose
scratch does not fit must be refused before any launch.
"""
import math

import numpy as np
import pytest

from structured_sparse_output_b200 import haste as H
from structured_sparse_output_b200 import inputs as I
from tests.helpers import assert_close, to_np64, to_torch

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.mark.parametrize("B,d,n_groups,G,k,dtype", [
    (256, 768, 500, 64, 128, "bf16"),
    (200, 320, 333, 32, 64, "bf16"),
    (32, 256, 256, 16, 32, "f32"),
])
def test_noalloc_dx_matches_workspace_dx_twice(B, d, n_groups, G, k, dtype):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    idx = I.make_idx(n_groups, k, d, 2)
    W = to_torch(I.make_normal((n_groups * G, k), 1.0 / math.sqrt(k), 2, 2, dtype))
    dY = to_torch(I.make_normal((B, n_groups * G), 1.0, 2, 3, dtype))
    plan = H.haste_plan(idx, G, d)
    ws = torch.empty(plan.workspace_size(B, H.dtype_code(W)), dtype=torch.uint8, device="cuda")
    ref = torch.empty((B, d), dtype=torch.float32, device="cuda")
    H.haste_backward_dx(plan, W, dY, ref, ws)
    torch.cuda.synchronize()
    ref64 = to_np64(ref)
    for call in range(2):
        out = torch.full((B, d), float("nan"), dtype=torch.float32, device="cuda")
        H.haste_backward_dx_noalloc(plan, W, dY, out)
        torch.cuda.synchronize()
        assert H.haste_device_status() == H.HASTE_OK
        assert_close(to_np64(out), ref64, f"noalloc dX, call {call + 1}")


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
