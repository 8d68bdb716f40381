"""The C ABI without a GPU: the library loads, exports every function that
include/haste.h declares, and its host plan builder is bit-exact against the
oracle's independent inverse-map construction (HASTE summary page,
Methodology 1: one fan-in index set per group, stored once per group)."""
import os
import re

import numpy as np
import pytest

from oracle import oracle as O
from structured_sparse_output_b200 import haste as H
from structured_sparse_output_b200 import inputs as I


def _declared():
    text = open(H.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(haste_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 16
    lib = H.lib()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.haste_abi_version() == 1


@pytest.mark.parametrize("n_groups,k,d", [(256, 32, 256), (20_944, 128, 768), (1000, 64, 97), (3, 5, 5)])
def test_host_plan_bit_exact_vs_oracle(n_groups, k, d):
    idx = I.make_idx(n_groups, k, d, 7)
    off, ent = H.haste_plan_inverse_host(idx, d)
    st, ref_off, ref_ent = O.plan(idx, d)
    assert st == O.OK
    assert np.array_equal(off, ref_off) and np.array_equal(ent, ref_ent)


def test_host_plan_error_codes_match_oracle():
    cases = [
        (np.array([[0, 4], [1, 2]], dtype=np.int32), 4),
        (np.array([[2, 2]], dtype=np.int32), 4),
        (np.array([[3, 1], [0, 9]], dtype=np.int32), 4),
        (np.array([[0, 9], [3, 1]], dtype=np.int32), 4),
        (np.array([[-5, 1]], dtype=np.int32), 4),
    ]
    big = I.make_idx(5000, 16, 64, 1)
    big[4321, 7] = big[4321, 6]          # a duplicate deep inside, on another thread's range
    cases.append((big, 64))
    for idx, d in cases:
        ref = O.validate(idx, d)
        assert ref != O.OK
        with pytest.raises(H.HasteError) as ei:
            H.haste_plan_inverse_host(idx, d)
        assert ei.value.status == ref


def test_head_workspace_size_is_host_only():
    assert H.haste_head_workspace_size(256, 4096, 768, H.HASTE_BF16) > 0
    assert H.haste_head_workspace_size(0, 4096, 768, H.HASTE_BF16) == 0


def test_calls_fail_cleanly_without_gpu():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = H.lib().haste_head_forward(256, 256, 256, H.HASTE_BF16, None, None, None, None, 1.0, None, None, 0, None)
    assert st == H.HASTE_ERR_CUDA
    assert H.lib().haste_last_error()


def test_binding_rejects_host_tensors():
    """A host tensor's pointer never reaches a kernel: the binding refuses it."""
    torch = pytest.importorskip("torch")
    with pytest.raises(ValueError, match="CUDA tensors"):
        H._tptr(torch.zeros(8))
    assert H._tptr(None) is None


def _fake_plan(device=0):
    """Shape fields of a plan without a library handle (no GPU needed): 4 groups of
    G = 16 labels, k = 64, d = 128, on CUDA device `device`."""
    return H.Plan(None, 4, 16, 64, 128, device)


def test_binding_checks_shapes_dtypes_and_devices_before_any_pointer():
    """Wrong shapes, dtypes or devices never reach the library: every case raises
    ValueError in the binding (these run without a GPU and without a plan handle)."""
    torch = pytest.importorskip("torch")
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    p = _fake_plan()
    B, L, k, d = 8, 64, 64, 128
    X, W = torch.zeros(B, d, dtype=bf), torch.zeros(L, k, dtype=bf)
    cases = [
        (lambda: H.haste_forward(p, X, torch.zeros(L, k + 1, dtype=bf), torch.zeros(B, L, dtype=bf), None), "shape"),
        (lambda: H.haste_forward(p, torch.zeros(B, d + 8, dtype=bf), W, torch.zeros(B, L, dtype=bf), None), "shape"),
        (lambda: H.haste_forward(p, X, W, torch.zeros(B, L, dtype=f32), None), "dtype"),
        (lambda: H.haste_backward_dw(p, X, torch.zeros(B, L + 16, dtype=bf), torch.zeros(L, k, dtype=bf), None),
         "shape"),
        (lambda: H.haste_backward_dx(p, W, torch.zeros(B, L, dtype=f32), torch.zeros(B, d), None), "dtype"),
        (lambda: H.haste_backward_dx(p, W, torch.zeros(B, L, dtype=bf), torch.zeros(B, d, dtype=bf), None), "dtype"),
        (lambda: H.haste_backward_dx_noalloc(p, W, torch.zeros(B, L, dtype=bf), torch.zeros(B, d + 1)), "shape"),
        (lambda: H.haste_bce_step(p, X, W, torch.zeros(B, dtype=i32), torch.zeros(3, dtype=i32), 0.1, None,
                                  torch.zeros(L, k, dtype=bf), torch.zeros(B, d), None), "row_ptr"),
        (lambda: H.haste_bce_step(p, X, W, torch.zeros(B + 1, dtype=i32), torch.zeros(3, dtype=torch.int64), 0.1,
                                  None, torch.zeros(L, k, dtype=bf), torch.zeros(B, d), None), "ids"),
        (lambda: H.haste_topk(p, X, W, 5, 4, 2, torch.zeros(B, 4), torch.zeros(B, 5, dtype=i32), None), "shape"),
        (lambda: H.haste_head_forward(X, torch.zeros(16, d + 8, dtype=bf), torch.zeros(B, 16, dtype=bf), None),
         "shape"),
        (lambda: H.haste_head_backward(X, torch.zeros(16, d, dtype=bf), torch.zeros(B, 16, dtype=bf),
                                       torch.zeros(16, d, dtype=bf), torch.zeros(B, d, dtype=bf), None), "dtype"),
        # right shapes, host tensors
        (lambda: H.haste_forward(p, X, W, torch.zeros(B, L, dtype=bf), None), "CUDA"),
        (lambda: H.haste_head_backward(X, torch.zeros(16, d, dtype=bf), torch.zeros(B, 16, dtype=bf),
                                       torch.zeros(16, d, dtype=bf), torch.zeros(B, d), None), "CUDA"),
    ]
    for i, (call, what) in enumerate(cases):
        with pytest.raises(ValueError, match=what):
            call()


def test_binding_refuses_tensors_off_the_plans_device():
    """A plan lives on one device: tensors elsewhere are refused by name."""
    torch = pytest.importorskip("torch")
    p = _fake_plan(device=1)
    X, W = torch.zeros(8, 128, dtype=torch.bfloat16), torch.zeros(64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="X is on cpu"):
        H.haste_forward(p, X, W, torch.zeros(8, 64, dtype=torch.bfloat16), None)
