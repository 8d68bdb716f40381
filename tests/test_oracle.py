"""Pins of the fp64 oracle against what the HASTE page and plain mathematics fix.

Every check here compares the oracle with something other than itself: a dense
masked product computed by numpy, brute-force Python loops, finite differences,
closed forms, special cases that reduce to a plain dense layer, and the index
memory the page states (indices stored once per group).
Source: "HASTE: Hardware-Aware Dynamic Sparse Training for Large Output Spaces"
(summary page), Methodology 1 (structure, hardware alignment, memory efficiency)
and Methodology 2 (head-tail decomposition).
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import oracle as O
from structured_sparse_output_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(B=8, d=40, n_groups=6, G=3, k=7, seed=3, dtype="f32"):
    idx = I.make_idx(n_groups, k, d, seed)
    X = I.make_normal((B, d), 1.0, seed, 1, dtype)
    W = I.make_normal((n_groups * G, k), 1.0 / math.sqrt(k), seed, 2, dtype)
    dY = I.make_normal((B, n_groups * G), 1.0, seed, 3, dtype)
    return idx, X, W, dY


def _dense_w(W64, idx, G, d):
    """Dense [L, d] weight that is zero off each group's shared mask."""
    n_groups, k = idx.shape
    Wd = np.zeros((n_groups * G, d))
    for g in range(n_groups):
        Wd[g * G:(g + 1) * G][:, idx[g]] = W64[g * G:(g + 1) * G]
    return Wd


def _mask(idx, G, d):
    n_groups = idx.shape[0]
    m = np.zeros((n_groups * G, d), dtype=bool)
    for g in range(n_groups):
        m[g * G:(g + 1) * G, idx[g]] = True
    return m


SHAPES = [
    dict(B=8, d=40, n_groups=6, G=3, k=7),
    dict(B=5, d=17, n_groups=9, G=1, k=4),      # G = 1: standard per-label fixed fan-in
    dict(B=3, d=12, n_groups=2, G=5, k=12),     # k = d
    dict(B=33, d=64, n_groups=20, G=16, k=16),
]


# ---------------------------------------------------------------- plan
@pytest.mark.parametrize("shape", SHAPES)
def test_plan_matches_stable_argsort(shape):
    idx = I.make_idx(shape["n_groups"], shape["k"], shape["d"], 5)
    st, inv_off, inv_ent = O.plan(idx, shape["d"])
    assert st == O.OK
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")          # entries by feature, ties by e
    counts = np.bincount(flat, minlength=shape["d"])
    assert np.array_equal(inv_ent, order.astype(np.int32))
    assert np.array_equal(inv_off, np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))


def test_plan_invariants():
    n_groups, k, d = 300, 24, 97
    idx = I.make_idx(n_groups, k, d, 11)
    st, off, ent = O.plan(idx, d)
    assert st == O.OK
    assert off[0] == 0 and off[-1] == n_groups * k
    assert np.all(np.diff(off) >= 0)
    assert np.array_equal(np.sort(ent), np.arange(n_groups * k))
    flat = idx.ravel()
    for f in range(d):
        seg = ent[off[f]:off[f + 1]]
        assert np.all(flat[seg] == f)
        assert np.all(np.diff(seg // k) > 0)       # strictly ascending group


def test_plan_brute_force_tiny():
    idx = np.array([[0, 2, 5], [1, 2, 3], [0, 3, 5]], dtype=np.int32)
    st, off, ent = O.plan(idx, 7)
    assert st == O.OK
    exp_ent, exp_off = [], [0]
    for f in range(7):
        for g in range(3):
            for s in range(3):
                if idx[g, s] == f:
                    exp_ent.append(g * 3 + s)
        exp_off.append(len(exp_ent))
    assert off.tolist() == exp_off and ent.tolist() == exp_ent
    assert off.tolist() == [0, 2, 3, 5, 7, 7, 9, 9]   # feature 4 and 6 are in no group


def test_plan_validation_codes():
    good = np.array([[0, 3], [1, 2]], dtype=np.int32)
    assert O.validate(good, 4) == O.OK
    assert O.validate(np.array([[0, 4], [1, 2]], dtype=np.int32), 4) == O.ERR_RANGE
    assert O.validate(np.array([[-1, 2]], dtype=np.int32), 4) == O.ERR_RANGE
    assert O.validate(np.array([[2, 2]], dtype=np.int32), 4) == O.ERR_UNSORTED
    assert O.validate(np.array([[3, 1]], dtype=np.int32), 4) == O.ERR_UNSORTED
    # the first offending element in row-major order decides
    assert O.validate(np.array([[3, 1], [0, 9]], dtype=np.int32), 4) == O.ERR_UNSORTED
    assert O.validate(np.array([[0, 9], [3, 1]], dtype=np.int32), 4) == O.ERR_RANGE


def test_index_memory_golden():
    """Indices are stored once per group: L/G*k ints instead of L*k
    (HASTE summary page, Methodology 1, "memory efficiency")."""
    with open(os.path.join(GOLDEN, "index_memory.json")) as fh:
        gold = json.load(fh)
    for name, row in gold["workloads"].items():
        wl = I.WORKLOADS[name]
        assert O.index_bytes(wl.n_groups, wl.k) == row["group_shared_bytes"]
        assert row["per_label_bytes"] == 4 * wl.L * wl.k
        assert row["per_label_bytes"] == wl.G * row["group_shared_bytes"]


# ------------------------------------------------------------- forward
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_equals_dense_masked(shape, dtype):
    idx, X, W, _ = _case(**shape, dtype=dtype)
    G, d = shape["G"], shape["d"]
    ref = O.to_f64(X) @ _dense_w(O.to_f64(W), idx, G, d).T
    got = O.forward(X, W, idx, G)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_forward_brute_force_bitwise():
    idx, X, W, _ = _case(B=3, d=10, n_groups=2, G=2, k=4)
    Xf, Wf = O.to_f64(X), O.to_f64(W)
    got = O.forward(X, W, idx, 2)
    for b in range(3):
        for g in range(2):
            for j in range(2):
                acc = 0.0
                for s in range(4):
                    acc += Xf[b, idx[g, s]] * Wf[g * 2 + j, s]
                assert got[b, g * 2 + j] == acc


def test_forward_k_equals_d_is_dense_layer():
    B, d, n_groups, G = 6, 9, 4, 3
    idx = np.tile(np.arange(d, dtype=np.int32), (n_groups, 1))
    X = I.make_normal((B, d), 1.0, 0, 1, "f32")
    W = I.make_normal((n_groups * G, d), 1.0, 0, 2, "f32")
    np.testing.assert_allclose(O.forward(X, W, idx, G), O.to_f64(X) @ O.to_f64(W).T,
                               rtol=1e-13, atol=1e-13)


def test_forward_linearity_and_group_permutation():
    idx, X, W, _ = _case(B=4, d=30, n_groups=5, G=2, k=6)
    X2 = I.make_normal(X.shape, 1.0, 9, 1, "f32")
    a, b = 0.75, -1.5
    lin = O.forward(a * X.astype(np.float64) + b * X2.astype(np.float64), W, idx, 2)
    np.testing.assert_allclose(lin, a * O.forward(X, W, idx, 2) + b * O.forward(X2, W, idx, 2),
                               rtol=1e-12, atol=1e-12)
    perm = np.array([3, 0, 4, 1, 2])
    lperm = np.concatenate([np.arange(g * 2, g * 2 + 2) for g in perm])
    got = O.forward(X, W[lperm], idx[perm], 2)
    np.testing.assert_array_equal(got, O.forward(X, W, idx, 2)[:, lperm])


# ------------------------------------------------------------------ dW, dX
@pytest.mark.parametrize("shape", SHAPES)
def test_dw_equals_masked_dense_gradient(shape):
    idx, X, W, dY = _case(**shape)
    G, d = shape["G"], shape["d"]
    dW = O.backward_dw(X, dY, idx, G)
    dense = O.to_f64(dY).T @ O.to_f64(X)                   # [L, d]
    m = _mask(idx, G, d)
    scattered = np.zeros_like(dense)
    for g in range(idx.shape[0]):
        scattered[g * G:(g + 1) * G][:, idx[g]] = dW[g * G:(g + 1) * G]
    np.testing.assert_allclose(scattered, dense * m, rtol=1e-12, atol=1e-12)
    assert np.all(scattered[~m] == 0.0)                      # exactly zero off-mask


@pytest.mark.parametrize("shape", SHAPES)
def test_dx_equals_dense_product(shape):
    idx, X, W, dY = _case(**shape)
    G, d = shape["G"], shape["d"]
    dX = O.backward_dx(W, dY, idx, G, d)
    ref = O.to_f64(dY) @ _dense_w(O.to_f64(W), idx, G, d)
    np.testing.assert_allclose(dX, ref, rtol=1e-12, atol=1e-12)
    covered = np.zeros(d, dtype=bool)
    covered[np.unique(idx)] = True
    assert np.all(dX[:, ~covered] == 0.0)                    # features in no group


def test_dx_dw_are_adjoints_of_forward():
    """<dY, forward(X, W)> = <dX, X> = <dW, W> (the layer is bilinear)."""
    idx, X, W, dY = _case(B=7, d=50, n_groups=8, G=4, k=9)
    z = O.forward(X, W, idx, 4)
    lhs = float(np.sum(O.to_f64(dY) * z))
    dX = O.backward_dx(W, dY, idx, 4, 50)
    dW = O.backward_dw(X, dY, idx, 4)
    assert math.isclose(lhs, float(np.sum(dX * O.to_f64(X))), rel_tol=1e-12)
    assert math.isclose(lhs, float(np.sum(dW * O.to_f64(W))), rel_tol=1e-12)


# ----------------------------------------------------------------- BCE
def test_bce_at_zero_logits_closed_form():
    B, L = 4, 10
    rp = np.array([0, 1, 3, 3, 4], dtype=np.int32)
    ids = np.array([2, 0, 9, 5], dtype=np.int32)
    loss, dY = O.bce(np.zeros((B, L)), rp, ids, 0.25)
    assert math.isclose(loss, 0.25 * B * L * math.log(2.0), rel_tol=1e-15)
    y = np.zeros((B, L))
    for b in range(B):
        y[b, ids[rp[b]:rp[b + 1]]] = 1.0
    np.testing.assert_array_equal(dY, 0.25 * (0.5 - y))


def test_bce_against_logaddexp():
    rng = np.random.default_rng(7)
    z = rng.normal(0, 8, size=(6, 50))                      # includes large |z|
    rp = np.array([0, 2, 2, 5, 6, 8, 9], dtype=np.int32)
    ids = np.array([3, 40, 0, 1, 49, 7, 20, 21, 10], dtype=np.int32)
    y = np.zeros_like(z)
    for b in range(6):
        y[b, ids[rp[b]:rp[b + 1]]] = 1.0
    loss, dY = O.bce(z, rp, ids, 1.0 / 6)
    ref_loss = np.sum(np.logaddexp(0.0, z) - z * y) / 6
    assert math.isclose(loss, ref_loss, rel_tol=1e-13)
    np.testing.assert_allclose(dY, (0.5 * (1 + np.tanh(z / 2)) - y) / 6, rtol=1e-12, atol=1e-15)


def test_bce_step_finite_differences():
    """Central differences of the oracle's loss in fp64 match dW and dX."""
    B, d, n_groups, G, k = 5, 30, 6, 4, 8
    idx = I.make_idx(n_groups, k, d, 2)
    X = I.make_normal((B, d), 1.0, 2, 1, "f32").astype(np.float64)
    W = I.make_normal((n_groups * G, k), 0.5, 2, 2, "f32").astype(np.float64)
    rp, ids = I.make_zipf_positives(B, n_groups * G, 3, 1.0, 2)
    scale = 1.0 / B
    loss, _, dW, dX = O.bce_step(X, W, idx, G, rp, ids, scale)
    h = 1e-6

    def L(Xv, Wv):
        return O.bce(O.forward(Xv, Wv, idx, G), rp, ids, scale, want_grad=False)[0]

    rng = np.random.default_rng(0)
    for _ in range(12):
        l, s = rng.integers(n_groups * G), rng.integers(k)
        Wp, Wm = W.copy(), W.copy()
        Wp[l, s] += h
        Wm[l, s] -= h
        fd = (L(X, Wp) - L(X, Wm)) / (2 * h)
        assert abs(fd - dW[l, s]) <= 1e-6 * max(1.0, abs(dW[l, s])) + 1e-9
        b, f = rng.integers(B), rng.choice(np.unique(idx))
        Xp, Xm = X.copy(), X.copy()
        Xp[b, f] += h
        Xm[b, f] -= h
        fd = (L(Xp, W) - L(Xm, W)) / (2 * h)
        assert abs(fd - dX[b, f]) <= 1e-6 * max(1.0, abs(dX[b, f])) + 1e-9


# ------------------------------------------------------- sampled evaluations
def test_sampled_evaluations_match_full():
    B, d, n_groups, G, k = 6, 40, 10, 4, 8
    idx = I.make_idx(n_groups, k, d, 4)
    X = I.make_normal((B, d), 1.0, 4, 1, "bf16")
    W = I.make_normal((n_groups * G, k), 0.4, 4, 2, "bf16")
    dY = I.make_normal((B, n_groups * G), 1.0, 4, 3, "bf16")
    rp, ids = I.make_zipf_positives(B, n_groups * G, 3, 1.0, 4)
    rng = np.random.default_rng(1)
    bs = rng.integers(0, B, 20).astype(np.int32)
    ls = rng.integers(0, n_groups * G, 20)
    ss = rng.integers(0, k, 20).astype(np.int32)
    fs = idx.ravel()[rng.integers(0, idx.size, 20)].astype(np.int32)
    z = O.forward(X, W, idx, G)
    np.testing.assert_array_equal(O.logits_at(X, W, idx, G, bs, ls), z[bs, ls])
    dW = O.backward_dw(X, dY, idx, G)
    np.testing.assert_allclose(O.dw_at(X, W, idx, G, ls, ss, dY=dY), dW[ls, ss], rtol=1e-13, atol=1e-13)
    dX = O.backward_dx(W, dY, idx, G, d)
    np.testing.assert_allclose(O.dx_at(X, W, idx, G, bs, fs, dY=dY), dX[bs, fs], rtol=1e-12, atol=1e-12)
    _, _, dWf, dXf = O.bce_step(X, W, idx, G, rp, ids, 1.0 / B)
    np.testing.assert_allclose(O.dw_at(X, W, idx, G, ls, ss, pos=(rp, ids), scale=1.0 / B),
                               dWf[ls, ss], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(O.dx_at(X, W, idx, G, bs, fs, pos=(rp, ids), scale=1.0 / B),
                               dXf[bs, fs], rtol=1e-12, atol=1e-14)


def test_bce_loss_alone_matches_the_pinned_step_and_closed_forms():
    """The loss-only evaluation (no B x L logits kept) against numpy logaddexp of a
    numpy masked-dense forward, for f32 and bf16 inputs; W = 0 gives n * ln 2."""
    B, d, n_groups, G, k = 7, 48, 9, 4, 8
    for dt in ("f32", "bf16"):
        idx = I.make_idx(n_groups, k, d, 6)
        X = I.make_normal((B, d), 1.0, 6, 1, dt)
        W = I.make_normal((n_groups * G, k), 0.7, 6, 2, dt)
        rp, ids = I.make_zipf_positives(B, n_groups * G, 3, 1.0, 6)
        z = O.to_f64(X) @ _dense_w(O.to_f64(W), idx, G, d).T
        y = np.zeros_like(z)
        for b in range(B):
            y[b, ids[rp[b]:rp[b + 1]]] = 1.0
        ref = float(np.sum(np.logaddexp(0.0, z) - z * y)) / B
        assert math.isclose(O.bce_loss(X, W, idx, G, rp, ids, 1.0 / B), ref, rel_tol=1e-12)
        assert math.isclose(O.bce_loss(X, W, idx, G, rp, ids, 1.0 / B),
                            O.bce_step(X, W, idx, G, rp, ids, 1.0 / B)[0], rel_tol=1e-13)
    W0 = np.zeros((n_groups * G, k), dtype=np.float32)
    X = I.make_normal((B, d), 1.0, 6, 1, "f32")
    got = O.bce_loss(X, W0, I.make_idx(n_groups, k, d, 6), G, rp, ids, 0.5)
    assert math.isclose(got, 0.5 * B * n_groups * G * math.log(2.0), rel_tol=1e-14)


# ------------------------------------------------------- optimizer update
def test_sgd_update_matches_torch_sgd_over_three_steps():
    """The update equals torch.optim.SGD (momentum, no dampening, no Nesterov) on
    the same gradients, step after step (the momentum buffer starts at zero)."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    W = rng.normal(size=(12, 8))
    grads = [rng.normal(size=(12, 8)) for _ in range(3)]
    for lr, mu in ((0.1, 0.9), (0.5, 0.0), (0.03, 0.5)):
        p = torch.nn.Parameter(torch.tensor(W, dtype=torch.float64))
        opt = torch.optim.SGD([p], lr=lr, momentum=mu)
        Wo, Mo = W.copy(), np.zeros_like(W)
        for g in grads:
            p.grad = torch.tensor(g, dtype=torch.float64)
            opt.step()
            Wo, Mo = O.sgd_update(Wo, Mo if mu else None, g, lr, mu)
        np.testing.assert_allclose(Wo, p.detach().numpy(), rtol=1e-13, atol=1e-15)


def test_sgd_update_special_cases():
    rng = np.random.default_rng(4)
    W, M, g = rng.normal(size=(5, 4)), rng.normal(size=(5, 4)), rng.normal(size=(5, 4))
    W1, M1 = O.sgd_update(W, M, g, 0.0, 0.7)           # lr = 0: weights unchanged
    assert np.array_equal(W1, W) and np.allclose(M1, 0.7 * M + g, rtol=0, atol=1e-15)
    W2, M2 = O.sgd_update(W, None, g, 0.25, 0.0)       # no momentum: W - lr g
    assert np.array_equal(M2, g) and np.allclose(W2, W - 0.25 * g, rtol=0, atol=1e-15)
    Wb = I.make_normal((5, 4), 1.0, 4, 2, "bf16")       # bf16 bits widen exactly
    W3, _ = O.sgd_update(Wb, None, np.zeros((5, 4)), 3.0, 0.0)
    assert np.array_equal(W3, O.to_f64(Wb))


def test_fused_step_with_update_is_step_then_update():
    """dX uses the weights before the update; W' follows from the step's dW."""
    B, d, n_groups, G, k = 6, 40, 7, 4, 8
    idx = I.make_idx(n_groups, k, d, 8)
    X = I.make_normal((B, d), 1.0, 8, 1, "f32")
    W = I.make_normal((n_groups * G, k), 0.5, 8, 2, "f32")
    M = I.make_normal((n_groups * G, k), 0.1, 8, 4, "f32")
    rp, ids = I.make_zipf_positives(B, n_groups * G, 3, 1.0, 8)
    loss, dX, W1, M1 = O.bce_step_sgd(X, W, M, idx, G, rp, ids, 1.0 / B, 0.2, 0.9)
    r_loss, _, dW, r_dX = O.bce_step(X, W, idx, G, rp, ids, 1.0 / B)
    assert loss == r_loss and np.array_equal(dX, r_dX)
    np.testing.assert_allclose(M1, 0.9 * M.astype(np.float64) + dW, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(W1, W.astype(np.float64) - 0.2 * M1, rtol=1e-14, atol=1e-15)


# ------------------------------------------------------------------- head
def test_head_is_the_dense_special_case_of_the_sparse_layer():
    """A dense head over H labels is one group of G = H labels with k = d."""
    B, d, H = 5, 12, 7
    Xh = I.make_normal((B, d), 1.0, 6, 5, "bf16")
    Wh = I.make_normal((H, d), 0.3, 6, 6, "bf16")
    idx = np.arange(d, dtype=np.int32)[None, :]
    np.testing.assert_allclose(O.head_forward(Xh, Wh), O.forward(Xh, Wh, idx, H), rtol=1e-13, atol=1e-13)
    dYh = I.make_normal((B, H), 1.0, 6, 7, "f32").astype(np.float64)
    dWh, dXh = O.head_backward(Xh, Wh, dYh)
    np.testing.assert_allclose(dWh, O.backward_dw(Xh, dYh, idx, H), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dXh, O.backward_dx(Wh, dYh, idx, H, d), rtol=1e-12, atol=1e-13)


def test_head_forward_brute_force():
    Xh = I.make_normal((3, 5), 1.0, 8, 5, "f32")
    Wh = I.make_normal((4, 5), 1.0, 8, 6, "f32")
    z = O.head_forward(Xh, Wh)
    for b in range(3):
        for h in range(4):
            ref = sum(float(Xh[b, i]) * float(Wh[h, i]) for i in range(5))
            assert math.isclose(z[b, h], ref, rel_tol=1e-14, abs_tol=1e-14)


def test_head_step_finite_differences():
    B, d, H = 4, 6, 5
    Xh = I.make_normal((B, d), 1.0, 9, 5, "f32").astype(np.float64)
    Wh = I.make_normal((H, d), 0.5, 9, 6, "f32").astype(np.float64)
    rp = np.array([0, 1, 1, 3, 4], dtype=np.int32)
    ids = np.array([0, 1, 4, 2], dtype=np.int32)
    loss, dY, dWh, dXh = O.head_step(Xh, Wh, rp, ids, 1.0 / B)
    h = 1e-6

    def L(Xv, Wv):
        return O.bce(O.head_forward(Xv, Wv), rp, ids, 1.0 / B, want_grad=False)[0]

    for (r, c) in [(0, 0), (2, 3), (4, 5)]:
        Wp, Wm = Wh.copy(), Wh.copy()
        Wp[r, c] += h
        Wm[r, c] -= h
        assert abs((L(Xh, Wp) - L(Xh, Wm)) / (2 * h) - dWh[r, c]) < 1e-8
    for (r, c) in [(0, 1), (3, 5)]:
        Xp, Xm = Xh.copy(), Xh.copy()
        Xp[r, c] += h
        Xm[r, c] -= h
        assert abs((L(Xp, Wh) - L(Xm, Wh)) / (2 * h) - dXh[r, c]) < 1e-8


# ------------------------------------------------------------ input recipe
def test_input_generator_recipe():
    idx = I.make_idx(1000, 128, 768, 0)
    assert idx.dtype == np.int32 and idx.min() >= 0 and idx.max() < 768
    assert np.all(np.diff(idx, axis=1) > 0)
    # uniform: every feature is chosen by about n_groups*k/d groups
    cnt = np.bincount(idx.ravel(), minlength=768)
    assert abs(cnt.mean() - 1000 * 128 / 768) < 1e-9 and cnt.min() > 100
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], dtype=np.float32)
    bits = I.f32_to_bf16_bits(x)
    back = I.bf16_bits_to_f32(bits)
    np.testing.assert_array_equal(back, np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5, 0.0], dtype=np.float32))
    rp, ids = I.make_zipf_positives(64, 1000, 5, 1.0, 0)
    assert np.all(np.diff(rp) == 5)
    for b in range(64):
        r = ids[rp[b]:rp[b + 1]]
        assert np.all(np.diff(r) > 0) and r.min() >= 0 and r.max() < 1000
    (hp, hi), (tp, ti) = I.split_head_tail(rp, ids, 100)
    assert hp[-1] + tp[-1] == len(ids) and (hi < 100).all() and (ti >= 0).all()


# ------------------------------------------------------- two-stage top-k scoring
# "A Faster Generalized Two-Stage Approximate Top-K" (summary page), Methodology:
# stage 1 keeps the top K' of each bucket, stage 2 the top K of the survivors.
def _exact_topk(z, K):
    """Top K of each row by (larger value, smaller id): a full lexicographic sort."""
    out_v, out_i = [], []
    for row in z:
        order = np.lexsort((np.arange(len(row)), -row))[:K]
        out_v.append(row[order])
        out_i.append(order)
    return np.array(out_v), np.array(out_i)


def _topk_case(seed=0, B=6, d=64, n_groups=40, G=16, k=8):
    idx = I.make_idx(n_groups, k, d, seed)
    X = I.make_normal((B, d), 1.0, seed, 1, "f32")
    W = I.make_normal((n_groups * G, k), 1.0 / math.sqrt(k), seed, 2, "f32")
    return idx, X, W, O.forward(X, W, idx, G)


@pytest.mark.parametrize("K,nb", [(1, 1), (5, 7), (8, 40), (3, 13)])
def test_topk_with_kp_equal_k_is_the_exact_top_k(K, nb):
    idx, X, W, z = _topk_case()
    v, i = O.topk(X, W, idx, 16, K, K, nb)
    ev, ei = _exact_topk(z, K)
    assert np.array_equal(i, ei) and np.allclose(v, ev, rtol=0, atol=1e-12)


def test_topk_one_per_group_brute_force():
    # nb = n_groups and K' = 1: the survivors are the group maxima
    idx, X, W, z = _topk_case(seed=3)
    G, K, n_groups = 16, 6, 40
    v, i = O.topk(X, W, idx, G, K, 1, n_groups)
    for r in range(z.shape[0]):
        cand = []
        for g in range(n_groups):
            seg = z[r, g * G:(g + 1) * G]
            j = int(np.lexsort((np.arange(G), -seg))[0])
            cand.append((-seg[j], g * G + j))
        best = sorted(cand)[:K]
        assert [c[1] for c in best] == list(i[r]) and np.allclose([-c[0] for c in best], v[r], atol=1e-12)


def test_topk_recall_grows_with_kp_and_survivors_are_true_scores():
    idx, X, W, z = _topk_case(seed=5, B=8, n_groups=64)
    K, nb = 8, 4
    ev, ei = _exact_topk(z, K)
    prev = -1.0
    for Kp in (1, 2, 4, 8):
        v, i = O.topk(X, W, idx, 16, K, Kp, nb, rows=np.arange(8))
        # every returned entry is a real (label, logit) pair, ids distinct, ranked
        for r in range(8):
            ok = i[r] < 2**62
            assert np.allclose(v[r][ok], z[r, i[r][ok]], atol=1e-12)
            assert len(set(i[r][ok].tolist())) == ok.sum()
            assert np.all(np.diff(v[r][ok]) <= 0)
        recall = np.mean([len(set(i[r].tolist()) & set(ei[r].tolist())) / K for r in range(8)])
        assert recall >= prev
        prev = recall
    assert prev == 1.0


def test_topk_bucket_partition_planted_logits():
    """Buckets that do not divide the groups evenly, and K' < K.  97 groups in 13
    buckets: bucket j = groups [floor(97 j / 13), floor(97 (j+1) / 13)), boundaries
    0 7 14 22 29 37 44 52 59 67 74 82 89 97.  X is all ones and W[l, 0] = v[l] with
    the other slots 0, so logit(l) = v[l]: a baseline -1 - l/1000 plus planted
    values.  Expected answers are derived by hand from the bucket boundaries; a
    partition with boundaries 7j, a ceil-based one, or one that loses the last
    groups each drops a different planted label."""
    n_groups, G, k, d, nb, K, Kp = 97, 4, 2, 8, 13, 5, 2
    L = n_groups * G
    idx = np.tile(np.array([0, 5], dtype=np.int32), (n_groups, 1))
    v = -1.0 - np.arange(L) / 1000.0
    planted = {85: 10.0, 87: 9.0,   # group 21, last group of bucket 2 = [14, 22)
               88: 8.0,             # group 22, first group of bucket 3
               386: 7.0,            # group 96, last group of the last bucket
               0: 6.0,              # group 0
               58: 5.0}             # group 14, first group of bucket 2: third best there, dropped
    for l, val in planted.items():
        v[l] = val
    W = np.zeros((L, k), dtype=np.float64)
    W[:, 0] = v
    X = np.stack([np.ones(d), -np.ones(d)])
    vals, ids = O.topk(X, W, idx, G, K, Kp, nb)
    # row 0: bucket 2 keeps 10 and 9 (5 is its third), bucket 3 keeps 8, the last
    # bucket 7, bucket 0 keeps 6
    assert ids[0].tolist() == [85, 87, 88, 386, 0]
    assert vals[0].tolist() == [10.0, 9.0, 8.0, 7.0, 6.0]
    # row 1: logits -v, so larger labels rank first (the planted ones are now far
    # below).  Each bucket passes its two largest labels: the last bucket
    # (labels 356..387, 386 planted) passes 387 and 385, bucket 11 (labels
    # 328..355) passes 355 and 354, bucket 10 (labels 296..327) passes 327.
    assert ids[1].tolist() == [387, 385, 355, 354, 327]
    np.testing.assert_allclose(vals[1], 1.0 + np.array([387, 385, 355, 354, 327]) / 1000.0, rtol=0, atol=1e-15)
