"""GPU parity of the C-ABI path against the fp64 oracle (B200, sm_100a).

Every call goes through libhaste.so; inputs come from the seeded generator and are
fed to both sides bit-identically.  Floating-point tolerance: relative L2 <= 5e-3
and elementwise max-abs relative error <= 2e-2 (helpers.assert_close); the plan
is bit-exact.  Shapes span several tiles with ragged tails (batch not a multiple
of 128, feature bands cut short, group counts not a multiple of the grid).
Source: "HASTE: Hardware-Aware Dynamic Sparse Training for Large Output Spaces"
(summary page), Methodology 1 and 2.
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


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    H.lib()
    yield
    torch.cuda.synchronize()
    assert H.haste_device_status() == H.HASTE_OK


def _inputs(B, d, n_groups, G, k, dtype, seed=0):
    idx = I.make_idx(n_groups, k, d, seed)
    X = I.make_normal((B, d), 1.0, seed, 1, dtype)
    W = I.make_normal((n_groups * G, k), 1.0 / math.sqrt(k), seed, 2, dtype)
    dY = I.make_normal((B, n_groups * G), 1.0, seed, 3, dtype)
    return idx, X, W, dY


def _ws(plan, B, dtype_code):
    n = plan.workspace_size(B, dtype_code)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


TAIL_CASES = [
    dict(B=32, d=256, n_groups=256, G=16, k=32, dtype="f32"),       # the tiny workload
    dict(B=130, d=200, n_groups=100, G=32, k=64, dtype="f32"),
    dict(B=200, d=320, n_groups=333, G=32, k=64, dtype="bf16"),
    dict(B=256, d=768, n_groups=500, G=64, k=128, dtype="bf16"),
    dict(B=512, d=1024, n_groups=256, G=16, k=128, dtype="bf16"),
    dict(B=128, d=512, n_groups=64, G=128, k=64, dtype="bf16"),
    dict(B=64, d=96, n_groups=40, G=48, k=64, dtype="bf16"),
    # dX band kernel: one 128-row batch tile, G = 16 (32-byte rows), one band of 208 cut to 200 features
    dict(B=100, d=200, n_groups=150, G=16, k=64, dtype="bf16"),
    # fewer groups than group chunks: one group per CTA, one batch tile
    dict(B=64, d=768, n_groups=5, G=32, k=128, dtype="bf16"),
    # three batch tiles (k = 64: padded M = 128 dW product), and a ragged third tile of one row
    dict(B=384, d=768, n_groups=300, G=64, k=64, dtype="bf16"),
    dict(B=257, d=1024, n_groups=129, G=32, k=128, dtype="bf16"),
    # four bands, the last one 232 features wide
    dict(B=256, d=1000, n_groups=97, G=16, k=128, dtype="bf16"),
    # degenerate counts: a batch of one row; a single group (one chunk, one CTA per band)
    dict(B=1, d=256, n_groups=50, G=32, k=64, dtype="bf16"),
    dict(B=37, d=256, n_groups=1, G=32, k=64, dtype="bf16"),
]


def _case_id(c):
    return "B{B}_d{d}_n{n_groups}_G{G}_k{k}_{dtype}".format(**c)


@pytest.mark.parametrize("case", TAIL_CASES, ids=_case_id)
def test_tail_forward_dw_dx(case):
    B, d, n_groups, G, k, dt = (case[x] for x in ("B", "d", "n_groups", "G", "k", "dtype"))
    idx, X, W, dY = _inputs(B, d, n_groups, G, k, dt)
    plan = H.haste_plan(idx, G, d)
    Xt, Wt, dYt = to_torch(X), to_torch(W), to_torch(dY)
    code = H.dtype_code(Xt)
    ws = _ws(plan, B, code)
    L = n_groups * G
    logits = torch.empty((B, L), dtype=Xt.dtype, device="cuda")
    H.haste_forward(plan, Xt, Wt, logits, ws)
    dW = torch.empty((L, k), dtype=Xt.dtype, device="cuda")
    H.haste_backward_dw(plan, Xt, dYt, dW, ws)
    dX = torch.full((B, d), float("nan"), dtype=torch.float32, device="cuda")
    H.haste_backward_dx(plan, Wt, dYt, dX, ws)
    torch.cuda.synchronize()
    assert H.haste_device_status() == H.HASTE_OK
    assert_close(to_np64(logits), O.forward(X, W, idx, G), "logits")
    assert_close(to_np64(dW), O.backward_dw(X, dY, idx, G), "dW")
    ref_dx = O.backward_dx(W, dY, idx, G, d)
    got_dx = to_np64(dX)
    assert_close(got_dx, ref_dx, "dX")
    uncovered = np.setdiff1d(np.arange(d), np.unique(idx))
    assert np.all(got_dx[:, uncovered] == 0.0)
    # accumulate = 1 adds into the existing dX
    H.haste_backward_dx(plan, Wt, dYt, dX, ws, accumulate=True)
    torch.cuda.synchronize()
    assert_close(to_np64(dX), 2 * ref_dx, "dX accumulated")


def test_plan_export_bit_exact_and_index_memory():
    for (n_groups, k, d, G) in [(256, 32, 256, 16), (20_944, 128, 768, 32)]:
        idx = I.make_idx(n_groups, k, d, 3)
        plan = H.haste_plan(idx, G, d)
        e_idx, off, ent = plan.export()
        st, r_off, r_ent = O.plan(idx, d)
        assert np.array_equal(e_idx, idx)
        assert np.array_equal(off, r_off) and np.array_equal(ent, r_ent)
        ib, invb = plan.info()
        assert ib == O.index_bytes(n_groups, k) == 4 * n_groups * k
        assert ib * G == 4 * n_groups * G * k           # per-label storage would be G times larger
        assert invb == 4 * (d + 1 + n_groups * k)


STEP_CASES = [
    dict(B=130, d=384, n_groups=250, G=32, k=64, dtype="bf16", H=64, p=5),
    dict(B=256, d=768, n_groups=300, G=64, k=128, dtype="bf16", H=128, p=8),
    dict(B=32, d=256, n_groups=256, G=16, k=32, dtype="f32", H=32, p=5),
    dict(B=300, d=512, n_groups=200, G=16, k=64, dtype="bf16", H=0, p=6),
    dict(B=100, d=256, n_groups=120, G=16, k=64, dtype="bf16", H=0, p=5),   # one batch tile, G = 16
    dict(B=1, d=256, n_groups=40, G=32, k=64, dtype="bf16", H=16, p=3),     # a batch of one row
    dict(B=37, d=256, n_groups=1, G=32, k=64, dtype="bf16", H=0, p=2),      # a single group
    dict(B=200, d=384, n_groups=301, G=16, k=128, dtype="bf16", H=0, p=6),  # CTA pairs, G = 16
    dict(B=256, d=512, n_groups=5, G=32, k=128, dtype="bf16", H=0, p=4),    # fewer groups than CTA pairs
    dict(B=200, d=512, n_groups=151, G=64, k=64, dtype="bf16", H=0, p=6),   # G = 64, k = 64, ragged batch
    dict(B=90, d=384, n_groups=3, G=64, k=128, dtype="bf16", H=0, p=3),     # G = 64, fewer groups than SMs
]


def _step_inputs(c, seed=0):
    B, d, n_groups, G, k, dt = (c[x] for x in ("B", "d", "n_groups", "G", "k", "dtype"))
    idx, X, W, _ = _inputs(B, d, n_groups, G, k, dt, seed)
    L = n_groups * G
    rp, ids = I.make_zipf_positives(B, c["H"] + L, c["p"], 1.0, seed)
    (hp, hi), (tp, ti) = I.split_head_tail(rp, ids, c["H"])
    return idx, X, W, (tp, ti), (hp, hi)


def _run_step(plan, X, W, pos, scale):
    B = X.shape[0]
    Xt, Wt = to_torch(X), to_torch(W)
    rp, ids = to_torch(pos[0]), to_torch(pos[1] if len(pos[1]) else np.zeros(1, np.int32))
    ws = _ws(plan, B, H.dtype_code(Xt))
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    dW = torch.empty((plan.L, plan.k), dtype=Xt.dtype, device="cuda")
    dX = torch.full((B, plan.d), float("nan"), dtype=torch.float32, device="cuda")
    H.haste_bce_step(plan, Xt, Wt, rp, ids, scale, loss, dW, dX, ws)
    torch.cuda.synchronize()
    return loss, dW, dX


@pytest.mark.parametrize("case", STEP_CASES, ids=lambda c: _case_id(c) + f"_H{c['H']}")
def test_fused_bce_step(case):
    idx, X, W, tpos, _ = _step_inputs(case)
    B, d, G = case["B"], case["d"], case["G"]
    plan = H.haste_plan(idx, G, d)
    scale = 1.0 / B
    loss, dW, dX = _run_step(plan, X, W, tpos, scale)
    assert H.haste_device_status() == H.HASTE_OK
    r_loss, _, r_dW, r_dX = O.bce_step(X, W, idx, G, tpos[0], tpos[1], scale)
    got_loss = float(loss.item())
    assert abs(got_loss - r_loss) <= 5e-3 * abs(r_loss), (got_loss, r_loss)
    assert_close(to_np64(dW), r_dW, "dW")
    assert_close(to_np64(dX), r_dX, "dX")
    # determinism: a second run gives the same bits
    loss2, dW2, dX2 = _run_step(plan, X, W, tpos, scale)
    assert torch.equal(loss, loss2) and torch.equal(dW, dW2) and torch.equal(dX, dX2)


HEAD_CASES = [
    dict(B=256, Hh=384, d=192, dtype="bf16"),
    dict(B=128, Hh=256, d=128, dtype="f32"),
    dict(B=256, Hh=4096, d=768, dtype="bf16"),
    dict(B=100, Hh=200, d=136, dtype="bf16"),   # ragged: last 8 columns of every output tile, partial M tile
    dict(B=70, Hh=100, d=36, dtype="f32"),
]


@pytest.mark.parametrize("case", HEAD_CASES, ids=lambda c: "B{B}_H{Hh}_d{d}_{dtype}".format(**c))
def test_head_forward_backward(case):
    B, Hh, d, dt = case["B"], case["Hh"], case["d"], case["dtype"]
    Xh = I.make_normal((B, d), 1.0, 5, 5, dt)
    Wh = I.make_normal((Hh, d), 1.0 / math.sqrt(d), 5, 6, dt)
    rp, ids = I.make_zipf_positives(B, Hh, 4, 1.0, 5)
    Xht, Wht = to_torch(Xh), to_torch(Wh)
    ws = torch.empty(H.haste_head_workspace_size(B, Hh, d, H.dtype_code(Xht)), dtype=torch.uint8, device="cuda")
    logits = torch.empty((B, Hh), dtype=Xht.dtype, device="cuda")
    H.haste_head_forward(Xht, Wht, logits, ws)
    torch.cuda.synchronize()
    z = O.head_forward(Xh, Wh)
    assert_close(to_np64(logits), z, "head logits")
    # plain-torch fp32 cross-check of the same product
    ref32 = Xht.float() @ Wht.float().T
    assert_close(to_np64(logits), ref32.double().cpu().numpy(), "head logits vs torch")
    dYh = torch.empty_like(logits)
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    H.haste_head_forward(Xht, Wht, dYh, ws, to_torch(rp), to_torch(ids), 1.0 / B, loss)
    dWh = torch.empty_like(Wht)
    dXh = torch.empty((B, d), dtype=torch.float32, device="cuda")
    H.haste_head_backward(Xht, Wht, dYh, dWh, dXh, ws)
    torch.cuda.synchronize()
    r_loss, r_dY, r_dWh, r_dXh = O.head_step(Xh, Wh, rp, ids, 1.0 / B)
    assert abs(loss.item() - r_loss) <= 5e-3 * abs(r_loss)
    assert_close(to_np64(dYh), r_dY, "head dY")
    assert_close(to_np64(dWh), r_dWh, "head dW")
    assert_close(to_np64(dXh), r_dXh, "head dX")


def test_k_equals_d_reduces_to_dense_layer():
    """idx = [0..d) in every group: the sparse forward is a dense X . W^T."""
    B, d, n_groups, G = 128, 64, 32, 16
    idx = np.tile(np.arange(d, dtype=np.int32), (n_groups, 1))
    X = I.make_normal((B, d), 1.0, 9, 1, "bf16")
    W = I.make_normal((n_groups * G, d), 0.125, 9, 2, "bf16")
    plan = H.haste_plan(idx, G, d)
    Xt, Wt = to_torch(X), to_torch(W)
    ws = _ws(plan, B, H.HASTE_BF16)
    out = torch.empty((B, n_groups * G), dtype=torch.bfloat16, device="cuda")
    H.haste_forward(plan, Xt, Wt, out, ws)
    torch.cuda.synchronize()
    ref = (Xt.float() @ Wt.float().T).double().cpu().numpy()
    assert_close(to_np64(out), ref, "dense special case")


def test_error_statuses():
    idx = I.make_idx(64, 64, 256, 1)
    plan = H.haste_plan(idx, 16, 256)
    X = torch.zeros((32, 256), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((64 * 16, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((32, 64 * 16), dtype=torch.bfloat16, device="cuda")
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(H.HasteError) as e:
        H.haste_forward(plan, X, W, out, small)
    assert e.value.status == H.HASTE_ERR_WORKSPACE
    bad = H.haste_plan(I.make_idx(8, 48, 256, 1), 16, 256)       # k*2 bytes not a multiple of 128
    Wb = torch.zeros((8 * 16, 48), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(H.HasteError) as e:
        H.haste_forward(bad, X, Wb, torch.empty((32, 128), dtype=torch.bfloat16, device="cuda"), None)
    assert e.value.status == H.HASTE_ERR_UNSUPPORTED_SHAPE
    with pytest.raises(H.HasteError) as e:
        H.haste_plan(np.array([[0, 0]], dtype=np.int32), 16, 8)
    assert e.value.status == H.HASTE_ERR_INDEX_UNSORTED_OR_DUP


def test_bounded_wait_timeout_is_reported_and_context_survives():
    assert H.haste_device_status() == H.HASTE_OK
    assert H.lib().haste_selftest_wait_timeout(H._stream(None)) == H.HASTE_OK
    assert H.haste_device_status() == H.HASTE_ERR_TIMEOUT
    assert H.haste_device_status() == H.HASTE_OK          # cleared after reporting
    a = torch.ones(1024, device="cuda")
    assert float((a * 2).sum().item()) == 2048.0


def test_short_wait_limit_reaches_the_abort_paths_and_the_context_survives():
    """A 1 ns limit on the pipelined kernels' inter-warp waits makes the step
    kernel's first wait of every warp run out at once (a limit below one sleep
    raises the CTA's abort flag at the start), and the top-k kernel's first wait
    that has to sleep, so that each takes its abort path (drain its own copies,
    commit and wait for its issued MMAs, free TMEM).  The timeout is reported once;
    with the default limit restored, the same calls give the oracle's results."""
    c = dict(B=256, d=768, n_groups=300, G=32, k=128, dtype="bf16", H=0, p=5)
    idx, X, W, tpos, _ = _step_inputs(c)
    plan = H.haste_plan(idx, c["G"], c["d"])
    scale = 1.0 / c["B"]
    nb, K, kp = 37, 5, 4
    ws = torch.empty(H.haste_topk_workspace_size(plan, c["B"], H.HASTE_BF16, nb, kp), dtype=torch.uint8,
                     device="cuda")
    ov = torch.empty((c["B"], K), device="cuda")
    oi = torch.empty((c["B"], K), dtype=torch.int32, device="cuda")
    try:
        H.haste_set_wait_limit_ns(1)
        _run_step(plan, X, W, tpos, scale)
        assert H.haste_device_status() == H.HASTE_ERR_TIMEOUT
        H.haste_topk(plan, to_torch(X), to_torch(W), K, kp, nb, ov, oi, ws)
        assert H.haste_device_status() == H.HASTE_ERR_TIMEOUT
    finally:
        H.haste_set_wait_limit_ns(0)
    assert H.haste_device_status() == H.HASTE_OK
    loss, dW, dX = _run_step(plan, X, W, tpos, scale)
    assert H.haste_device_status() == H.HASTE_OK
    r_loss, _, r_dW, r_dX = O.bce_step(X, W, idx, c["G"], tpos[0], tpos[1], scale)
    assert abs(float(loss.item()) - r_loss) <= 5e-3 * abs(r_loss)
    assert_close(to_np64(dW), r_dW, "dW after the aborted call")
    assert_close(to_np64(dX), r_dX, "dX after the aborted call")
    with pytest.raises(H.HasteError):
        H.haste_set_wait_limit_ns(10 ** 12)       # above the 2 s default


SGD_CASES = [
    dict(B=256, d=768, n_groups=300, G=64, k=128, dtype="bf16", H=0, p=8, lr=8.0, mu=0.9),
    dict(B=130, d=384, n_groups=250, G=32, k=64, dtype="bf16", H=0, p=5, lr=16.0, mu=0.0),
    dict(B=100, d=256, n_groups=120, G=16, k=64, dtype="bf16", H=0, p=5, lr=12.0, mu=0.5),
    dict(B=180, d=384, n_groups=211, G=16, k=128, dtype="bf16", H=0, p=5, lr=10.0, mu=0.9),
]


@pytest.mark.parametrize("case", SGD_CASES, ids=lambda c: _case_id(c) + f"_mu{c['mu']}")
def test_fused_step_with_sgd_update_two_steps(case):
    """haste_bce_step_sgd over two steps, alternating two weight buffers as a
    training loop does: the loss and dX of each step use that step's input
    weights, the momentum buffer and the new weights follow the oracle's SGD
    update.  lr is large, so that the update dominates W' and the bf16 rounding
    of W' (about 2^-9 of W' in relative terms) stays well inside the tolerance on
    W' - W; with an update the size of W, that rounding alone is about half the
    rel-L2 tolerance."""
    idx, X, W0, tpos, _ = _step_inputs(case)
    B, d, G, k = case["B"], case["d"], case["G"], case["k"]
    lr, mu = case["lr"], case["mu"]
    plan = H.haste_plan(idx, G, d)
    scale = 1.0 / B
    M0 = I.make_normal((plan.L, k), 0.03, 0, 4, "bf16") if mu else None
    Xt = to_torch(X)
    rp, ids = to_torch(tpos[0]), to_torch(tpos[1])
    ws = _ws(plan, B, H.HASTE_BF16)
    bufs = [to_torch(W0), torch.empty_like(to_torch(W0))]
    Mt = to_torch(M0) if mu else None
    W_ref, M_ref = W0, M0
    for step in range(2):
        Win, Wout = bufs[step % 2], bufs[(step + 1) % 2]
        Win_before = Win.clone()
        loss = torch.zeros(1, device="cuda")
        dX = torch.full((B, d), float("nan"), device="cuda")
        H.haste_bce_step_sgd(plan, Xt, Win, rp, ids, scale, loss, lr, mu, Mt, Wout, dX, ws)
        torch.cuda.synchronize()
        assert H.haste_device_status() == H.HASTE_OK
        assert torch.equal(Win.view(torch.int16), Win_before.view(torch.int16))   # W is only read
        r_loss, r_dX, r_W, r_M = O.bce_step_sgd(X, W_ref, M_ref, idx, G, tpos[0], tpos[1], scale, lr, mu)
        assert abs(float(loss.item()) - r_loss) <= 5e-3 * abs(r_loss), (step, float(loss.item()), r_loss)
        assert_close(to_np64(dX), r_dX, f"dX, step {step + 1}")
        W_in64 = O.to_f64(W_ref)
        assert_close(to_np64(Wout) - W_in64, r_W - W_in64, f"W' - W, step {step + 1}")
        if mu:
            assert_close(to_np64(Mt), r_M, f"momentum, step {step + 1}")
            M_ref = Mt.view(torch.int16).cpu().numpy().view(np.uint16).copy()
        # the next step starts from the GPU's rounded weights, as the oracle's input
        W_ref = Wout.view(torch.int16).cpu().numpy().view(np.uint16).copy()


def test_fused_update_argument_errors():
    idx = I.make_idx(40, 64, 256, 0)
    plan = H.haste_plan(idx, 32, 256)
    B = 8
    X = torch.zeros((B, 256), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((40 * 32, 64), dtype=torch.bfloat16, device="cuda")
    rp = torch.zeros(B + 1, dtype=torch.int32, device="cuda")
    ids = torch.zeros(1, dtype=torch.int32, device="cuda")
    dX = torch.empty((B, 256), device="cuda")
    ws = _ws(plan, B, H.HASTE_BF16)
    with pytest.raises(H.HasteError) as e:                       # the update must not overwrite W
        H.haste_bce_step_sgd(plan, X, W, rp, ids, 0.1, None, 0.1, 0.0, None, W, dX, ws)
    assert e.value.status == H.HASTE_ERR_INVALID_ARG
    with pytest.raises(ValueError):                             # momentum needs its buffer
        H.haste_bce_step_sgd(plan, X, W, rp, ids, 0.1, None, 0.1, 0.9, None, torch.empty_like(W), dX, ws)
    Xf = torch.zeros((B, 256), device="cuda")
    with pytest.raises(H.HasteError) as e:                       # fp32 runs the staged kernels: no fused update
        H.haste_bce_step_sgd(plan, Xf, W.float(), rp, ids, 0.1, None, 0.1, 0.0, None, torch.empty_like(W.float()),
                             dX, _ws(plan, B, H.HASTE_F32))
    assert e.value.status == H.HASTE_ERR_UNSUPPORTED_SHAPE


def _rewire(idx, d, frac_groups, frac_slots, seed):
    """A random prune/regrow edit, the test's own rule: in a fraction of the groups,
    drop a fraction of the features and draw replacements among the features the
    group does not use, then sort the row.  Returns (groups, rows, new idx)."""
    rng = np.random.default_rng(seed)
    n_groups, k = idx.shape
    groups = np.sort(rng.choice(n_groups, max(1, int(frac_groups * n_groups)), replace=False)).astype(np.int32)
    rows = idx[groups].copy()
    n_drop = max(1, int(frac_slots * k))
    for r in range(len(groups)):
        kept = rows[r][rng.choice(k, k - n_drop, replace=False)]
        new = rng.choice(np.setdiff1d(np.arange(d), rows[r]), n_drop, replace=False)
        rows[r] = np.sort(np.concatenate([kept, new]))
    out = idx.copy()
    out[groups] = rows
    return groups, rows, out


@pytest.mark.parametrize("n_groups,k,d", [(20_944, 128, 768), (1000, 64, 97), (7, 3, 5), (134_376, 128, 768)])
def test_plan_update_is_bit_exact_against_the_oracle(n_groups, k, d):
    """Three rounds of rewiring; after each, the device arrays equal the oracle's
    stable counting sort of the new index sets."""
    idx = I.make_idx(n_groups, k, d, 3)
    plan = H.haste_plan(idx, 32, d)
    e_idx, e_off, e_ent = plan.export()
    st, r_off, r_ent = O.plan(idx, d)
    assert np.array_equal(e_off, r_off) and np.array_equal(e_ent, r_ent)   # the device-built plan
    for it in range(3):
        frac = 0.01 if n_groups > 100_000 else 0.05
        groups, rows, idx = _rewire(idx, d, frac, 0.25 if k > 4 else 0.34, it)
        plan.update(groups, rows)
        torch.cuda.synchronize()
        e_idx, e_off, e_ent = plan.export()
        st, r_off, r_ent = O.plan(idx, d)
        assert st == O.OK
        assert np.array_equal(e_idx, idx), it
        assert np.array_equal(e_off, r_off) and np.array_equal(e_ent, r_ent), it


def test_fused_step_after_a_plan_update_uses_the_new_sets():
    c = dict(B=130, d=384, n_groups=250, G=32, k=64, dtype="bf16", H=0, p=5)
    idx, X, W, tpos, _ = _step_inputs(c)
    plan = H.haste_plan(idx, c["G"], c["d"])
    groups, rows, idx2 = _rewire(idx, c["d"], 0.3, 0.5, 11)
    plan.update(groups, rows)
    scale = 1.0 / c["B"]
    loss, dW, dX = _run_step(plan, X, W, tpos, scale)
    assert H.haste_device_status() == H.HASTE_OK
    r_loss, _, r_dW, r_dX = O.bce_step(X, W, idx2, c["G"], tpos[0], tpos[1], scale)
    assert abs(float(loss.item()) - r_loss) <= 5e-3 * abs(r_loss)
    assert_close(to_np64(dW), r_dW, "dW after the update")
    assert_close(to_np64(dX), r_dX, "dX after the update")


def test_plan_update_rejects_bad_edits_and_keeps_the_plan():
    idx = I.make_idx(50, 16, 64, 2)
    plan = H.haste_plan(idx, 16, 64)
    good = np.sort(np.random.default_rng(0).choice(64, 16, replace=False)).astype(np.int32)
    bad_rows = [good.copy(), good.copy()]
    bad_rows[0][3] = bad_rows[0][2]                 # a duplicate
    bad_rows[1][-1] = 64                            # out of range
    for row, code in zip(bad_rows, (H.HASTE_ERR_INDEX_UNSORTED_OR_DUP, H.HASTE_ERR_INDEX_OUT_OF_RANGE)):
        with pytest.raises(H.HasteError) as e:
            plan.update(np.array([4]), row[None, :])
        assert e.value.status == code
    for groups in (np.array([5, 5]), np.array([7, 3]), np.array([50])):   # repeated, descending, out of range
        with pytest.raises(H.HasteError) as e:
            plan.update(groups, np.tile(good, (len(groups), 1)))
        assert e.value.status == H.HASTE_ERR_INVALID_ARG
    e_idx, e_off, e_ent = plan.export()
    st, r_off, r_ent = O.plan(idx, 64)
    assert np.array_equal(e_idx, idx) and np.array_equal(e_off, r_off) and np.array_equal(e_ent, r_ent)
