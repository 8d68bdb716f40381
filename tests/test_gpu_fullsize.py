"""Full-size GPU parity on sampled outputs, in the launch configuration bench.py times.

Each workload of the benchmark (670K, 3M and 8.6M labels with the fused BCE step
and the dense head; the 1M-label group-size sweep at G = 16, 32, 64 with a given
gradient) runs once through bench.Runner, i.e. through the C ABI exactly as the
benchmark calls it.  The oracle evaluates the same seeded inputs one output at a
time (dW entries, dX entries, logits) in fp64; the head is compared in full.  The
samples include the first and last group, label, feature and batch row.  A second
run checks that every output is bitwise identical (no float atomics, fixed
reduction order).
Source: "HASTE: Hardware-Aware Dynamic Sparse Training for Large Output Spaces"
(summary page), Methodology 1 (group-shared fan-in layer) and 2 (dense head).
"""
import numpy as np
import pytest

from oracle import oracle as O
from structured_sparse_output_b200 import inputs as I
from tests.helpers import assert_close, to_np64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield


def _samples(wl, n_dw=48, n_dx=24, seed=11):
    rng = np.random.default_rng(seed)
    ls = np.concatenate([[0, wl.G - 1, wl.L - wl.G, wl.L - 1], rng.integers(0, wl.L, n_dw - 4)]).astype(np.int64)
    ss = np.concatenate([[0, wl.k - 1, 0, wl.k - 1], rng.integers(0, wl.k, n_dw - 4)]).astype(np.int32)
    bs = np.concatenate([[0, wl.B - 1, wl.B // 2], rng.integers(0, wl.B, n_dx - 3)]).astype(np.int32)
    fs = np.concatenate([[0, wl.d - 1, wl.d // 2], rng.integers(0, wl.d, n_dx - 3)]).astype(np.int32)
    return ls, ss, bs, fs


def _same(a, b):
    """Bitwise equality (bf16 tensors compared through their bit patterns)."""
    if a.dtype == torch.bfloat16:
        a, b = a.view(torch.int16), b.view(torch.int16)
    return torch.equal(a, b)


def _run(run):
    run.step()
    torch.cuda.synchronize()
    from structured_sparse_output_b200 import haste as H
    assert H.haste_device_status() == H.HASTE_OK


def _row_subset(pos, rows):
    """The positives CSR of the given batch rows only."""
    rp, ids = pos
    sub_rp = np.concatenate([[0], np.cumsum([rp[b + 1] - rp[b] for b in rows])]).astype(np.int32)
    sub_ids = np.concatenate([ids[rp[b]:rp[b + 1]] for b in rows]).astype(np.int32)
    return sub_rp, sub_ids


@pytest.mark.parametrize("name", ["670k", "3m", "8.6m"])
def test_fused_step_full_size_sampled(name):
    import bench
    wl = I.WORKLOADS[name]
    run = bench.Runner(wl, seed=0)
    inp = run.inp
    _run(run)
    dW1, dX1, dWh1, dXh1 = (t.clone() for t in (run.dW, run.dX, run.dWh, run.dXh))
    loss1 = run.loss.clone()
    _run(run)
    # bitwise run-to-run determinism of every output of the step
    for a, b in ((dW1, run.dW), (dX1, run.dX), (dWh1, run.dWh), (dXh1, run.dXh), (loss1, run.loss)):
        assert _same(a, b)
    scale = 1.0 / wl.B
    # the tail loss over every sample and label
    r_loss = O.bce_loss(inp.X, inp.W, inp.idx, wl.G, inp.tail_pos[0], inp.tail_pos[1], scale)
    assert abs(float(run.loss[0].item()) - r_loss) <= 5e-3 * abs(r_loss), (float(run.loss[0].item()), r_loss)
    ls, ss, bs, fs = _samples(wl, n_dw=400, n_dx=64)
    dW = run.dW.float().cpu().numpy()
    dX = run.dX.cpu().numpy()
    r_dw = O.dw_at(inp.X, inp.W, inp.idx, wl.G, ls, ss, pos=inp.tail_pos, scale=scale)
    r_dx = O.dx_at(inp.X, inp.W, inp.idx, wl.G, bs, fs, pos=inp.tail_pos, scale=scale)
    assert_close(dW[ls, ss].astype(np.float64), r_dw, f"{name} dW samples")
    assert_close(dX[bs, fs].astype(np.float64), r_dx, f"{name} dX samples")
    if name == "670k":
        # whole dX rows: a row's gradient depends on that row only, so the oracle's
        # step over a subset of rows (same scale) gives those rows exactly
        rows = np.array([0, 1, 2, 3, 128, wl.B - 1])
        _, _, _, r_rows = O.bce_step(inp.X[rows], inp.W, inp.idx, wl.G, *_row_subset(inp.tail_pos, rows), scale)
        assert_close(dX[rows].astype(np.float64), r_rows, f"{name} dX rows {rows.tolist()}")
    # the dense head in full
    h_loss, _, h_dWh, h_dXh = O.head_step(inp.Xh, inp.Wh, inp.head_pos[0], inp.head_pos[1], scale)
    assert_close(to_np64(run.dWh), h_dWh, f"{name} head dWh")
    assert_close(to_np64(run.dXh), h_dXh, f"{name} head dXh")
    assert abs(float(run.loss[1].item()) - h_loss) <= 5e-3 * abs(h_loss)


@pytest.mark.parametrize("name", ["sweep16", "sweep32", "sweep64"])
def test_given_gradient_full_size_sampled(name):
    import bench
    wl = I.WORKLOADS[name]
    run = bench.Runner(wl, seed=0)
    inp = run.inp
    _run(run)
    lg1, dW1, dX1 = run.logits.clone(), run.dW.clone(), run.dX.clone()
    _run(run)
    assert _same(lg1, run.logits) and _same(dW1, run.dW) and _same(dX1, run.dX)
    ls, ss, bs, fs = _samples(wl)
    rng = np.random.default_rng(5)
    lb = np.concatenate([[0, wl.B - 1], rng.integers(0, wl.B, 46)]).astype(np.int32)
    ll = np.concatenate([[0, wl.L - 1], rng.integers(0, wl.L, 46)]).astype(np.int64)
    r_lg = O.logits_at(inp.X, inp.W, inp.idx, wl.G, lb, ll)
    r_dw = O.dw_at(inp.X, inp.W, inp.idx, wl.G, ls, ss, dY=inp.dY)
    r_dx = O.dx_at(inp.X, inp.W, inp.idx, wl.G, bs, fs, dY=inp.dY)
    logits = run.logits
    got_lg = np.array([float(logits[int(b), int(l)].item()) for b, l in zip(lb, ll)])
    dW = run.dW.float().cpu().numpy()
    dX = run.dX.cpu().numpy()
    assert_close(got_lg, r_lg, f"{name} logits samples")
    assert_close(dW[ls, ss].astype(np.float64), r_dw, f"{name} dW samples")
    assert_close(dX[bs, fs].astype(np.float64), r_dx, f"{name} dX samples")
