"""Multi-rank host logic of bench.py on CPU ranks (gloo, world size 2).

The layer runs as independent replicas, one per GPU, each on its own batch
(weak scaling, no collective on the data path).  What crosses ranks is the
timing: every rank reports its own device time and the job takes the slowest
rank's; the whole-job value counts the samples of all ranks.  The reference arm
(the oracle on host cores) runs on rank 0 only; other ranks exit without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    from structured_sparse_output_b200 import inputs as I
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        own = 10.0 + 7.5 * rank                       # rank 1 is the slow one
        slow = bench.max_over_ranks(own, "cpu")
        value = bench.job_value(world, 256, 20, slow)
        # every rank draws its own batch: seeds differ, shapes agree
        X = I.make_normal((4, 8), 1.0, rank, 1, "bf16")
        gathered = [torch.zeros(32, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(X.astype("int32").ravel()))
        same = bool(torch.equal(gathered[0], gathered[1]))
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as fh:
            json.dump({"slow": slow, "value": value, "same_batch": same}, fh)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["slow"] == 17.5                      # both ranks see the slowest rank's time
        assert r["value"] == pytest.approx(world * 256 * 20 / 17.5e-3)
        assert r["same_batch"] is False               # replicas run on different batches
    assert res[0] == res[1]


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--config", "tiny", "--steps", "3", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr
    line = json.loads(p.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "samples/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
