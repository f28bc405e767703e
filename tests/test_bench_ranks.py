"""Host logic of bench.py's multi-rank mode, on CPU with the gloo backend
(world size 2): every rank takes the same collective steps, the reported
device time is the maximum over ranks, the whole-job value counts every
rank's replica, each rank draws its own seeded workload of the same shape,
and the reference arm runs on rank 0 only.  Also on CPU: the unmasked-pair
counts behind the bench's FLOP figures equal the oracle's."""
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
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # rank-specific "device times": the maximum must win element-wise
        got = bench.reduce_max([10.0 + rank, 5.0 - rank, 7.5], world, "cpu")
        wl = bench.workload("n8192", rank)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": got, "seed": wl["seed"], "shape": [wl["n"], wl["B"], wl["H"], wl["D"]],
                       "lts0": int(wl["masks"][1][1][0].vectors()[0][0])}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_workloads_world2(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == [11.0, 5.0, 7.5]
        assert r["shape"] == [8192, 2, 16, 128]
    assert res[0]["seed"] != res[1]["seed"]  # weak scaling: each rank its own replica of the workload


def test_job_value_counts_every_rank():
    # 2 ranks, each 1e12 flop per step, 4 steps, slowest rank 2000 ms -> 4 TFLOP/s for the job
    assert bench.job_tflops(2, 1e12, 4, 2000.0) == pytest.approx(4.0)
    assert bench.job_tflops(1, 1e12, 4, 2000.0) == pytest.approx(2.0)
    assert bench.reduce_max([3.0, 1.0], 1, "cpu") == [3.0, 1.0]


def test_reference_arm_only_on_rank0():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("config", ["n8192", "n32768", "n131072"])
def test_bench_unmasked_pairs_match_oracle(config):
    """The U behind every effective-TFLOP/s figure of the bench (4·D·U·H forward, 10·D·U·H
    backward): the bench's interval count equals the oracle's count for each batch row of each
    mask of the workload."""
    import oracle
    wl = bench.workload(config, 0)
    n = wl["n"]
    for name, rows in wl["masks"]:
        got = bench.unmasked_pairs(rows, n)
        want = [oracle.count_unmasked(n, n, *s.vectors()) for s in rows]
        assert got == want, name


def test_bench_unmasked_pairs_match_dense_small():
    import oracle
    import synth
    n = 384
    rows = [synth.make_family(f, n, 3) for f in synth.SWEEP_FAMILIES]
    assert bench.unmasked_pairs(rows, n) == [oracle.count_unmasked_dense(n, n, *s.vectors()) for s in rows]
