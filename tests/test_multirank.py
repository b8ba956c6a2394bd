"""The multi-process path of bench.py (one process per GPU under torchrun) on CPU: two ranks over gloo.

bench.py runs independent replicas (the decode rows and the prefill are independent units; there is no
data-path exchange), so the only multi-rank logic is the process group, the barriers around the timed
region, the max over ranks of the device time, the whole-job rate, and rank 0 alone printing the line.
"""
import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    ws, r, local = bench.dist_setup(world, backend="gloo")
    assert (ws, r, local) == (world, rank, rank)
    bench.barrier(ws, cuda=False)
    # a per-rank "device time": rank 1 is the slow one
    t = bench.barrier_max(0.5 + rank, ws, device="cpu")
    rate = bench.whole_job_rate(4 * 100, ws, t)
    bench.barrier(ws, cuda=False)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"t": t, "rate": rate}, f)


def test_two_ranks_gloo(tmp_path):
    import torch.multiprocessing as mp

    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    # both ranks agree on the slowest rank's time, and the rate counts both ranks' units
    assert res[0]["t"] == res[1]["t"] == pytest.approx(1.5)
    assert res[0]["rate"] == res[1]["rate"] == pytest.approx(2 * 400 / 1.5)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.barrier_max(0.25, 1, device="cpu") == 0.25
    assert bench.whole_job_rate(400, 1, 2.0) == 200.0


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    """under torchrun only rank 0 runs the oracle arm; the others return at once"""
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, gpus = 1, 0, 2

    assert bench.run_reference(Args()) is None
