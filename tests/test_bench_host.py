"""Host logic of bench.py's multi-GPU mode (replicas only), on CPU with gloo.

Every rank runs its own replica of the workload; the process group is used
only for the barrier and for the whole-job numbers: the slowest rank's time
(max over ranks) and the units all ranks processed (sum over ranks).
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, local, w = bench.dist_init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    dev = torch.device("cpu")
    bench.barrier(w, None)
    # rank r "took" (r + 1) seconds for 10 steps of (r + 1) GB each
    slowest = bench.reduce_max(float(rank + 1), w, dev)
    gbs, tps = bench.aggregate((rank + 1) * 1e9, 1000.0 * (rank + 1), 10, slowest, w, dev)
    out_q.put((rank, slowest, gbs, tps))
    dist.destroy_process_group()


def test_two_replicas_aggregate_with_max_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, gbs, tps in res:
        assert slowest == 2.0                         # max over ranks
        assert gbs == pytest.approx((1 + 2) * 10 / 2.0)  # all ranks' bytes / slowest time
        assert tps == pytest.approx((1000 + 2000) * 10 / 2.0)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, 1, None) == 3.5
    gbs, tps = bench.aggregate(2e9, 100.0, 5, 2.0, 1, None)
    assert gbs == pytest.approx(5.0) and tps == pytest.approx(250.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line(capsys):
    sys.path.insert(0, ROOT)
    import json
    import bench
    assert bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1",
                       "--warmup", "3"]) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
