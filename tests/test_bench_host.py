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


NCU_CSV = '''==PROF== Connected to process 4242
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"3","4242","python3","127.0.0.1","void pa::plan_kernel(const int *, int)","1","7","(1024, 1, 1)","(1, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","4,096"
"4","4242","python3","127.0.0.1","void pa::decode_kernel<1, true, 128, 16>(pa::DecodeArgs)","1","7","(128, 1, 1)","(444, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","1,077.45"
"4","4242","python3","127.0.0.1","void pa::decode_kernel<1, true, 128, 16>(pa::DecodeArgs)","1","7","(128, 1, 1)","(444, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","7,160,000"
"4","4242","python3","127.0.0.1","void pa::decode_kernel<1, true, 128, 16>(pa::DecodeArgs)","1","7","(128, 1, 1)","(444, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","ns","183900"
'''


def test_ingest_ncu_records_scaled_traffic(tmp_path, monkeypatch):
    """An ncu metrics log of the decode kernel on 64 of the headline batch's
    256 sequences becomes a traffic record scaled x4 to the full batch, keyed
    to the kernel's source hash; bench reads it back only while the hash
    matches."""
    sys.path.insert(0, ROOT)
    import json
    import bench
    csv_path = tmp_path / "launches.csv"
    csv_path.write_text(NCU_CSV)
    traffic = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(traffic))
    launches = bench.parse_ncu_csv(str(csv_path), "decode_kernel")
    assert list(launches) == ["4"]
    m = launches["4"]
    assert m["dram__bytes_read.sum"] == pytest.approx(1.07745e9)
    assert m["gpu__time_duration.sum"] == pytest.approx(183.9e-6)
    assert bench.main(["--ingest-ncu", str(csv_path), "--num-seqs", "64",
                       "--ingest-command", "ncu ... bench.py --num-seqs 64"]) == 0
    rec = json.loads(traffic.read_text())["decode_kernel:llama70b_gqa"]
    assert rec["scale_to_full"] == pytest.approx(4.0)
    assert rec["dram_bytes_per_launch_full"] == round((1.07745e9 + 7.16e6) * 4)
    assert rec["source_sha16"] == bench.source_hash("decode_kernel")
    got, _ = bench.profiled_traffic("llama70b_gqa")
    assert got == rec["dram_bytes_per_launch_full"]
    # a changed kernel source makes the figure stale
    monkeypatch.setattr(bench, "source_hash", lambda k: "0" * 16)
    assert bench.profiled_traffic("llama70b_gqa")[0] is None


def test_config_memory_figures():
    """Paged waste is the unfilled tail of each last block; a contiguous
    reservation wastes its length minus the context; the shared-prefix batch
    holds its prompt blocks once for four samples."""
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_416_b200 import workloads as W
    w = W.make("tiny")
    m = bench.config_memory(w, "tiny")
    # lens [40, 16, 1, 63] in blocks of 16: 3 + 1 + 1 + 4 blocks, 144 slots, 120 used
    assert m["paged_unused_slots"] == 24 and m["reserved_unused_slots"] == 4 * 2048 - 120
    w = W.make("shared_prefix_tails", prompts=3)
    m = bench.config_memory(w, "shared_prefix_tails")
    assert m["blocks_shared"] < m["blocks_unshared"]
    assert 0 < m["memory_saved_pct"] < 75


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("llama13b_mha", dict(num_seqs=6)),
                                     ("llama70b_gqa", dict(num_seqs=3, context_len=1000)),
                                     ("shared_prefix_fork", dict(prompts=3)),
                                     ("shared_prefix_tails", dict(prompts=3)),
                                     ("fp8_longtail_bs16", dict(num_seqs=10, max_len=6000)),
                                     ("fp8_longtail_bs32", dict(num_seqs=10))])
def test_lengths_without_pools_match_the_generators(name, kw):
    sys.path.insert(0, ROOT)
    import numpy as np
    from paged_kv_cache_416_b200 import workloads as W
    w = W.make(name, **kw)
    assert np.array_equal(W.context_lens(name, **kw), w.context_lens)
    assert W.kv_bytes_of(name, **kw) == w.kv_bytes
