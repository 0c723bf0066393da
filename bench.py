#!/usr/bin/env python
"""Benchmark of the paged decode step on B200; prints ONE JSON line (rank 0).

A step is one pass of the whole hot path over one batch: copy-on-write block
copies (none in the default workload), the cache write of every sequence's
new token (pa_write_kv), and paged decode attention over all sequences
(pa_decode: plan kernel + decode kernel, which also merges split contexts).

Default workload: the Llama-3-70B-shaped GQA decode layer -- 256 sequences
x 4096 tokens, 64 query / 8 KV heads, head_dim 128, bf16, block_size 16,
physical blocks randomly permuted (4 GiB of K+V read per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Multi-GPU (torchrun, one process per GPU): replicas only -- every rank runs
its own copy of the workload, no collective touches the data path; the
barrier and the max-over-ranks timing use the process group.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attn: KV-read GB/s (% of HBM peak), seq-tokens/s"
NOMINAL_HBM_GBS = 8000.0      # the "~8 TB/s" B200 figure the target is stated against
FALLBACK_HBM_GBS = 6650.0     # used only when MEASURED_PEAKS.json is absent
DEFAULT_WORKLOAD = "llama70b_gqa"
# DRAM bytes per launch of each kernel, taken from ncu captures by
# `bench.py --ingest-ncu`; an entry counts only while the kernel's sources
# hash as they did when it was captured
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")
CSRC = os.path.join(ROOT, "paged_kv_cache_416_b200", "csrc")
KERNEL_SOURCES = {
    "decode_kernel": ("decode.cuh", "common.cuh"),
    "cascade_kernel": ("cascade.cuh", "decode.cuh", "common.cuh"),
}
# the five benchmark configurations as workloads (config 4 is two steps of one
# batch, config 5 runs at block sizes 16 and 32), in the order they are named
CONFIG_WORKLOADS = ["tiny", "llama13b_mha", "llama70b_gqa", "shared_prefix_fork",
                    "shared_prefix_tails", "fp8_longtail_bs16", "fp8_longtail_bs32"]
# tokens a contiguous (maximum-length) reservation would hold per sequence:
# each generator's length bound (the tiny batch takes the 2048 of the pages'
# worked example; shared prefix: 1024 + 15 prompt tokens, 512 own tokens, the
# fork step's token and the step's token)
RESERVATION_TOKENS = {"tiny": 2048, "llama13b_mha": 2048, "llama70b_gqa": 4096,
                      "shared_prefix_fork": 1024 + 15 + 512 + 2,
                      "shared_prefix_tails": 1024 + 15 + 512 + 2,
                      "fp8_longtail_bs16": 32768, "fp8_longtail_bs32": 32768}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=None,
                    help="input seed (default: the workload's own, 1..5 by configuration)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config-cpu-seconds", type=float, default=3.0,
                    help="target CPU time of each configuration's oracle sample")
    ap.add_argument("--config-iters", type=int, default=30,
                    help="timed iterations per configuration in the `configs` object")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration measurements (profiling runs)")
    ap.add_argument("--ingest-ncu", default=None, metavar="CSV",
                    help="read an ncu --csv capture of one kernel (dram__bytes_read.sum, "
                         "dram__bytes_write.sum) of --workload [--num-seqs] and record its "
                         "per-launch DRAM bytes, scaled to the full workload, in "
                         "profiles/decode_traffic.json; no GPU work")
    ap.add_argument("--ingest-kernel", default="decode_kernel", choices=sorted(KERNEL_SOURCES))
    ap.add_argument("--ingest-command", default="",
                    help="the command line that produced the capture (recorded)")
    ap.add_argument("--ingest-source-sha16", default=None,
                    help="source hash of the kernel when it was captured (bench.py "
                         "--print-source-sha16 on the capturing machine); must match the "
                         "sources here, else nothing is recorded")
    ap.add_argument("--print-source-sha16", action="store_true",
                    help="print the decode and cascade kernels' source hashes and exit")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiling only)")
    ap.add_argument("--op", choices=["decode", "swap", "hash", "prefill", "shared_prefix"],
                    default="decode",
                    help="decode: the decode step (the headline line); the others time "
                         "one companion operation on one GPU and print its own line")
    return ap.parse_args(argv)


# ------------------------------------------------------------ distributed
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def dist_init(backend: str, timeout_s: int = 300):
    import torch.distributed as dist
    rank, local, world = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, local, world


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def reduce_max(x: float, world: int, device) -> float:
    """Max of x over ranks (x itself at world 1)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x: float, world: int, device) -> float:
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(bytes_per_step_per_rank: float, tokens_per_step_per_rank: float, steps: int,
              max_seconds: float, world: int, device):
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    total_bytes = reduce_sum(bytes_per_step_per_rank * steps, world, device)
    total_tokens = reduce_sum(tokens_per_step_per_rank * steps, world, device)
    return total_bytes / max_seconds / 1e9, total_tokens / max_seconds


# ----------------------------------------------------------------- clocks
NVML_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """Reads the SM clock and clock-event reasons through NVML on a thread
    while running (read-only queries; no setting is changed)."""

    def __init__(self, torch_device_index: int = 0, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        self._th = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            h = None
            try:
                uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.h = h
            self.nv = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = get_r(self.h)
                self.samples.append((float(sm), int(r)))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._th = threading.Thread(target=self._run, daemon=True)
            self._th.start()

    def stop(self):
        if self._th is not None:
            self._stop.set()
            self._th.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = sorted(s[0] for s in self.samples)
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = [n for b, n in NVML_REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ----------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _load_traffic():
    if not os.path.exists(TRAFFIC_FILE):
        return {}
    with open(TRAFFIC_FILE) as f:
        return json.load(f)


def profiled_traffic(workload: str, kernel: str = "decode_kernel"):
    """DRAM bytes per launch of `kernel` on the full `workload`, from the
    recorded ncu capture, while the kernel's sources still hash as captured
    (else None).  Returns (bytes or None, the record or None)."""
    rec = _load_traffic().get(f"{kernel}:{workload}")
    if rec is None:
        return None, None
    if rec.get("source_sha16") != source_hash(kernel):
        return None, rec
    return int(rec["dram_bytes_per_launch_full"]), rec


_NCU_UNITS = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
              "nsecond": 1e-9, "usecond": 1e-6, "msecond": 1e-3, "second": 1.0,
              "ns": 1e-9, "us": 1e-6, "ms": 1e-3, "s": 1.0}


def parse_ncu_csv(path: str, kernel: str):
    """Per-launch metric values of the launches of `kernel` in an ncu --csv
    metrics log: {launch id: {metric: value in base units}}."""
    import csv
    with open(path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]
    rows = list(csv.DictReader(lines))
    out = {}
    for r in rows:
        if kernel not in r.get("Kernel Name", ""):
            continue
        unit = r.get("Metric Unit", "").strip().lower()
        val = float(r["Metric Value"].replace(",", ""))
        out.setdefault(r["ID"], {})[r["Metric Name"]] = val * _NCU_UNITS.get(unit, 1.0)
    return out


def ingest_ncu(args):
    """Record the DRAM traffic of one captured kernel launch per workload."""
    from paged_kv_cache_416_b200 import workloads as W
    here = source_hash(args.ingest_kernel)
    if args.ingest_source_sha16 is not None and args.ingest_source_sha16 != here:
        raise SystemExit(f"the capture is of {args.ingest_kernel} source {args.ingest_source_sha16}, "
                         f"the sources here hash {here}: not recorded")
    launches = parse_ncu_csv(args.ingest_ncu, args.ingest_kernel)
    if not launches:
        raise SystemExit(f"no {args.ingest_kernel} launch in {args.ingest_ncu}")
    rd = [m["dram__bytes_read.sum"] for m in launches.values()]
    wr = [m["dram__bytes_write.sum"] for m in launches.values()]
    seed = args.seed
    kw = _sample_kw(args.workload, args.num_seqs) if args.num_seqs else {}
    cap_bytes = W.kv_bytes_of(args.workload, seed, **kw)
    full_bytes = W.kv_bytes_of(args.workload, seed)
    cap_seqs = len(W.context_lens(args.workload, seed, **kw))
    full_seqs = len(W.context_lens(args.workload, seed))
    scale = full_bytes / cap_bytes
    per_launch = (sum(rd) + sum(wr)) / len(rd)
    rec = {
        "kernel": args.ingest_kernel, "workload": args.workload,
        "source_sha16": source_hash(args.ingest_kernel),
        "sources": list(KERNEL_SOURCES[args.ingest_kernel]),
        "captured_num_seqs": cap_seqs, "full_num_seqs": full_seqs,
        "launches": len(rd),
        "dram_bytes_read_per_launch": round(sum(rd) / len(rd)),
        "dram_bytes_write_per_launch": round(sum(wr) / len(wr)),
        "algorithmic_kv_bytes_captured": cap_bytes,
        "scale_to_full": scale,
        "dram_bytes_per_launch_full": round(per_launch * scale),
        "ratio_to_algorithmic": round(per_launch / cap_bytes, 4),
        "command": args.ingest_command,
    }
    if "gpu__time_duration.sum" in next(iter(launches.values())):
        rec["ncu_us_per_launch"] = round(sum(m["gpu__time_duration.sum"] for m in launches.values())
                                         / len(launches) * 1e6, 2)
    if "lts__t_sector_hit_rate.pct" in next(iter(launches.values())):
        rec["l2_sector_hit_rate_pct"] = round(sum(m["lts__t_sector_hit_rate.pct"]
                                                  for m in launches.values()) / len(launches), 2)
    data = _load_traffic()
    data[f"{args.ingest_kernel}:{args.workload}"] = rec
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps(rec))


# ------------------------------------------------------------ CPU baseline
def _oracle_tasks(w):
    """One oracle task per sequence: its q row and compact K/V pools."""
    import numpy as np
    from paged_kv_cache_416_b200.workloads import raw
    ts = []
    bs = w.block_size
    for s in range(w.num_seqs):
        nb = -(-int(w.context_lens[s]) // bs)
        ids = w.block_tables[s, :nb].astype(np.int64)
        ts.append((raw(w.q[s:s + 1]), w.q_dtype, raw(w.k_pool)[ids], raw(w.v_pool)[ids],
                   w.cache_dtype, np.arange(nb)[None], w.context_lens[s:s + 1], w.scale,
                   w.num_kv_heads, w.k_scale, w.v_scale))
    return ts


def oracle_rate(name: str, seed, target_seconds: float, pool):
    """Time the oracle (as it stands) on a bounded sample of sequences of the
    workload on the host's cores (`pool`: an oracle.parallel.OraclePool).
    Returns a cpu_baseline dict (GB/s of KV read, seq-tokens/s, the sample,
    cores, CPU model, seconds)."""
    from oracle.parallel import cpu_model
    from paged_kv_cache_416_b200 import workloads as W

    def sample(n):
        w = W.make(name, seed=seed, device="cpu", **_sample_kw(name, n))
        return w, _oracle_tasks(w)

    # calibrate on one sequence per worker, then size the sample
    workers = pool.workers
    w, ts = sample(workers)
    _, wall = pool.run(ts)
    rounds = max(1, int(target_seconds / max(wall, 1e-3)))
    n = min(workers * rounds, _full_seqs(name))
    if n > w.num_seqs:
        w, ts = sample(n)
        _, wall = pool.run(ts)
    desc = (f"oracle (numpy fp64) decode of {w.num_seqs} of the workload's {_full_seqs(name)} "
            f"sequences (same shapes; lengths from the same generator), {workers} spawned "
            f"workers, 1 BLAS thread each")
    return {"value": round(w.kv_bytes / wall / 1e9, 4), "unit": "GB/s", "cores": workers,
            "kind": "oracle", "sample": desc, "cpu_model": cpu_model(),
            "seq_tokens_per_s": round(w.seq_tokens / wall, 1), "seconds": round(wall, 2)}


def workload_seed(name: str, seed=None) -> int:
    """The seed a run uses: --seed if given, else the workload's own."""
    from paged_kv_cache_416_b200 import workloads as W
    return W.default_seed(name) if seed is None else int(seed)


def _full_seqs(name):
    return {"llama70b_gqa": 256, "llama13b_mha": 64, "fp8_longtail_bs16": 128,
            "fp8_longtail_bs32": 128, "shared_prefix_tails": 128, "shared_prefix_fork": 128,
            "tiny": 4, "e4m3_uniform": 128}[name]


def _sample_kw(name, n):
    if name in ("llama70b_gqa", "llama13b_mha", "fp8_longtail_bs16", "fp8_longtail_bs32",
                "e4m3_uniform"):
        return {"num_seqs": n}
    if name.startswith("shared_prefix"):
        return {"prompts": max(1, n // 4)}
    return {}


# ----------------------------------------------------------------- our arm
def run_ours(args, rank, local, world):
    import numpy as np
    import torch

    from paged_kv_cache_416_b200 import build as _build
    _build.build()
    from paged_kv_cache_416_b200 import pagedattn as pa
    from paged_kv_cache_416_b200 import workloads as W

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    kw = _sample_kw(args.workload, args.num_seqs) if args.num_seqs else {}
    w = W.make(args.workload, seed=workload_seed(args.workload, args.seed) + rank, device=device, **kw)
    stream = torch.cuda.current_stream()
    kp, vp = w.k_pool, w.v_pool
    q = w.q.contiguous()
    new_k, new_v = w.new_k.contiguous(), w.new_v.contiguous()
    slots = torch.from_numpy(w.slot_mapping).to(device)
    tables = torch.from_numpy(w.block_tables).to(device)
    lens = torch.from_numpy(w.context_lens).to(device)
    pairs = torch.from_numpy(w.cow_pairs).to(device)
    out = torch.empty_like(q)
    split = pa.decode_split_tokens(w.num_seqs, w.num_kv_heads, w.block_size, w.max_context_len)
    ws = torch.empty(max(256, pa.decode_workspace_size(
        w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.max_context_len)),
        dtype=torch.uint8, device=device)
    launches_per_step = (1 if len(w.cow_pairs) else 0) + 1 + 2 + (1 if split < w.max_context_len else 0)

    def step(dec_events=None):
        if len(w.cow_pairs):
            pa.copy_blocks(kp, vp, pairs)
        pa.write_kv(new_k, new_v, slots, kp, vp, w.k_scale, w.v_scale)
        if dec_events is not None:
            dec_events[0].record(stream)
        pa.decode(q, kp, vp, tables, lens, w.scale, w.max_context_len, k_scale=w.k_scale,
                  v_scale=w.v_scale, out=out, workspace=ws)
        if dec_events is not None:
            dec_events[1].record(stream)

    # correctness of the run itself: no device-side error
    step()
    pa.sync_status()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world, device)
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for i in range(K):
        step(dec_ev[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    barrier(world, device)
    pa.sync_status()
    sec = t0.elapsed_time(t1) / 1e3
    dec_ms = [a.elapsed_time(b) for a, b in dec_ev]
    max_sec = reduce_max(sec, world, device)
    value, tok_s = aggregate(w.kv_bytes, w.seq_tokens, K, max_sec, world, device)

    # ---- end to end through the public API with host buffers
    E = args.e2e_steps or K
    host_in = {n: t.detach().cpu().pin_memory() for n, t in
               (("q", q), ("new_k", new_k), ("new_v", new_v), ("slots", slots),
                ("tables", tables), ("lens", lens), ("pairs", pairs))}
    dev_in = {n: torch.empty_like(t, device=device) for n, t in host_in.items()}
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for n, t in host_in.items() if n != "pairs" or len(w.cow_pairs))
    d2h = out.numel() * out.element_size()

    def e2e_step():
        for n, t in host_in.items():
            if n == "pairs" and not len(w.cow_pairs):
                continue
            dev_in[n].copy_(t, non_blocking=True)
        if len(w.cow_pairs):
            pa.copy_blocks(kp, vp, dev_in["pairs"])
        pa.write_kv(dev_in["new_k"], dev_in["new_v"], dev_in["slots"], kp, vp, w.k_scale, w.v_scale)
        pa.decode(dev_in["q"], kp, vp, dev_in["tables"], dev_in["lens"], w.scale, w.max_context_len,
                  k_scale=w.k_scale, v_scale=w.v_scale, out=out, workspace=ws)
        out_host.copy_(out, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world, device)
    pa.sync_status()
    serial_sec = reduce_max(e0.elapsed_time(e1) / 1e3, world, device)
    serial_value, _ = aggregate(w.kv_bytes, w.seq_tokens, E, serial_sec, world, device)

    # the same steps through DecodePipeline: each step's inputs still come in
    # from pinned host memory and its output goes back every step, but on two
    # copy streams that overlap them with the neighbouring steps' device work
    from paged_kv_cache_416_b200.pipeline import DecodePipeline
    pipe = DecodePipeline(kp, vp, w.scale, w.max_context_len, w.k_scale, w.v_scale, workspace=ws)
    host_pipe = {n: t for n, t in host_in.items() if n != "pairs" or len(w.cow_pairs)}
    outs_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    for i in range(max(3, args.warmup)):
        pipe.submit(host_pipe, outs_host[i % 2])
    torch.cuda.synchronize()
    barrier(world, device)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    pipe.start_after(e2)
    for i in range(E):
        pipe.submit(host_pipe, outs_host[i % 2])
    pipe.drain(stream)
    e3.record(stream)
    torch.cuda.synchronize()
    barrier(world, device)
    pa.sync_status()
    e2e_sec = reduce_max(e2.elapsed_time(e3) / 1e3, world, device)
    e2e_value, _ = aggregate(w.kv_bytes, w.seq_tokens, E, e2e_sec, world, device)

    peak, peak_kind = measured_peaks()
    dec_mean_s = float(np.mean(dec_ms)) / 1e3
    achieved = w.kv_bytes / dec_mean_s / 1e9
    traffic, traffic_rec = profiled_traffic(w.name)

    configs = None
    if not args.no_configs and world == 1 and args.num_seqs is None:
        configs = measure_configs(args, pa, W, device, w, dec_ms, peak, peak_kind)

    if rank != 0:
        return None
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        from oracle.parallel import OraclePool, host_cores
        with OraclePool(host_cores()) as pool:
            cpu = oracle_rate(args.workload, args.seed, args.cpu_seconds, pool)
            for name, c in (configs or {}).items():
                c["cpu_baseline"] = oracle_rate(name, None, args.config_cpu_seconds, pool)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(max_sec / K * 1e3, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"f16": "f16", "bf16": "bf16", "e4m3": "e4m3"}[w.cache_dtype],
        "data": "synthetic",
        "config": {
            "workload": w.name, "num_seqs": w.num_seqs, "context_lens": _lens_desc(w),
            "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "block_size": w.block_size, "cache_dtype": w.cache_dtype,
            "num_blocks": w.num_blocks, "split_tokens": split,
            "kv_bytes_per_step": w.kv_bytes, "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2: {w.kv_bytes / 2**30:.2f} GiB of K/V streamed per step "
                  f"vs 126 MB L2; no flush",
        },
        "seq_tokens_per_s": round(tok_s, 1),
        "pct_of_8tbs": round(100 * value / NOMINAL_HBM_GBS, 2),
        "roofline": {
            "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "traffic_source": _traffic_note(traffic_rec, traffic),
            "kernel": "pa_decode (plan_kernel + decode_kernel)",
            "algorithmic_bytes_per_launch": w.kv_bytes, "peak_kind": peak_kind,
            "mean_launch_us": round(dec_mean_s * 1e6, 2),
        },
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_sec / E * 1e3, 4),
                "how": "DecodePipeline: pinned host inputs in and the output out every step, "
                       "on two copy streams overlapped with the neighbouring steps' kernels"},
        "e2e_serial": {"value": round(serial_value, 2), "unit": "GB/s",
                       "ms_per_step": round(serial_sec / E * 1e3, 4),
                       "how": "the same copies and kernels in one stream, one step after another"},
        "gpu_launches": launches_per_step * K,
        "clocks": clocks.summary(),
    }
    if configs is not None:
        line["configs"] = configs
    return line


def _traffic_note(rec, traffic):
    if rec is None:
        return "no ncu capture recorded for this workload"
    if traffic is None:
        return "the kernel changed since its capture: traffic not counted"
    return (f"ncu capture of {rec['captured_num_seqs']} of {rec['full_num_seqs']} sequences "
            f"({rec['launches']} launch(es)) scaled x{rec['scale_to_full']:.4g} by the K/V bytes; "
            f"profiles/decode_traffic.json")


def _stats_us(xs):
    import numpy as np
    a = np.asarray(xs, dtype=np.float64)
    return {"median": round(float(np.median(a)), 2), "min": round(float(a.min()), 2),
            "mean": round(float(a.mean()), 2)}


def config_memory(w, name):
    """Closed-form memory figures of one configuration's batch: slots left
    unused by paging (the unfilled tail of each last block) against a
    contiguous reservation of the generator's length bound per sequence, and
    for the shared-prefix batch the physical blocks in use against the blocks
    the same sequences would hold without sharing."""
    import numpy as np
    bs = w.block_size
    lens = w.context_lens.astype(np.int64)
    nb = -(-lens // bs)
    alloc_slots = int(nb.sum()) * bs
    used = int(lens.sum())
    R = RESERVATION_TOKENS[name]
    out = {
        "paged_unused_slots": alloc_slots - used,
        "paged_waste_pct": round(100.0 * (alloc_slots - used) / alloc_slots, 3),
        "reservation_tokens_per_seq": R,
        "reserved_unused_slots": len(lens) * R - used,
        "reserved_waste_pct": round(100.0 * (len(lens) * R - used) / (len(lens) * R), 2),
    }
    if name.startswith("shared_prefix"):
        phys = set()
        for s in range(w.num_seqs):
            phys.update(int(b) for b in w.block_tables[s, :int(nb[s])])
        out.update({"blocks_unshared": int(nb.sum()), "blocks_shared": len(phys),
                    "memory_saved_pct": round(100.0 * (1 - len(phys) / int(nb.sum())), 2)})
    return out


def measure_configs(args, pa, W, device, head_w, head_dec_ms, peak, peak_kind):
    """Every benchmark configuration, each on its own seeded batch: pa_decode
    (plan + attention kernel) and the whole step (copy-on-write copies, cache
    write, decode) timed per iteration by CUDA events on the launching stream,
    median / min / mean over the iterations.  A configuration whose distinct
    K/V bytes are under 4x the L2 size gets L2 flushed before every timed
    iteration, outside the events: a 4x-L2 buffer is written, then a second
    one read, so the L2 holds none of the inputs and no dirty lines whose
    write-back would land inside the timed kernel."""
    import numpy as np
    import torch
    l2 = int(torch.cuda.get_device_properties(device).L2_cache_size)
    flush_buf = torch.empty(4 * l2, dtype=torch.uint8, device=device)
    flush_rd = torch.zeros(4 * l2, dtype=torch.uint8, device=device)

    def flush_l2():
        flush_buf.zero_()
        flush_rd.sum(dtype=torch.int64)
    stream = torch.cuda.current_stream()
    iters = max(3, args.config_iters)
    results = {}
    for name in CONFIG_WORKLOADS:
        own = name != head_w.name
        w = W.make(name, device=device) if own else head_w
        kp, vp = w.k_pool, w.v_pool
        q = w.q.contiguous()
        nk, nv = w.new_k.contiguous(), w.new_v.contiguous()
        slots = torch.from_numpy(w.slot_mapping).to(device)
        tables = torch.from_numpy(w.block_tables).to(device)
        lens = torch.from_numpy(w.context_lens).to(device)
        pairs = torch.from_numpy(w.cow_pairs).to(device) if len(w.cow_pairs) else None
        out = torch.empty_like(q)
        ws = torch.empty(max(256, pa.decode_workspace_size(
            w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
            w.max_context_len)), dtype=torch.uint8, device=device)
        unique = unique_kv_bytes(w)
        flush = unique < 4 * l2

        def step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            if pairs is not None:
                pa.copy_blocks(kp, vp, pairs)
            pa.write_kv(nk, nv, slots, kp, vp, w.k_scale, w.v_scale)
            if ev is not None:
                ev[1].record(stream)
            pa.decode(q, kp, vp, tables, lens, w.scale, w.max_context_len, k_scale=w.k_scale,
                      v_scale=w.v_scale, out=out, workspace=ws)
            if ev is not None:
                ev[2].record(stream)

        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
        pa.sync_status()
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(iters)]
        clocks = ClockSampler(device.index)
        clocks.start()
        for i in range(iters):
            if flush:
                flush_l2()
            step(evs[i])
        torch.cuda.synchronize()
        clocks.stop()
        pa.sync_status()
        dec = [b.elapsed_time(c) * 1e3 for a, b, c in evs]
        stp = [a.elapsed_time(c) * 1e3 for a, b, c in evs]
        dstat, sstat = _stats_us(dec), _stats_us(stp)
        med_s = dstat["median"] / 1e6
        gbs = w.kv_bytes / med_s / 1e9
        traffic, rec = profiled_traffic(name)
        r = {
            "num_seqs": w.num_seqs, "heads": f"{w.num_q_heads}/{w.num_kv_heads}",
            "head_dim": w.head_dim, "block_size": w.block_size, "cache_dtype": w.cache_dtype,
            "q_dtype": w.q_dtype, "context_lens": _lens_desc(w), "cow_pairs": int(len(w.cow_pairs)),
            "kv_bytes": w.kv_bytes, "unique_kv_bytes": unique,
            "pa_decode_us": dstat, "step_us": sstat, "iterations": iters,
            "gbs": round(gbs, 1), "pct_of_8tbs": round(100 * gbs / NOMINAL_HBM_GBS, 2),
            "seq_tokens_per_s": round(w.seq_tokens / med_s, 1),
            "seq_tokens_per_s_step": round(w.seq_tokens / (sstat["median"] / 1e6), 1),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "peak_kind": peak_kind,
                         "bytes": "algorithmic (logical) K/V bytes, median pa_decode time",
                         "traffic": traffic, "traffic_source": _traffic_note(rec, traffic)},
            "l2": (f"flushed before every timed iteration ({4 * l2 / 2**20:.0f} MiB written, "
                   f"then another {4 * l2 / 2**20:.0f} MiB read): "
                   f"{unique / 2**20:.1f} MiB of distinct K/V < 4x L2" if flush else
                   f"no flush: {unique / 2**30:.2f} GiB of distinct K/V >= 4x L2"),
            "memory": config_memory(w, name),
            "clocks": clocks.summary(),
        }
        if unique != w.kv_bytes:
            ug = unique / med_s / 1e9
            r["gbs_unique"] = round(ug, 1)
            r["roofline_unique"] = {"achieved": round(ug, 1), "frac": round(ug / peak, 4)}
        if "group_start" in w.meta:
            gs = torch.from_numpy(w.meta["group_start"]).to(device)
            gq = torch.from_numpy(w.meta["group_seqs"]).to(device)
            sws = torch.empty(max(256, pa.shared_prefix_workspace_size(
                w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                w.max_context_len)), dtype=torch.uint8, device=device)
            out2 = torch.empty_like(q)

            def shared():
                pa.decode_shared_prefix(q, kp, vp, tables, lens, gs, gq, w.scale,
                                        w.max_context_len, out=out2, workspace=sws)

            for _ in range(3):
                shared()
            sev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(iters)]
            for i in range(iters):
                if flush:
                    flush_l2()
                sev[i][0].record(stream)
                shared()
                sev[i][1].record(stream)
            torch.cuda.synchronize()
            pa.sync_status()
            sp = _stats_us([a.elapsed_time(b) * 1e3 for a, b in sev])
            sp_s = sp["median"] / 1e6
            r["pa_decode_shared_prefix"] = {
                "us": sp, "gbs_logical": round(w.kv_bytes / sp_s / 1e9, 1),
                "gbs_unique": round(unique / sp_s / 1e9, 1),
                "frac_unique": round(unique / sp_s / 1e9 / peak, 4),
                "speedup_vs_pa_decode": round(dstat["median"] / sp["median"], 3)}
            del out2, sws
        results[name] = r
        del kp, vp, q, out, ws
        if own:
            del w
        torch.cuda.empty_cache()
    del flush_buf, flush_rd
    torch.cuda.empty_cache()
    return results


def _lens_desc(w):
    import numpy as np
    c = w.context_lens
    if (c == c[0]).all():
        return f"all {int(c[0])}"
    return f"min {int(c.min())} median {int(np.median(c))} max {int(c.max())} sum {int(c.sum())}"


# ---------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host's cores, on a bounded sample
    of the workload per step."""
    if rank != 0:
        return None
    from oracle.parallel import host_cores, run_decode_tasks
    import numpy as np
    from paged_kv_cache_416_b200 import workloads as W
    from paged_kv_cache_416_b200.workloads import raw

    cores = host_cores()
    n = min(_full_seqs(args.workload), cores)  # one sequence per core per step
    w = W.make(args.workload, seed=args.seed, device="cpu", **_sample_kw(args.workload, n))
    bs = w.block_size
    tasks = []
    for s in range(w.num_seqs):
        nb = -(-int(w.context_lens[s]) // bs)
        ids = w.block_tables[s, :nb].astype(np.int64)
        tasks.append((raw(w.q[s:s + 1]), w.q_dtype, raw(w.k_pool)[ids], raw(w.v_pool)[ids],
                      w.cache_dtype, np.arange(nb)[None], w.context_lens[s:s + 1], w.scale,
                      w.num_kv_heads, w.k_scale, w.v_scale))
    for _ in range(args.warmup):
        run_decode_tasks(tasks[:1], 1)
    total = 0.0
    for _ in range(args.steps):
        _, wall = run_decode_tasks(tasks, cores)
        total += wall
    gbs = w.kv_bytes * args.steps / total / 1e9
    desc = (f"oracle (numpy fp64) decode of {w.num_seqs} of the workload's "
            f"{_full_seqs(args.workload)} sequences per step, {cores} spawned workers")
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "sample_seqs": w.num_seqs},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ------------------------------------------------------- companion operations
def _events_time(fn, iters, warmup=3):
    """Mean seconds per call of fn() on the current stream, by CUDA events."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / iters


def run_swap(args):
    """pa_swap_blocks: move 2048 blocks of the Llama-3-70B-shaped pool (bs 16,
    8 kv heads, D 128, bf16: 64 KiB of K+V per block) from the device pool to
    pinned host memory and back, scattered ids.  Roofline: one large pinned
    cudaMemcpy of the same bytes in the same direction, timed in this run."""
    import torch
    from paged_kv_cache_416_b200 import build as _build
    _build.build()
    from paged_kv_cache_416_b200 import pagedattn as pa
    torch.cuda.set_device(0)
    nb, shape = 2048, (16, 8, 128)
    g = torch.Generator(device="cuda").manual_seed(workload_seed("llama70b_gqa", args.seed))
    dev_k = torch.randn((8192,) + shape, generator=g, device="cuda").to(torch.bfloat16)
    dev_v = torch.randn((8192,) + shape, generator=g, device="cuda").to(torch.bfloat16)
    host_k = torch.empty((nb,) + shape, dtype=torch.bfloat16).pin_memory()
    host_v = torch.empty((nb,) + shape, dtype=torch.bfloat16).pin_memory()
    gc = torch.Generator().manual_seed(workload_seed("llama70b_gqa", args.seed))
    src = torch.randperm(8192, generator=gc)[:nb]
    dst = torch.randperm(nb, generator=gc)
    out_pairs = torch.stack([src, dst], 1).to(torch.int64).cuda()
    in_pairs = torch.stack([dst, src], 1).to(torch.int64).cuda()
    moved = 2 * nb * 16 * 8 * 128 * 2
    iters = max(3, min(args.steps, 50))
    t_out = _events_time(lambda: pa.swap_blocks(dev_k, dev_v, host_k, host_v, out_pairs), iters)
    t_in = _events_time(lambda: pa.swap_blocks(host_k, host_v, dev_k, dev_v, in_pairs), iters)
    pa.sync_status()
    flat_dev = torch.empty(moved, dtype=torch.uint8, device="cuda")
    flat_host = torch.empty(moved, dtype=torch.uint8).pin_memory()
    t_d2h = _events_time(lambda: flat_host.copy_(flat_dev, non_blocking=True), iters)
    t_h2d = _events_time(lambda: flat_dev.copy_(flat_host, non_blocking=True), iters)
    out_gbs, in_gbs = moved / t_out / 1e9, moved / t_in / 1e9
    return {
        "metric": "block swap GB/s (device pool <-> pinned host)", "op": "swap",
        "value": round(min(out_gbs, in_gbs), 2), "unit": "GB/s", "n_gpus": 1,
        "steps": iters, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "2048 scattered blocks of 16x8x128 bf16 (K and V), 256 MiB moved",
                   "bytes_per_call": moved},
        "swap_out_gbs": round(out_gbs, 2), "swap_in_gbs": round(in_gbs, 2),
        "swap_out_us": round(t_out * 1e6, 1), "swap_in_us": round(t_in * 1e6, 1),
        "roofline": {"bound": "host link", "achieved": round(min(out_gbs, in_gbs), 2),
                     "peak": round(min(moved / t_d2h, moved / t_h2d) / 1e9, 2), "unit": "GB/s",
                     "frac": round(min(out_gbs / (moved / t_d2h / 1e9), in_gbs / (moved / t_h2d / 1e9)), 4),
                     "peak_kind": "one pinned cudaMemcpy of the same bytes, measured in this run",
                     "memcpy_d2h_gbs": round(moved / t_d2h / 1e9, 2),
                     "memcpy_h2d_gbs": round(moved / t_h2d / 1e9, 2)},
        "gpu_launches": 2 * iters,
    }


def run_hash(args):
    """pa_hash_blocks over 256 sequences x 4096 token ids (bs 16, 65,536
    full blocks).  The bound is latency, not a unit's throughput: a
    sequence's block hashes form a chain, each block's FNV-1a over its
    parent's hash and its own inner hash being 16 dependent byte steps, so
    one call is at least 256 x 16 = 4096 dependent steps long.  The line
    reports the time per dependent step (the call's time over the chain
    length) in ns and in SM clock cycles at the sampled clock."""
    import torch
    from paged_kv_cache_416_b200 import build as _build
    _build.build()
    from paged_kv_cache_416_b200 import pagedattn as pa
    torch.cuda.set_device(0)
    B, L, bs = 256, 4096, 16
    g = torch.Generator(device="cuda").manual_seed(workload_seed("llama70b_gqa", args.seed))
    toks = torch.randint(0, 128256, (B, L), generator=g, device="cuda", dtype=torch.int32)
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    out = torch.empty((B, L // bs), dtype=torch.int64, device="cuda")
    iters = max(3, min(args.steps, 50))
    clocks = ClockSampler(0)
    clocks.start()
    t = _events_time(lambda: pa.hash_blocks(toks, lens, bs, out=out), iters)
    clocks.stop()
    pa.sync_status()
    tps = B * L / t
    chain = (L // bs) * 16               # dependent FNV byte steps of one sequence's chain
    ck = clocks.summary()
    mhz = ck.get("sm_mhz") or clocks.max_mhz or 1965.0
    ns_step = t * 1e9 / chain
    return {
        "metric": "prefix-cache block hashing, token ids hashed per second", "op": "hash",
        "value": round(tps, 1), "unit": "tokens/s", "n_gpus": 1, "steps": iters,
        "higher_is_better": True, "dtype": "int32", "data": "synthetic",
        "config": {"workload": "256 sequences x 4096 token ids, block_size 16", "blocks": B * L // bs},
        "us_per_call": round(t * 1e6, 2),
        "roofline": {"bound": "latency", "achieved": round(ns_step, 3),
                     "unit": "ns per dependent step of the per-sequence hash chain",
                     "peak": None, "frac": None, "chain_steps": chain,
                     "cycles_per_step": round(ns_step * mhz / 1e3, 2), "sm_mhz": mhz,
                     "note": "each sequence's 256 block hashes form a serial chain of 16 "
                             "dependent FNV-1a byte steps per block; the call takes this many "
                             "cycles per step, the inner hashes of the blocks included"},
        "clocks": ck,
        "gpu_launches": iters,
    }


def run_prefill(args):
    """pa_prefill: full prefill of 8 sequences x 4096 tokens on the
    Llama-3-70B-shaped layer (64/8 heads, D 128, bf16, bs 16), causal.
    Roofline: tensor -- causal attention flops (4 * D * Hq * sum of keys seen
    per query) against the dense bf16 peak (measured, else a 1590 TFLOP/s fallback)."""
    import torch
    from paged_kv_cache_416_b200 import build as _build
    _build.build()
    from paged_kv_cache_416_b200 import pagedattn as pa
    from paged_kv_cache_416_b200 import workloads as W
    torch.cuda.set_device(0)
    n = 4096
    pw = W.prefill(seed=workload_seed("llama70b_gqa", args.seed), device="cuda", ctxs=(n,) * 8, nqs=(n,) * 8, hq=64, hkv=8,
                   bs=16, dtype="bf16")
    b = pw.base
    q = pw.q
    bt = torch.from_numpy(b.block_tables).cuda()
    cl = torch.from_numpy(b.context_lens).cuda()
    qs = torch.from_numpy(pw.query_start).cuda()
    out = torch.empty_like(q)
    iters = max(3, min(args.steps, 20))
    t = _events_time(lambda: pa.prefill(q, b.k_pool, b.v_pool, bt, cl, qs, b.scale,
                                        pw.max_query_len, b.max_context_len, out=out), iters)
    pa.sync_status()
    tflops = pw.flops / t / 1e12
    peak, peak_kind = 1590.0, "fallback dense bf16 (burst)"
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            peak, peak_kind = float(json.load(f)["bf16_tflops"]), "measured dense bf16 (burst)"

    return {
        "metric": "paged prefill attention TFLOP/s (causal)", "op": "prefill",
        "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": 1, "steps": iters,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "8 sequences x 4096 new tokens, 64/8 heads, D 128, bf16, bs 16",
                   "flops_per_call": pw.flops},
        "ms_per_call": round(t * 1e3, 3),
        "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                     "peak_kind": peak_kind},
        "gpu_launches": iters,
    }


def unique_kv_bytes(w) -> int:
    """K+V bytes of the distinct physical blocks the step reads (each block
    counted up to the furthest token any sequence reads in it)."""
    import numpy as np
    bs = w.block_size
    used = {}
    for s in range(w.num_seqs):
        n = int(w.context_lens[s])
        for j in range(-(-n // bs)):
            b = int(w.block_tables[s, j])
            used[b] = max(used.get(b, 0), min(bs, n - j * bs))
    tokens = int(np.sum(list(used.values())))
    return tokens * w.num_kv_heads * w.head_dim * 2 * {"e4m3": 1}.get(w.cache_dtype, 2)


def run_shared_prefix(args):
    """pa_decode_shared_prefix on the shared-prefix workload (32 prompts x 4
    samples, 32/8 heads, D 128, bf16, bs 16, 1024 + r shared tokens, tails
    U{0..512}): every prompt's blocks are read once for its four samples.
    Timed beside pa_decode on the same inputs.  Roofline: HBM, on the unique
    bytes (the distinct blocks read), against the measured copy bandwidth."""
    import torch
    from paged_kv_cache_416_b200 import build as _build
    _build.build()
    from paged_kv_cache_416_b200 import pagedattn as pa
    from paged_kv_cache_416_b200 import workloads as W
    torch.cuda.set_device(0)
    w = W.make("shared_prefix_tails", seed=args.seed, device="cuda")  # None: its own seed
    kp, vp = w.k_pool, w.v_pool
    pa.write_kv(w.new_k, w.new_v, torch.from_numpy(w.slot_mapping).cuda(), kp, vp)
    q = w.q.contiguous()
    bt = torch.from_numpy(w.block_tables).cuda()
    cl = torch.from_numpy(w.context_lens).cuda()
    gs = torch.from_numpy(w.meta["group_start"]).cuda()
    gq = torch.from_numpy(w.meta["group_seqs"]).cuda()
    out = torch.empty_like(q)
    ws = pa.workspace_for(q.device, pa.shared_prefix_workspace_size(
        w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.max_context_len))
    iters = max(20, min(args.steps, 200))
    t_shared = _events_time(lambda: pa.decode_shared_prefix(
        q, kp, vp, bt, cl, gs, gq, w.scale, w.max_context_len, out=out, workspace=ws), iters)
    t_plain = _events_time(lambda: pa.decode(q, kp, vp, bt, cl, w.scale, w.max_context_len,
                                             out=out), iters)
    pa.sync_status()
    logical = w.kv_bytes
    unique = unique_kv_bytes(w)
    peak, peak_kind = measured_peaks()
    ach = unique / t_shared / 1e9
    return {
        "metric": "shared-prefix decode: KV-read GB/s (logical bytes)", "op": "shared_prefix",
        "value": round(logical / t_shared / 1e9, 1), "unit": "GB/s", "n_gpus": 1,
        "steps": iters, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "shared_prefix_tails: 32 prompts x 4 samples, 32/8 heads, D 128, "
                               "bf16, bs 16, 1024 + r shared tokens, tails U{0..512}",
                   "logical_kv_bytes": logical, "unique_kv_bytes": unique},
        "us_per_call": round(t_shared * 1e6, 2),
        "plain_decode_us_per_call": round(t_plain * 1e6, 2),
        "speedup_vs_plain_decode": round(t_plain / t_shared, 3),
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(ach / peak, 4), "bytes": "unique",
                     "peak_kind": peak_kind},
        "gpu_launches": 4 * iters,
    }


def main(argv=None):
    args = parse_args(argv)
    if args.print_source_sha16:
        print(json.dumps({k: source_hash(k) for k in KERNEL_SOURCES}))
        return 0
    if args.ingest_ncu:
        ingest_ncu(args)
        return 0
    if args.warmup < 3:
        args.warmup = 3
    rank, local, world = dist_env()
    if args.impl == "reference":
        if world > 1:
            import torch.distributed as dist
            if rank != 0:
                return 0
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    if args.op != "decode":
        if rank != 0:
            return 0
        line = {"swap": run_swap, "hash": run_hash, "prefill": run_prefill,
                "shared_prefix": run_shared_prefix}[args.op](args)
        print(json.dumps(line), flush=True)
        return 0
    import torch
    if world > 1:
        torch.cuda.set_device(local)
    rank, local, world = dist_init("nccl")
    try:
        line = run_ours(args, rank, local, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
