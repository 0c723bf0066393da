"""Test harness: run one decode step through the CUDA library and through the
oracle on the same seeded inputs, and compare.

A step is: copy-on-write block copies (if any) -> write of the new tokens ->
decode over every sequence.  The oracle works on host copies of the raw
input words; nothing it receives comes from the CUDA path.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_416_b200.workloads import Workload, raw

ATOL, RTOL = 2e-3, 1e-2  # |gpu - ref| <= ATOL + RTOL * |ref|, fp16/bf16/e4m3 caches


def assert_attention_close(got: np.ndarray, ref: np.ndarray, what: str = "") -> None:
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = ~(err <= bound)  # NaN fails too
    if bad.any():
        idx = np.unravel_index(np.argmax(np.where(np.isnan(err), np.inf, err - bound)), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outputs outside |err| <= {ATOL} + {RTOL}|ref|; "
            f"worst at {idx}: got {got[idx]!r} ref {ref[idx]!r}")


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def gpu_step(pa, w: Workload, split_tokens: int = 0, device="cuda"):
    """Run the step on the GPU; returns (out, k_pool, v_pool) device tensors."""
    kp = w.k_pool.to(device).clone()
    vp = w.v_pool.to(device).clone()
    if len(w.cow_pairs):
        pa.copy_blocks(kp, vp, torch.from_numpy(w.cow_pairs).to(device))
    pa.write_kv(w.new_k.to(device).contiguous(), w.new_v.to(device).contiguous(),
                torch.from_numpy(w.slot_mapping).to(device), kp, vp, w.k_scale, w.v_scale)
    out = pa.decode(w.q.to(device).contiguous(), kp, vp,
                    torch.from_numpy(w.block_tables).to(device),
                    torch.from_numpy(w.context_lens).to(device), w.scale, w.max_context_len,
                    k_scale=w.k_scale, v_scale=w.v_scale, split_tokens=split_tokens)
    pa.sync_status()
    return out, kp, vp


def oracle_step(w: Workload, seqs=None):
    """Run the step in the oracle; returns (out fp64, k_pool raw, v_pool raw)."""
    kp = raw(w.k_pool).copy()
    vp = raw(w.v_pool).copy()
    if len(w.cow_pairs):
        oracle.copy_blocks(kp, vp, w.cow_pairs)
    oracle.write_kv(raw(w.new_k), raw(w.new_v), w.q_dtype, w.slot_mapping, kp, vp,
                    w.cache_dtype, w.k_scale, w.v_scale)
    out = oracle.decode(raw(w.q), w.q_dtype, kp, vp, w.cache_dtype, w.block_tables,
                        w.context_lens, w.scale, w.num_kv_heads, w.k_scale, w.v_scale, seqs=seqs)
    return out, kp, vp


def compact_oracle_step(w: Workload, seqs):
    """Oracle step for the listed sequences only, on a small pool holding just
    their blocks (pulled from wherever the workload's pools live).  The
    blocks are renumbered 0..n-1 in the order first named; results do not
    depend on physical ids.  Returns fp64 [len(seqs), Hq, D].  Workloads with
    copy-on-write pairs are not supported here."""
    assert not len(w.cow_pairs)
    bs = w.block_size
    ids, remap = [], {}
    rows = []
    for s in seqs:
        n = int(w.context_lens[s])
        nb = -(-n // bs)
        row = []
        for b in w.block_tables[s, :nb]:
            b = int(b)
            if b not in remap:
                remap[b] = len(ids)
                ids.append(b)
            row.append(remap[b])
        rows.append(row)
    idx = torch.tensor(ids, dtype=torch.int64, device=w.k_pool.device)
    kp = raw(w.k_pool.index_select(0, idx)) if ids else raw(w.k_pool[:1])
    vp = raw(w.v_pool.index_select(0, idx)) if ids else raw(w.v_pool[:1])
    width = max(1, max(len(r) for r in rows))
    tables = np.full((len(seqs), width), -1, dtype=np.int64)
    for i, r in enumerate(rows):
        tables[i, :len(r)] = r
    # the new tokens of these sequences, with slots moved to the renumbered blocks
    sel = [t for t, sl in enumerate(w.slot_mapping) if sl >= 0 and int(sl) // bs in remap]
    slots = np.array([remap[int(w.slot_mapping[t]) // bs] * bs + int(w.slot_mapping[t]) % bs
                      for t in sel], dtype=np.int64)
    if sel:
        ti = torch.tensor(sel, dtype=torch.int64, device=w.new_k.device)
        oracle.write_kv(raw(w.new_k.index_select(0, ti)), raw(w.new_v.index_select(0, ti)),
                        w.q_dtype, slots, kp, vp, w.cache_dtype, w.k_scale, w.v_scale)
    qi = torch.tensor(list(seqs), dtype=torch.int64, device=w.q.device)
    out = oracle.decode(raw(w.q.index_select(0, qi)), w.q_dtype, kp, vp, w.cache_dtype, tables,
                        w.context_lens[list(seqs)], w.scale, w.num_kv_heads, w.k_scale, w.v_scale)
    return out
