"""The decode kernel's bounded waits give up, report PA_ERR_TIMEOUT, and
leave the context usable.

A test build of the library (compiled into a temporary directory with
PA_TEST_STAGE_EXTRA_TX=16 and a 10 ms wait limit) makes every stage barrier
of the decode kernel expect 16 bytes more than its two tile copies deliver.
Every copy is still a valid, in-bounds load that lands; only the stage never
completes, so each wait runs out after 10 ms, the warp records the timeout,
stops issuing and drains its ring with bounded waits.  The call must report
PA_ERR_TIMEOUT at pa_sync_status and leave the pools untouched; the library
build then decodes the same inputs normally in the same process.
"""

import ctypes

import numpy as np
import pytest
import torch

from harness import as_f64, assert_attention_close
from paged_kv_cache_416_b200 import build
from paged_kv_cache_416_b200 import workloads as W
from paged_kv_cache_416_b200.workloads import raw

pytestmark = pytest.mark.gpu


def test_decode_wait_timeout_is_reported_and_the_context_stays_usable(pa, tmp_path):
    path = build.build(out=tmp_path / "libpagedattn_stall.so",
                       extra_flags=["-DPA_TEST_STAGE_EXTRA_TX=16",
                                    "-DPA_WAIT_LIMIT_NS=10000000ull"])
    stall = pa.declare(ctypes.CDLL(str(path)))
    w = W.make("fp8_longtail_bs16", num_seqs=6, max_len=3000)
    dev = "cuda"
    q = w.q.to(dev).contiguous()
    kp, vp = w.k_pool.to(dev), w.v_pool.to(dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    k_before, v_before = raw(kp).copy(), raw(vp).copy()
    out = torch.zeros_like(q)
    split = 256  # several ranges per sequence: the merge path runs too
    ws = torch.empty(max(256, pa.decode_workspace_size(
        w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.max_context_len,
        split)), dtype=torch.uint8, device=dev)
    st = stall.pa_decode(pa._ptr(out), pa._ptr(q), pa._dtype(q), pa._ptr(kp), pa._ptr(vp),
                         pa._dtype(kp), pa._ptr(bt), bt.shape[1], pa._ptr(cl), w.max_context_len,
                         w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                         w.num_blocks, w.scale, w.k_scale, w.v_scale, split, pa._ptr(ws),
                         ws.numel(), pa._stream())
    assert st == 0
    assert stall.pa_sync_status(pa._stream()) == 10  # PA_ERR_TIMEOUT
    assert b"gave up waiting" in stall.pa_last_error()
    assert stall.pa_sync_status(pa._stream()) == 0   # the word was cleared
    assert np.array_equal(raw(kp), k_before) and np.array_equal(raw(vp), v_before)
    # the context is still usable: the library build decodes the same inputs
    got = pa.decode(q, kp, vp, bt, cl, w.scale, w.max_context_len, k_scale=w.k_scale,
                    v_scale=w.v_scale, split_tokens=split)
    pa.sync_status()
    ref = compact_oracle_step_without_write(w)
    assert_attention_close(as_f64(got), ref, "decode after a timed-out call")


def compact_oracle_step_without_write(w):
    """The oracle's decode of every sequence over the pools as given (this
    test writes no new token)."""
    import oracle
    return oracle.decode(raw(w.q), w.q_dtype, raw(w.k_pool), raw(w.v_pool), w.cache_dtype,
                         w.block_tables, w.context_lens, w.scale, w.num_kv_heads, w.k_scale,
                         w.v_scale)
