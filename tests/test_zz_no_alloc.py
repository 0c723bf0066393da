"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers may not call cudaMalloc: a plugin inside a host framework that
owns every device allocation and hands it only inputs and outputs, or a
serving loop whose device memory is budgeted up front.  For them the library
offers pa_decode_noalloc, which takes its scratch from an array reserved when
the library is loaded instead of a caller-provided workspace.

The GPU test calls it through the C ABI twice in a row (the second call finds
the first call's leftovers in the shared scratch) and checks each output
against pa_decode with a workspace, within the attention tolerance the other
tests use.  This file is collected last so that a run stopping at the first
failure has run every other test before it.
"""

import ctypes

import numpy as np
import pytest
import torch

from harness import ATOL, RTOL, assert_attention_close, as_f64
from paged_kv_cache_416_b200 import build


@pytest.fixture(scope="module")
def lib():
    build.build()
    from paged_kv_cache_416_b200 import pagedattn
    return pagedattn


def _noalloc(pa, out, w, q, kp, vp, bt, cl, split):
    return pa.pa_decode_noalloc(
        pa._ptr(out), pa._ptr(q), pa._dtype(q), pa._ptr(kp), pa._ptr(vp), pa._dtype(kp),
        pa._ptr(bt), bt.shape[1], pa._ptr(cl), w.max_context_len, w.num_seqs, w.num_q_heads,
        w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks, w.scale, w.k_scale, w.v_scale,
        split, pa._stream())


def test_noalloc_refuses_sizes_beyond_its_scratch(lib):
    # 4096 sequences of 32k tokens cut into 16-token ranges need far more than
    # the built-in scratch: refused on the host, before any launch
    need = lib.pa_decode_workspace_size(4096, 32, 8, 128, 16, 32768, 16)
    assert need > lib.NOALLOC_SCRATCH_BYTES
    st = lib.pa_decode_noalloc(None, None, 1, None, None, 1, None, 2048, None, 32768, 4096, 32, 8,
                               128, 16, 1 << 20, 0.1, 1.0, 1.0, 16, None)
    assert st == 9  # PA_ERR_WORKSPACE
    assert b"scratch" in lib.pa_last_error()


@pytest.mark.gpu
def test_noalloc_matches_decode_with_workspace_on_two_calls(lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_416_b200 import workloads as W
    pa = lib
    cases = [
        # split contexts: the scratch holds range offsets and partials
        (W.make("fp8_longtail_bs16", num_seqs=10, max_len=6000), 64),
        # one item per (sequence, kv head): only the counter and offsets
        (W.make("llama70b_gqa", num_seqs=4, context_len=700), 0),
    ]
    for w, split in cases:
        assert pa.decode_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                        w.block_size, w.max_context_len, split) <= pa.NOALLOC_SCRATCH_BYTES
    for call, (w, split) in enumerate(cases):  # two calls in a row
        dev = "cuda"
        q = w.q.to(dev).contiguous()
        kp, vp = w.k_pool.to(dev), w.v_pool.to(dev)
        bt = torch.from_numpy(w.block_tables).to(dev)
        cl = torch.from_numpy(w.context_lens).to(dev)
        ref = pa.decode(q, kp, vp, bt, cl, w.scale, w.max_context_len, k_scale=w.k_scale,
                        v_scale=w.v_scale, split_tokens=split)
        out = torch.full_like(q, float("nan"))
        pa.check(_noalloc(pa, out, w, q, kp, vp, bt, cl, split))
        pa.sync_status()
        assert_attention_close(as_f64(out), as_f64(ref), f"no-alloc call {call + 1}")
