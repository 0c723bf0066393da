"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers may not call cudaMalloc: a plugin inside a host framework that
owns every device allocation and hands it only inputs and outputs, or a
serving loop whose device memory is budgeted up front.  For them the library
offers pa_decode_noalloc, which takes its scratch from an array reserved when
the library is loaded instead of a caller-provided workspace.

The GPU test calls it through the C ABI twice in a row (the second call finds
the first call's leftovers in the shared scratch): once with split contexts
(range offsets and partials in the scratch) and once unsplit (only the work
counter and offsets).  Each output is checked against the fp64 oracle within
the attention tolerance the other tests use, and against pa_decode with a
caller workspace, which must give the same bits; the device memory in use
must not change across the two calls.  This file is collected last so that a
run stopping at the first failure has run every other test before it.
"""

import re

import pytest
import torch

from harness import as_f64, assert_attention_close, compact_oracle_step
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


def test_noalloc_scratch_size_comes_from_the_header(lib):
    with open(lib.HEADER_PATH) as f:
        m = re.search(r"#define\s+PA_DECODE_NOALLOC_SCRATCH_BYTES\s+\((\d+)u \* (\d+)u \* (\d+)u\)",
                      f.read())
    assert m is not None
    assert lib.NOALLOC_SCRATCH_BYTES == int(m.group(1)) * int(m.group(2)) * int(m.group(3))


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
def test_noalloc_matches_oracle_and_decode_on_two_calls(lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_416_b200 import workloads as W
    pa = lib
    cases = [
        # split contexts: the scratch holds range offsets and partials
        (W.make("fp8_longtail_bs16", num_seqs=10, max_len=6000), 64),
        # one item per (sequence, kv head): only the counter and offsets
        (W.make("llama70b_gqa", num_seqs=4, context_len=200), 0),
    ]
    w0, s0 = cases[0]
    assert pa.decode_split_tokens(w0.num_seqs, w0.num_kv_heads, w0.block_size,
                                  w0.max_context_len, s0) < w0.max_context_len
    w1, s1 = cases[1]
    assert pa.decode_split_tokens(w1.num_seqs, w1.num_kv_heads, w1.block_size,
                                  w1.max_context_len, s1) >= w1.max_context_len
    for w, split in cases:
        assert pa.decode_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                        w.block_size, w.max_context_len, split) <= pa.NOALLOC_SCRATCH_BYTES

    # every device tensor the test needs, and pa_decode's results with a
    # caller workspace, before the calls under test
    dev = "cuda"
    runs = []
    for w, split in cases:
        t = dict(q=w.q.to(dev).contiguous(), kp=w.k_pool.to(dev), vp=w.v_pool.to(dev),
                 bt=torch.from_numpy(w.block_tables).to(dev),
                 cl=torch.from_numpy(w.context_lens).to(dev))
        # the step's cache write first, as the oracle's step does
        pa.write_kv(w.new_k.to(dev).contiguous(), w.new_v.to(dev).contiguous(),
                    torch.from_numpy(w.slot_mapping).to(dev), t["kp"], t["vp"], w.k_scale,
                    w.v_scale)
        t["ref"] = pa.decode(t["q"], t["kp"], t["vp"], t["bt"], t["cl"], w.scale,
                             w.max_context_len, k_scale=w.k_scale, v_scale=w.v_scale,
                             split_tokens=split)
        t["out"] = torch.empty_like(t["q"])
        t["warm"] = torch.empty_like(t["q"])
        runs.append((w, split, t))
    # a first call per case loads each kernel and looks up the scratch address
    for w, split, t in runs:
        pa.check(_noalloc(pa, t["warm"], w, t["q"], t["kp"], t["vp"], t["bt"], t["cl"], split))
    pa.sync_status()
    for _, _, t in runs:
        t["out"].fill_(float("nan"))
    torch.cuda.synchronize()
    used_before = torch.cuda.memory_allocated()
    free_before, _ = torch.cuda.mem_get_info()

    for w, split, t in runs:  # two calls in a row, sharing the scratch
        pa.check(_noalloc(pa, t["out"], w, t["q"], t["kp"], t["vp"], t["bt"], t["cl"], split))
    pa.sync_status()
    assert torch.cuda.memory_allocated() == used_before
    assert torch.cuda.mem_get_info()[0] == free_before

    for call, (w, split, t) in enumerate(runs):
        ref = compact_oracle_step(w, list(range(w.num_seqs)))
        assert_attention_close(as_f64(t["out"]), ref, f"no-alloc call {call + 1} vs the oracle")
        assert torch.equal(t["out"], t["ref"]), f"no-alloc call {call + 1} differs from pa_decode"
