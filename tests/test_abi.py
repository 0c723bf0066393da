"""The C-ABI library loads and exports every entry point its header declares;
host-side validation rejects bad arguments before any CUDA call (CPU only)."""

import numpy as np
import ctypes
import os
import re

import pytest

from paged_kv_cache_416_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedattn.h")


@pytest.fixture(scope="module")
def pa():
    build.build()  # nvcc cross-compiles without a GPU; no-op when up to date
    from paged_kv_cache_416_b200 import pagedattn
    return pagedattn


def declared_entry_points():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_calls():
    names = declared_entry_points()
    for n in ("pa_decode", "pa_write_kv", "pa_copy_blocks", "pa_decode_workspace_size",
              "pa_sync_status", "pa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(pa):
    lib = ctypes.CDLL(pa.LIB_PATH)
    for name in declared_entry_points():
        assert hasattr(lib, name), name
    assert set(declared_entry_points()) <= set(pa.ENTRY_POINTS)


def test_split_and_workspace_rules(pa):
    # one item per (sequence, kv head) when that fills the GPU
    assert pa.pa_decode_split_tokens(256, 8, 16, 4096, 0) == 4096
    # header, range offsets [257] int32, work order [256] int4
    assert pa.pa_decode_workspace_size(256, 64, 8, 128, 16, 4096, 0) == 256 + 1280 + 4096
    # long contexts are cut into ranges (multiples of the block size)
    s = pa.pa_decode_split_tokens(128, 8, 16, 32768, 0)
    assert s == 1024
    ranges = 128 * 32
    assert pa.pa_decode_workspace_size(128, 32, 8, 128, 16, 32768, 0) == \
        256 + 768 + ranges * 16 + 128 * 8 * 4 + ranges * 32 * 4 + ranges * 32 * 128 * 4
    # few sequences: split for parallelism
    s = pa.pa_decode_split_tokens(1, 8, 32, 16384, 0)
    assert 256 <= s < 16384 and s % 32 == 0
    # explicit split rounds up to the block size
    assert pa.pa_decode_split_tokens(4, 4, 16, 1000, 40) == 48
    assert pa.pa_decode_split_tokens(4, 4, 24, 1000, 0) == 0  # bad block size


def _decode(pa, **kw):
    args = dict(out=None, q=None, q_dtype=1, k_pool=None, v_pool=None, cache_dtype=1,
                block_tables=None, max_blocks=4, context_lens=None, max_ctx=64, B=2, hq=8, hkv=2,
                D=128, bs=16, N=32, scale=0.1, k_scale=1.0, v_scale=1.0, split=0, ws=None,
                ws_bytes=0, stream=None)
    args.update(kw)
    return pa.pa_decode(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(q_dtype=0, cache_dtype=1), 2),         # q must match a 16-bit cache
    (dict(q_dtype=2, cache_dtype=2), 2),         # fp8 queries are not supported
    (dict(q_dtype=7), 2),
    (dict(D=96), 3),
    (dict(bs=8), 3),
    (dict(max_ctx=65), 3),                       # exceeds max_blocks * bs
    (dict(hq=7), 4),
    (dict(hq=160, hkv=2), 4),                    # 80 query heads per kv head (> 64)
    (dict(hq=32, hkv=2), 1),                     # 16 per kv head: two column groups, valid
    (dict(cache_dtype=2, k_scale=0.0), 3),
    (dict(scale=float("inf")), 3),
    (dict(), 1),                                 # valid sizes, null pointers
])
def test_decode_rejects_bad_arguments_on_the_host(pa, kw, status):
    assert _decode(pa, **kw) == status
    assert pa.pa_last_error()


def test_decode_with_no_sequences_is_a_no_op(pa):
    assert _decode(pa, B=0) == 0


def test_write_and_copy_validation(pa):
    W = pa.pa_write_kv
    assert W(None, None, 1, None, 4, None, None, 0, 8, 16, 2, 128, 1.0, 1.0, None) == 2  # bf16 into f16
    assert W(None, None, 1, None, 4, None, None, 2, 8, 16, 2, 128, 0.0, 1.0, None) == 3  # bad scale
    assert W(None, None, 1, None, 4, None, None, 1, 8, 12, 2, 128, 1.0, 1.0, None) == 3  # bad bs
    assert W(None, None, 1, None, 4, None, None, 1, 8, 16, 2, 128, 1.0, 1.0, None) == 1  # nulls
    assert W(None, None, 1, None, 0, None, None, 1, 8, 16, 2, 128, 1.0, 1.0, None) == 0  # no tokens
    C = pa.pa_copy_blocks
    assert C(None, None, 1, 8, 16, 2, 128, None, 0, None) == 0
    assert C(None, None, 1, 8, 16, 2, 128, None, 3, None) == 1
    assert C(None, None, 9, 8, 16, 2, 128, None, 3, None) == 2


def test_python_binding_raises_with_the_message(pa):
    with pytest.raises(pa.PagedAttnError) as e:
        pa.check(_decode(pa, hq=7))
    assert "PA_ERR_HEADS" in str(e.value)


def _shared(pa, **kw):
    args = dict(out=None, q=None, q_dtype=1, k_pool=None, v_pool=None, cache_dtype=1,
                block_tables=None, max_blocks=4, context_lens=None, max_ctx=64, group_start=None,
                group_seqs=None, num_groups=1, B=2, hq=8, hkv=2, D=128, bs=16, N=32, scale=0.1,
                k_scale=1.0, v_scale=1.0, split=0, ws=None, ws_bytes=0, stream=None)
    args.update(kw)
    return pa.pa_decode_shared_prefix(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(q_dtype=2, cache_dtype=2), 2),         # an e4m3 query
    (dict(q_dtype=0, cache_dtype=1), 2),
    (dict(cache_dtype=2, k_scale=0.0), 3),       # e4m3 cache with a bad scale
    (dict(hq=34), 4),                            # 17 query heads per kv head
    (dict(hq=32, cache_dtype=2), 1),             # 16 per kv head, e4m3: valid, nulls
    (dict(D=96), 3),
    (dict(num_groups=-1), 3),
    (dict(max_ctx=65), 3),
    (dict(hq=7), 4),
    (dict(scale=float("nan")), 3),
    (dict(), 1),                                 # valid sizes, null pointers
])
def test_shared_prefix_decode_rejects_bad_arguments_on_the_host(pa, kw, status):
    assert _shared(pa, **kw) == status
    assert pa.pa_last_error()


def test_shared_prefix_workspace_is_bounded(pa):
    # the partial slots are bounded through the shortest range the host
    # fixes, so the workspace stays a few tens of MB at the bench's sizes
    n = pa.pa_decode_shared_prefix_workspace_size(128, 32, 8, 128, 16, 1568, 0)
    assert 0 < n < 64 << 20
    n_big = pa.pa_decode_shared_prefix_workspace_size(256, 64, 8, 128, 16, 32768, 0)
    assert 0 < n_big < 96 << 20
    assert pa.pa_decode_shared_prefix_workspace_size(4, 8, 2, 96, 16, 64, 0) == 0
    assert _shared(pa, B=0) == 0


def _prefill(pa, **kw):
    args = dict(out=None, q=None, q_dtype=1, k_pool=None, v_pool=None, cache_dtype=1,
                block_tables=None, max_blocks=4, context_lens=None, query_start=None, B=2,
                max_q=16, max_ctx=64, hq=32, hkv=8, D=128, bs=16, N=32, scale=0.1, stream=None)
    args.update(kw)
    return pa.pa_prefill(*args.values())


@pytest.mark.parametrize("kw,status", [
    (dict(cache_dtype=2), 2),                    # tensor-core path: 16-bit caches only
    (dict(q_dtype=0), 2),
    (dict(D=64), 1),                             # head_dim 64: valid
    (dict(D=96), 3),
    (dict(hq=24, hkv=8), 1),                     # G = 3: floor(128 / 3) tokens a CTA, valid
    (dict(hq=258, hkv=2), 4),                    # G = 129 > 128 rows
    (dict(), 1),
])
def test_prefill_rejects_bad_arguments_on_the_host(pa, kw, status):
    assert _prefill(pa, **kw) == status


def test_split_rule_properties(pa):
    """The split length stated in the header, over random sizes: a multiple
    of the block size, at most 1024 ranges per sequence, a requested length
    only ever raised (to a block multiple, then to the range cap); and the
    workspace grows with the number of sequences when the split is fixed (the
    automatic split grows with the batch, so there a smaller batch can need
    more, as the header says)."""
    rng = np.random.default_rng(7)
    for _ in range(3000):
        B = int(rng.integers(1, 4097))
        hkv = int(rng.choice([1, 2, 4, 8, 16]))
        bs = int(rng.choice([16, 32]))
        ctx = int(rng.integers(1, 262145))
        user = int(rng.choice([0, int(rng.integers(1, 70000))]))
        S = pa.pa_decode_split_tokens(B, hkv, bs, ctx, user)
        assert S >= bs and S % bs == 0, (B, hkv, bs, ctx, user, S)
        assert -(-ctx // S) <= 1024, (B, hkv, bs, ctx, user, S)
        if user:
            assert S >= user and (S - bs < user or -(-ctx // (S - bs)) > 1024), (ctx, user, S)
        hq = hkv * int(rng.choice([1, 4, 8]))
        d = int(rng.choice([64, 128]))
        w1 = pa.pa_decode_workspace_size(B, hq, hkv, d, bs, ctx, user)
        w2 = pa.pa_decode_workspace_size(B + 1, hq, hkv, d, bs, ctx, user)
        assert w1 > 0 and w2 > 0
        if user:
            assert w1 <= w2
