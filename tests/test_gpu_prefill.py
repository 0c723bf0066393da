"""Paged (chunked) prefill on the 5th-generation tensor cores against the
fp64 oracle: |gpu - ref| <= 2e-3 + 1e-2 |ref| element by element."""

import numpy as np
import pytest
import torch

import oracle
from harness import as_f64, assert_attention_close
from paged_kv_cache_416_b200 import workloads as W
from paged_kv_cache_416_b200.workloads import raw

pytestmark = pytest.mark.gpu


def run(pa, pw):
    b = pw.base
    out = pa.prefill(pw.q.cuda(), b.k_pool.cuda(), b.v_pool.cuda(),
                     torch.from_numpy(b.block_tables).cuda(),
                     torch.from_numpy(b.context_lens).cuda(),
                     torch.from_numpy(pw.query_start).cuda(), b.scale, pw.max_query_len,
                     b.max_context_len)
    pa.sync_status()
    return out


def ref(pw):
    b = pw.base
    return oracle.prefill(raw(pw.q), b.q_dtype, raw(b.k_pool), raw(b.v_pool), b.cache_dtype,
                          b.block_tables, b.context_lens, pw.query_start, b.scale, b.num_kv_heads)


@pytest.mark.parametrize("hq,hkv,bs,dtype", [(32, 8, 16, "bf16"), (64, 8, 16, "bf16"),
                                             (8, 8, 32, "f16"), (16, 4, 32, "bf16")])
def test_prefill_matches_oracle(pa, hq, hkv, bs, dtype):
    # full prefill, a chunk after a long context, one token, ragged tails,
    # and enough tokens for several query tiles at every group size
    pw = W.prefill(ctxs=(200, 300, 1, 77, 130), nqs=(200, 77, 1, 50, 130), hq=hq, hkv=hkv,
                   bs=bs, dtype=dtype)
    assert_attention_close(as_f64(run(pa, pw)), ref(pw), f"prefill {hq}/{hkv} bs{bs} {dtype}")


def test_prefill_of_one_token_equals_decode(pa):
    pw = W.prefill(ctxs=(333, 64, 17), nqs=(1, 1, 1), hq=32, hkv=8, bs=16, dtype="bf16")
    b = pw.base
    out = run(pa, pw)
    dec = pa.decode(pw.q.cuda(), b.k_pool.cuda(), b.v_pool.cuda(),
                    torch.from_numpy(b.block_tables).cuda(), torch.from_numpy(b.context_lens).cuda(),
                    b.scale, b.max_context_len)
    pa.sync_status()
    assert_attention_close(as_f64(out), as_f64(dec).astype(np.float64), "prefill vs decode")
    assert_attention_close(as_f64(out), ref(pw), "prefill one token")


@pytest.mark.parametrize("hq,hkv", [(12, 4), (96, 8)])
def test_prefill_group_sizes_that_do_not_divide_the_tile(pa, hq, hkv):
    # G = 3 and G = 12: a CTA takes floor(128 / G) tokens, the other rows of
    # its 128 are padding
    pw = W.prefill(ctxs=(90, 200), nqs=(90, 61), hq=hq, hkv=hkv, bs=16, dtype="bf16")
    assert_attention_close(as_f64(run(pa, pw)), ref(pw), f"prefill {hq}/{hkv}")


@pytest.mark.parametrize("hq,hkv,bs,dtype", [(16, 4, 16, "bf16"), (8, 8, 32, "f16")])
def test_prefill_head_dim_64(pa, hq, hkv, bs, dtype):
    # one 128-byte dim half per row: half the S k-steps, an O product of N = 64
    pw = W.prefill(ctxs=(40, 300, 130), nqs=(40, 90, 130), hq=hq, hkv=hkv, d=64, bs=bs,
                   dtype=dtype)
    assert_attention_close(as_f64(run(pa, pw)), ref(pw), f"prefill D64 {hq}/{hkv} bs{bs} {dtype}")


def test_prefill_rejects_unsupported_shapes(pa):
    pw = W.prefill(ctxs=(40,), nqs=(40,), hq=16, hkv=4, d=64, bs=16, dtype="bf16")
    b = pw.base
    with pytest.raises(pa.PagedAttnError) as e:  # e4m3 caches take no tensor-core path
        pa.prefill(pw.q.cuda(), b.k_pool.cuda().view(torch.float8_e4m3fn),
                   b.v_pool.cuda().view(torch.float8_e4m3fn),
                   torch.from_numpy(b.block_tables).cuda(), torch.from_numpy(b.context_lens).cuda(),
                   torch.from_numpy(pw.query_start).cuda(), b.scale, pw.max_query_len,
                   b.max_context_len)
    assert e.value.status == 2


def grow_keys(pw, rate):
    """Scale the key at position p by (1 + p * rate), so the scores, and with
    them each row's running max, keep growing along the context: the online
    softmax has to rescale O many times."""
    b = pw.base
    kp = b.k_pool.float()
    flat = kp.view(-1, b.num_kv_heads, kp.shape[-1])
    bs = kp.shape[1]
    for s in range(b.num_seqs):
        for p in range(int(b.context_lens[s])):
            flat[int(b.block_tables[s, p // bs]) * bs + p % bs] *= 1.0 + p * rate
    b.k_pool = kp.to(b.k_pool.dtype)
    return pw


@pytest.mark.parametrize("dtype,bs", [("bf16", 16), ("f16", 16), ("bf16", 32)])
def test_prefill_long_context_growing_scores(pa, dtype, bs):
    # a chunk late in a long context (many key tiles, both K/V stages and
    # every S / O barrier reused many times, the load warp's block ids read
    # across several 32-entry chunks) with scores that grow along the keys
    pw = grow_keys(W.prefill(seed=11, ctxs=(1500, 700), nqs=(96, 700), hq=32, hkv=8, bs=bs,
                             dtype=dtype), 1.0 / 48)
    assert_attention_close(as_f64(run(pa, pw)), ref(pw), f"prefill growing scores {dtype} bs{bs}")


def test_prefill_bad_table_entry_masks_its_block(pa):
    # a table entry outside the pool: the kernel reports it, masks that
    # block's keys and zeroes its values; the other outputs equal attention
    # over the remaining keys
    pw = W.prefill(seed=12, ctxs=(160,), nqs=(160,), hq=32, hkv=8, bs=16, dtype="bf16")
    b = pw.base
    # first a call whose values are all NaN, so that shared memory left over
    # from it holds NaN: a CTA whose first key tile holds the bad block (rows
    # 0-31 here, which never see it) must still zero that block's values
    nan_v = torch.full_like(b.v_pool, float("nan")).cuda()
    pa.prefill(pw.q.cuda(), b.k_pool.cuda(), nan_v, torch.from_numpy(b.block_tables).cuda(),
               torch.from_numpy(b.context_lens).cuda(), torch.from_numpy(pw.query_start).cuda(),
               b.scale, pw.max_query_len, b.max_context_len)
    pa.sync_status()
    b.block_tables = b.block_tables.copy()
    b.block_tables[0, 3] = b.k_pool.shape[0] + 5
    bt = torch.from_numpy(b.block_tables).cuda()
    out = pa.prefill(pw.q.cuda(), b.k_pool.cuda(), b.v_pool.cuda(), bt,
                     torch.from_numpy(b.context_lens).cuda(),
                     torch.from_numpy(pw.query_start).cuda(), b.scale, pw.max_query_len,
                     b.max_context_len)
    with pytest.raises(pa.PagedAttnError):
        pa.sync_status()
    got = as_f64(out)
    assert np.isfinite(got).all()
    # rows before block 3 never see it: they equal the oracle on the intact table
    good = ref(W.prefill(seed=12, ctxs=(160,), nqs=(160,), hq=32, hkv=8, bs=16, dtype="bf16"))
    assert_attention_close(got[:48], good[:48], "rows before the bad block")


def test_prefill_empty_chunks_and_an_inconsistent_length(pa):
    # a sequence with no new tokens in the batch; then one whose context is
    # shorter than its chunk: its rows are zeroed and reported, the others
    # still equal the oracle
    pw = W.prefill(seed=13, ctxs=(100, 50, 80, 30), nqs=(20, 0, 80, 10), hq=32, hkv=8, bs=16,
                   dtype="bf16")
    want = ref(pw)
    assert_attention_close(as_f64(run(pa, pw)), want, "prefill with an empty chunk")
    b = pw.base
    lens = b.context_lens.copy()
    lens[3] = 5  # 10 new tokens, 5 cached
    out = pa.prefill(pw.q.cuda(), b.k_pool.cuda(), b.v_pool.cuda(),
                     torch.from_numpy(b.block_tables).cuda(), torch.from_numpy(lens).cuda(),
                     torch.from_numpy(pw.query_start).cuda(), b.scale, pw.max_query_len,
                     b.max_context_len)
    with pytest.raises(pa.PagedAttnError) as e:
        pa.sync_status()
    assert e.value.status == 8  # PA_ERR_DEVICE_BOUNDS
    got = as_f64(out)
    q3 = int(pw.query_start[3])
    assert not got[q3:].any()
    assert_attention_close(got[:q3], want[:q3], "the consistent sequences")


def test_prefill_full_size_sampled(pa):
    """The benchmark's prefill (8 sequences x 4096 new tokens, 64/8 heads,
    D 128, bf16, bs 16, the benchmark's seed) in the launch configuration it
    times.  Sampled rows are checked one by one: the token at position p
    attends to keys 0..p, which is the oracle's decode of that query over a
    context of p + 1 tokens through the same block table."""
    n = 4096
    pw = W.prefill(seed=3, device="cuda", ctxs=(n,) * 8, nqs=(n,) * 8, hq=64, hkv=8, bs=16,
                   dtype="bf16")
    b = pw.base
    out = pa.prefill(pw.q, b.k_pool, b.v_pool, torch.from_numpy(b.block_tables).cuda(),
                     torch.from_numpy(b.context_lens).cuda(),
                     torch.from_numpy(pw.query_start).cuda(), b.scale, pw.max_query_len,
                     b.max_context_len)
    pa.sync_status()
    assert torch.isfinite(out.float()).all()
    rng = np.random.default_rng(0)
    picks = [(0, 0), (0, 15), (1, 16), (2, 63), (3, 64), (4, 127), (5, 128), (6, 2047),
             (7, n - 1), (5, n - 1)] + [(int(s), int(i)) for s, i in
                                        zip(rng.integers(0, 8, 6), rng.integers(0, n, 6))]
    kp, vp = raw(b.k_pool), raw(b.v_pool)
    for s, i in picks:
        row = int(pw.query_start[s]) + i
        pos = int(b.context_lens[s]) - n + i
        ref = oracle.decode(raw(pw.q[row:row + 1]), b.q_dtype, kp, vp, b.cache_dtype,
                            b.block_tables[s:s + 1], np.array([pos + 1]), b.scale,
                            b.num_kv_heads)
        assert_attention_close(as_f64(out[row:row + 1]), ref, f"prefill full size seq {s} token {i}")
