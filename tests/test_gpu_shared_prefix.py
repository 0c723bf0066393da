"""Shared-prefix (cascade) decode against the fp64 oracle and against plain
decode: |gpu - ref| <= 2e-3 + 1e-2 |ref| element by element.

The shared blocks of a group are attended once for all members' queries and
merged by log-sum-exp with each member's own tokens; the result must be the
plain decode attention of every sequence ("PagedAttention", §Diziler Arasında
Blokları Paylaşma: forked samples name the same blocks)."""

import numpy as np
import pytest
import torch

import oracle
from harness import as_f64, assert_attention_close
from paged_kv_cache_416_b200 import workloads as W
from paged_kv_cache_416_b200.workloads import raw

pytestmark = pytest.mark.gpu


def step_inputs(pa, w):
    """Device pools after the workload's decode step (copy-on-write, write)."""
    kp = w.k_pool.cuda().clone()
    vp = w.v_pool.cuda().clone()
    if len(w.cow_pairs):
        pa.copy_blocks(kp, vp, torch.from_numpy(w.cow_pairs).cuda())
    pa.write_kv(w.new_k.cuda().contiguous(), w.new_v.cuda().contiguous(),
                torch.from_numpy(w.slot_mapping).cuda(), kp, vp, w.k_scale, w.v_scale)
    return kp, vp


def run_shared(pa, w, kp, vp, group_start, group_seqs, split_tokens=0):
    out = pa.decode_shared_prefix(
        w.q.cuda().contiguous(), kp, vp, torch.from_numpy(w.block_tables).cuda(),
        torch.from_numpy(w.context_lens).cuda(),
        torch.from_numpy(np.asarray(group_start, np.int32)).cuda(),
        torch.from_numpy(np.asarray(group_seqs, np.int32)).cuda(), w.scale, w.max_context_len,
        k_scale=w.k_scale, v_scale=w.v_scale, split_tokens=split_tokens)
    return out


def run_plain(pa, w, kp, vp, split_tokens=0):
    return pa.decode(w.q.cuda().contiguous(), kp, vp, torch.from_numpy(w.block_tables).cuda(),
                     torch.from_numpy(w.context_lens).cuda(), w.scale, w.max_context_len,
                     k_scale=w.k_scale, v_scale=w.v_scale, split_tokens=split_tokens)


def oracle_out(w, kp, vp, seqs=None):
    return oracle.decode(raw(w.q), w.q_dtype, raw(kp), raw(vp), w.cache_dtype, w.block_tables,
                         w.context_lens, w.scale, w.num_kv_heads, w.k_scale, w.v_scale,
                         seqs=seqs)


def groups(w):
    return w.meta["group_start"], w.meta["group_seqs"]


@pytest.mark.parametrize("phase", ["fork", "tails"])
@pytest.mark.parametrize("split", [0, 64])
def test_shared_prefix_matches_oracle_and_plain_decode(pa, phase, split):
    # G = 4: chunks of 4 members, one pass over the shared blocks per prompt;
    # split 64 asks for short ranges, so every chunk is cut into several that
    # the last one merges
    w = W._shared_prefix(phase, 4, "cpu", prompts=5, samples=4, prefix=320, max_tail=200)
    kp, vp = step_inputs(pa, w)
    out = run_shared(pa, w, kp, vp, *groups(w), split_tokens=split)
    plain = run_plain(pa, w, kp, vp, split_tokens=split)
    pa.sync_status()
    ref = oracle_out(w, kp, vp)
    assert_attention_close(as_f64(out), ref, f"shared prefix {phase} split {split}")
    assert_attention_close(as_f64(out), as_f64(plain), "shared prefix vs plain decode")


@pytest.mark.parametrize("hq,hkv,d,bs,dtype", [(64, 8, 128, 16, "bf16"), (8, 8, 128, 16, "bf16"),
                                               (16, 4, 64, 32, "f16"), (32, 8, 64, 16, "bf16")])
def test_shared_prefix_shapes(pa, hq, hkv, d, bs, dtype):
    # G = 8 (two members per chunk), G = 1 (all 5 members in one chunk),
    # head_dim 64, block size 32, fp16
    w = W._shared_prefix("tails", 7, "cpu", prompts=3, samples=5, prefix=200, max_tail=90,
                         hq=hq, hkv=hkv, d=d, bs=bs)
    if dtype == "f16":  # same values stored as fp16 words
        for name in ("q", "k_pool", "v_pool", "new_k", "new_v"):
            setattr(w, name, getattr(w, name).to(torch.float16))
        w.q_dtype = w.cache_dtype = "f16"
    kp, vp = step_inputs(pa, w)
    out = run_shared(pa, w, kp, vp, *groups(w), split_tokens=96)
    pa.sync_status()
    assert_attention_close(as_f64(out), oracle_out(w, kp, vp), f"shared prefix {hq}/{hkv} D{d} bs{bs}")


@pytest.mark.parametrize("phase", ["fork", "tails"])
@pytest.mark.parametrize("hq,hkv,d,bs,split", [(32, 8, 128, 16, 0), (32, 8, 128, 16, 64),
                                               (16, 4, 64, 32, 96), (64, 8, 128, 32, 0)])
def test_shared_prefix_e4m3_cache(pa, phase, hq, hkv, d, bs, split):
    """e4m3 caches (q bf16, per-tensor scales): the 16-row tiles and the
    8-column form dequantise on load, against the oracle on the dequantised
    cache and against plain decode."""
    w = W._shared_prefix(phase, 12, "cpu", prompts=4, samples=4, prefix=288, max_tail=150,
                         hq=hq, hkv=hkv, d=d, bs=bs, cache="e4m3")
    kp, vp = step_inputs(pa, w)
    out = run_shared(pa, w, kp, vp, *groups(w), split_tokens=split)
    plain = run_plain(pa, w, kp, vp, split_tokens=split)
    pa.sync_status()
    ref = oracle_out(w, kp, vp)
    assert_attention_close(as_f64(out), ref, f"e4m3 shared prefix {phase} {hq}/{hkv} D{d} bs{bs}")
    assert_attention_close(as_f64(out), as_f64(plain), "e4m3 shared prefix vs plain decode")


@pytest.mark.parametrize("hq,hkv,cache,split", [(64, 4, "bf16", 0), (64, 4, "bf16", 64),
                                                (48, 4, "bf16", 0), (64, 4, "e4m3", 64),
                                                (96, 8, "e4m3", 0)])
def test_shared_prefix_more_than_eight_heads_per_kv_head(pa, hq, hkv, cache, split):
    """12 and 16 query heads per kv head: a chunk is one member whose heads
    fill the 16-row tile, for its shared and its own ranges."""
    w = W._shared_prefix("tails", 13, "cpu", prompts=3, samples=3, prefix=200, max_tail=120,
                         hq=hq, hkv=hkv, cache=cache)
    kp, vp = step_inputs(pa, w)
    out = run_shared(pa, w, kp, vp, *groups(w), split_tokens=split)
    pa.sync_status()
    assert_attention_close(as_f64(out), oracle_out(w, kp, vp),
                           f"shared prefix {hq}/{hkv} {cache} split {split}")


def test_ungrouped_and_unrelated_sequences_decode_plainly(pa):
    # only the first two prompts' samples are grouped; a third group joins
    # sequences of different prompts (their tables share no leading block)
    w = W._shared_prefix("tails", 9, "cpu", prompts=4, samples=3, prefix=160, max_tail=70)
    kp, vp = step_inputs(pa, w)
    gs = [0, 3, 6, 8]
    members = [0, 1, 2, 3, 4, 5, 6, 9]
    out = run_shared(pa, w, kp, vp, gs, members, split_tokens=64)
    pa.sync_status()
    assert_attention_close(as_f64(out), oracle_out(w, kp, vp), "partly grouped")


def test_bad_group_lists_decode_plainly_and_report(pa):
    # sequence 1 listed twice: both groups holding it decode plainly; an
    # index outside the batch the same way; the output is still attention
    w = W._shared_prefix("tails", 10, "cpu", prompts=3, samples=3, prefix=160, max_tail=70)
    kp, vp = step_inputs(pa, w)
    gs = [0, 3, 5, 8]
    members = [0, 1, 2, 1, 4, 6, 7, 99]
    out = run_shared(pa, w, kp, vp, gs, members)
    with pytest.raises(pa.PagedAttnError):
        pa.sync_status()
    assert_attention_close(as_f64(out), oracle_out(w, kp, vp), "bad group lists")


def test_no_groups_decodes_every_sequence_plainly(pa):
    # zero groups: every sequence is a chunk of its own (no shared blocks)
    w = W._shared_prefix("tails", 11, "cpu", prompts=2, samples=3, prefix=96, max_tail=50)
    kp, vp = step_inputs(pa, w)
    out = run_shared(pa, w, kp, vp, [0], [])
    pa.sync_status()
    assert_attention_close(as_f64(out), oracle_out(w, kp, vp), "no groups")


def test_shared_prefix_full_size_sampled(pa):
    # the full shared-prefix workload (32 prompts x 4 samples, 1024 + r shared
    # tokens, tails up to 512) in the configuration the bench times; sampled
    # sequences from several prompts and sample positions against the oracle
    w = W.make("shared_prefix_tails")
    kp, vp = step_inputs(pa, w)
    out = run_shared(pa, w, kp, vp, *groups(w))
    pa.sync_status()
    seqs = [0, 1, 3, 38, 77, 126, 127]
    ref = oracle_out(w, kp, vp, seqs=seqs)
    got = as_f64(out)
    assert_attention_close(got[seqs], ref[seqs], "full-size shared prefix (sampled)")
    assert np.isfinite(got).all()
