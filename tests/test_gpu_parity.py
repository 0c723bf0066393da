"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Writes and copies: bit-exact.  Attention: |gpu - ref| <= 2e-3 + 1e-2 |ref|
element by element (fp16 / bf16 caches with fp32 accumulation; for the e4m3
cache against the oracle run on the dequantised cache).  Workloads are the
seeded generators of paged_kv_cache_416_b200.workloads at sizes the oracle
finishes in seconds (several blocks per warp, ragged last blocks), plus the
benchmark sizes checked on sampled sequences.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from harness import (as_f64, assert_attention_close, compact_oracle_step, gpu_step,
                     oracle_step)
from paged_kv_cache_416_b200 import workloads as W
from paged_kv_cache_416_b200.workloads import raw

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": dict(),
    "llama13b_mha": dict(num_seqs=6),
    "llama70b_gqa": dict(num_seqs=3),
    "llama70b_gqa_ragged": dict(num_seqs=5, context_len=1000),
    "shared_prefix_fork": dict(prompts=3),
    "shared_prefix_tails": dict(prompts=3),
    "fp8_longtail_bs16": dict(num_seqs=10, max_len=6000),
    "fp8_longtail_bs32": dict(num_seqs=10, max_len=6000),
}


def small(name, seed=None, device="cpu"):
    base = "llama70b_gqa" if name == "llama70b_gqa_ragged" else name
    return W.make(base, seed=seed, device=device, **SMALL[name])


# ------------------------------------------------------------- cache writes

@pytest.mark.parametrize("in_dt,cache_dt", [("f16", "f16"), ("bf16", "bf16"), ("bf16", "e4m3"),
                                            ("f16", "e4m3")])
@pytest.mark.parametrize("bs,hkv,d", [(16, 8, 128), (32, 3, 64)])
def test_write_kv_bit_exact(pa, in_dt, cache_dt, bs, hkv, d):
    g = torch.Generator().manual_seed(7)
    N, T = 40, 300
    td = W.TORCH_DTYPE
    k = (torch.randn(T, hkv, d, generator=g) * 3).to(td[in_dt])
    v = (torch.randn(T, hkv, d, generator=g) * 3).to(td[in_dt])
    # distinct slots, some padding (-1)
    slots = torch.randperm(N * bs, generator=g)[:T].to(torch.int64)
    slots[::7] = -1
    kp = torch.randint(0, 255, (N, bs, hkv, d), generator=g, dtype=torch.uint8)
    vp = torch.randint(0, 255, (N, bs, hkv, d), generator=g, dtype=torch.uint8)
    if cache_dt != "e4m3":
        kp = torch.randint(-30000, 30000, (N, bs, hkv, d), generator=g, dtype=torch.int16).view(td[cache_dt])
        vp = torch.randint(-30000, 30000, (N, bs, hkv, d), generator=g, dtype=torch.int16).view(td[cache_dt])
    else:
        kp, vp = kp.view(torch.float8_e4m3fn), vp.view(torch.float8_e4m3fn)
    ks, vs = 0.0123, 0.5
    ok_, ov_ = raw(kp).copy(), raw(vp).copy()
    oracle.write_kv(raw(k), raw(v), in_dt, slots.numpy(), ok_, ov_, cache_dt, ks, vs)
    gk, gv = kp.cuda(), vp.cuda()
    pa.write_kv(k.cuda(), v.cuda(), slots.cuda(), gk, gv, ks, vs)
    pa.sync_status()
    assert np.array_equal(raw(gk), ok_)
    assert np.array_equal(raw(gv), ov_)


def test_write_kv_e4m3_edge_values(pa):
    """Ties, the saturation boundary, subnormals and infinities quantise as
    the oracle does (RNE, satfinite)."""
    vals = oracle.e4m3_finite_values()
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([vals, -vals, mids, -mids, [448.0, 464.0, 480.0, 1e30, np.inf, -np.inf,
                                                   2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11]])
    x = x.astype(np.float32)
    d = 128
    n = -(-len(x) // d) * d
    x = np.concatenate([x, np.zeros(n - len(x), np.float32)]).reshape(-1, 1, d)
    # values must be exact in bf16 for this test: keep those that are
    xb = torch.from_numpy(x).to(torch.bfloat16)
    T = xb.shape[0]
    slots = torch.arange(T, dtype=torch.int64)
    kp = torch.zeros(2, 16, 1, d, dtype=torch.float8_e4m3fn)
    ok_, ov_ = raw(kp).copy(), raw(kp).copy()
    oracle.write_kv(raw(xb), raw(xb), "bf16", slots.numpy(), ok_, ov_, "e4m3", 1.0, 1.0)
    gk, gv = kp.cuda(), kp.clone().cuda()
    pa.write_kv(xb.cuda(), xb.cuda(), slots.cuda(), gk, gv, 1.0, 1.0)
    pa.sync_status()
    assert np.array_equal(raw(gk), ok_) and np.array_equal(raw(gv), ov_)


# ------------------------------------------------------------- block copies

@pytest.mark.parametrize("cache_dt,bs,hkv,d", [("bf16", 16, 8, 128), ("e4m3", 32, 4, 64),
                                               ("f16", 16, 40, 128)])
def test_copy_blocks_bit_exact(pa, cache_dt, bs, hkv, d):
    g = torch.Generator().manual_seed(3)
    N = 200
    kp = torch.randint(0, 255, (N, bs, hkv, d), generator=g, dtype=torch.uint8)
    vp = torch.randint(0, 255, (N, bs, hkv, d), generator=g, dtype=torch.uint8)
    if cache_dt != "e4m3":
        kp = torch.randint(-30000, 30000, (N, bs, hkv, d), generator=g, dtype=torch.int16).view(W.TORCH_DTYPE[cache_dt])
        vp = torch.randint(-30000, 30000, (N, bs, hkv, d), generator=g, dtype=torch.int16).view(W.TORCH_DTYPE[cache_dt])
    else:
        kp, vp = kp.view(torch.float8_e4m3fn), vp.view(torch.float8_e4m3fn)
    perm = torch.randperm(N, generator=g)
    pairs = torch.stack([perm[:60], perm[60:120]], 1).to(torch.int64)  # disjoint src / dst
    ok_, ov_ = raw(kp).copy(), raw(vp).copy()
    oracle.copy_blocks(ok_, ov_, pairs.numpy())
    gk, gv = kp.cuda(), vp.cuda()
    pa.copy_blocks(gk, gv, pairs.cuda())
    pa.sync_status()
    assert np.array_equal(raw(gk), ok_) and np.array_equal(raw(gv), ov_)


def test_copy_then_write_leaves_the_source_intact(pa):
    """After a copy-on-write the two blocks are equal; a write into the copy
    leaves the source untouched."""
    kp = torch.randn(8, 16, 2, 64).to(torch.bfloat16).cuda()
    vp = torch.randn(8, 16, 2, 64).to(torch.bfloat16).cuda()
    src0k, src0v = kp[3].clone(), vp[3].clone()
    pa.copy_blocks(kp, vp, torch.tensor([[3, 5]], dtype=torch.int64, device="cuda"))
    pa.sync_status()
    assert torch.equal(kp[5], src0k) and torch.equal(vp[5], src0v)
    new = torch.randn(1, 2, 64).to(torch.bfloat16).cuda()
    pa.write_kv(new, new, torch.tensor([5 * 16 + 7], dtype=torch.int64, device="cuda"), kp, vp)
    pa.sync_status()
    assert torch.equal(kp[5, 7], new[0]) and torch.equal(kp[3], src0k)


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("name", list(SMALL))
def test_decode_step_matches_oracle(pa, name):
    w = small(name)
    out, kp, vp = gpu_step(pa, w)
    ref, okp, ovp = oracle_step(w)
    # the step's writes and copies are bit-exact
    assert np.array_equal(raw(kp), okp) and np.array_equal(raw(vp), ovp)
    assert_attention_close(as_f64(out), ref, name)


@pytest.mark.parametrize("name", ["fp8_longtail_bs16", "llama70b_gqa_ragged", "tiny",
                                  "shared_prefix_tails"])
def test_decode_split_size_does_not_change_the_result(pa, name):
    w = small(name)
    ref, _, _ = oracle_step(w)
    bs = w.block_size
    outs = []
    for split in (bs, 3 * bs, 256, 0, 1 << 20):
        out, _, _ = gpu_step(pa, w, split_tokens=split)
        assert_attention_close(as_f64(out), ref, f"{name} split {split}")
        outs.append(out)
    # the same call twice gives bit-identical output
    again, _, _ = gpu_step(pa, w, split_tokens=3 * bs)
    assert torch.equal(again, outs[1])


def test_decode_is_independent_of_physical_placement(pa):
    """Permuting physical block ids (contents moved along) gives a
    bit-identical output."""
    w = small("fp8_longtail_bs16")
    out1, _, _ = gpu_step(pa, w)
    g = torch.Generator().manual_seed(99)
    perm = torch.randperm(w.num_blocks, generator=g)  # old id i -> new id perm[i]
    kp2 = torch.empty_like(w.k_pool)
    vp2 = torch.empty_like(w.v_pool)
    kp2[perm] = w.k_pool
    vp2[perm] = w.v_pool
    bt = w.block_tables.copy()
    m = bt >= 0
    bt[m] = perm.numpy()[bt[m]]
    slots = w.slot_mapping.copy()
    ok_ = slots >= 0
    slots[ok_] = perm.numpy()[slots[ok_] // w.block_size] * w.block_size + slots[ok_] % w.block_size
    w2 = W.Workload(**{**w.__dict__, "k_pool": kp2, "v_pool": vp2, "block_tables": bt,
                       "slot_mapping": slots})
    out2, _, _ = gpu_step(pa, w2)
    assert torch.equal(out1, out2)


def test_shared_blocks_equal_unshared_copies(pa):
    """Sequences reading a shared prefix give bit-identical outputs to the
    same sequences reading private copies of it."""
    w = small("shared_prefix_tails")
    out_shared, _, _ = gpu_step(pa, w)
    # give every sequence private copies of every block it shares
    bt = w.block_tables.copy()
    kp, vp = w.k_pool.clone(), w.v_pool.clone()
    owner = {}
    extra_k, extra_v = [], []
    nxt = w.num_blocks
    for s in range(w.num_seqs):
        nb = -(-int(w.context_lens[s]) // w.block_size)
        for j in range(nb):
            b = int(bt[s, j])
            if b in owner and owner[b] != s:
                extra_k.append(kp[b].clone())
                extra_v.append(vp[b].clone())
                bt[s, j] = nxt
                nxt += 1
            else:
                owner[b] = s
    assert extra_k, "the workload shares blocks"
    kp = torch.cat([kp, torch.stack(extra_k)])
    vp = torch.cat([vp, torch.stack(extra_v)])
    w2 = W.Workload(**{**w.__dict__, "k_pool": kp, "v_pool": vp, "block_tables": bt,
                       "num_blocks": nxt})
    # the step's new tokens live in private blocks already (no remap needed)
    out_private, _, _ = gpu_step(pa, w2)
    assert torch.equal(out_shared, out_private)


def test_unused_table_entries_and_slots_are_never_read(pa):
    w = small("llama70b_gqa_ragged")
    out1, _, _ = gpu_step(pa, w)
    bt = w.block_tables.copy()
    # widen the table with garbage past every sequence's blocks
    bt = np.concatenate([bt, np.full((bt.shape[0], 5), 10 ** 9, np.int32)], 1)
    w2 = W.Workload(**{**w.__dict__, "block_tables": bt})
    out2, _, _ = gpu_step(pa, w2)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("d,bs,cache", [(64, 16, "f16"), (128, 32, "bf16"), (64, 32, "e4m3"),
                                         (128, 16, "e4m3")])
def test_decode_edge_lengths(pa, d, bs, cache):
    """Lengths 0, 1, bs-1, bs, bs+1, a multiple of bs, and a long one; one
    token gives that token's value row exactly."""
    lens = [0, 1, bs - 1, bs, bs + 1, 4 * bs, 777, 2]
    hq, hkv = 8, 2
    qd = "bf16" if cache != "f16" else "f16"
    w = W._generic("edge", lens, hq, hkv, d, bs, qd, cache, seed=17, device="cpu")
    out, kp, vp = gpu_step(pa, w, split_tokens=2 * bs)
    ref, _, ovp = oracle_step(w)
    assert_attention_close(as_f64(out), ref, "edge lengths")
    o = as_f64(out)
    assert not o[0].any()  # empty context
    if cache != "e4m3":
        # single token: the output is exactly the token's value row
        v = oracle.decode_cache(ovp, cache)
        slot = int(w.slot_mapping[1])
        for h in range(hq):
            assert np.array_equal(o[1, h], v[slot // bs, slot % bs, h // (hq // hkv)])


def test_e4m3_every_code_decodes_exactly(pa):
    """A one-token context returns v_scale * decode(code) for every one of the
    256 codes (exact in bf16), NaN codes giving NaN."""
    d, hkv, bs = 128, 2, 16
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(1, 1, hkv, d)
    vp = torch.zeros(1, bs, hkv, d, dtype=torch.uint8)
    vp[0, 0] = codes[0, 0]
    kp = torch.zeros(1, bs, hkv, d, dtype=torch.uint8)
    q = torch.randn(1, 4, d).to(torch.bfloat16)
    out = pa.decode(q.cuda(), kp.view(torch.float8_e4m3fn).cuda(), vp.view(torch.float8_e4m3fn).cuda(),
                    torch.zeros(1, 1, dtype=torch.int32, device="cuda"),
                    torch.ones(1, dtype=torch.int32, device="cuda"), 0.1, 1, k_scale=1.0, v_scale=1.0)
    pa.sync_status()
    got = as_f64(out)[0]  # [4 heads, D]
    want = oracle.e4m3_decode(codes.numpy().reshape(hkv, d))
    for h in range(4):
        np.testing.assert_array_equal(got[h], want[h // 2])


@pytest.mark.parametrize("split", [0, 64])
def test_e4m3_cache_takes_any_bf16_query_range(pa, split):
    """With an e4m3 cache the products run in fp16: each head's query is
    scaled by a power of two before its fp16 conversion, so queries far
    outside the fp16 range (components of 1e5 and 1e20) and far below it
    (1e-6, 1e-20) still match the oracle."""
    rng = np.random.default_rng(43)
    lens = rng.integers(1, 400, size=7)
    hq, hkv = 8, 2
    w = W._generic("q_range", lens, hq, hkv, 128, 16, "bf16", "e4m3", seed=43, device="cpu")
    factors = torch.tensor([1e5, 1e-6, 1.0, 7e4, 1e20, 1e-20, 300.0, 2.5e5])
    q = (w.q.float() * factors[None, :, None]).to(torch.bfloat16)
    assert (q.float().abs().amax(dim=(0, 2))[[0, 3, 4, 7]] > 65504).all()
    w2 = W.Workload(**{**w.__dict__, "q": q})
    out, _, _ = gpu_step(pa, w2, split_tokens=split)
    ref, _, _ = oracle_step(w2)
    assert torch.isfinite(out.float()).all()
    assert_attention_close(as_f64(out), ref, f"e4m3 cache, scaled queries, split {split}")


# ------------------------------------------------------ device error word

def test_out_of_range_indices_are_reported_not_faulted(pa):
    w = small("tiny")
    bt = w.block_tables.copy()
    bt[0, 1] = w.num_blocks + 5  # read by sequence 0 (40 tokens, 3 blocks)
    w2 = W.Workload(**{**w.__dict__, "block_tables": bt})
    with pytest.raises(pa.PagedAttnError) as e:
        gpu_step(pa, w2)
    assert e.value.status == 8
    pa.sync_status()  # the word was cleared
    slots = w.slot_mapping.copy()
    slots[2] = w.num_blocks * w.block_size + 3
    with pytest.raises(pa.PagedAttnError):
        gpu_step(pa, W.Workload(**{**w.__dict__, "slot_mapping": slots}))
    lens = w.context_lens.copy()
    lens[3] = w.max_context_len + 1  # above the stated maximum
    kp, vp = w.k_pool.cuda(), w.v_pool.cuda()
    with pytest.raises(pa.PagedAttnError):
        pa.decode(w.q.cuda(), kp, vp, torch.from_numpy(w.block_tables).cuda(),
                  torch.from_numpy(lens).cuda(), w.scale, w.max_context_len)
        pa.sync_status()
    with pytest.raises(pa.PagedAttnError):
        pa.copy_blocks(kp, vp, torch.tensor([[0, 64]], dtype=torch.int64, device="cuda"))
        pa.sync_status()
    pa.sync_status()


def test_validators_detect_bad_indices(pa):
    s = pa._stream()
    slots = torch.tensor([3, 9, -1, 3], dtype=torch.int64, device="cuda")
    assert pa.pa_validate_slot_mapping(pa._ptr(slots), 4, 4, 16, s) == 6
    slots = torch.tensor([3, 64], dtype=torch.int64, device="cuda")
    assert pa.pa_validate_slot_mapping(pa._ptr(slots), 2, 4, 16, s) == 5
    slots = torch.tensor([3, 63, -5], dtype=torch.int64, device="cuda")
    assert pa.pa_validate_slot_mapping(pa._ptr(slots), 3, 4, 16, s) == 0
    pairs = torch.tensor([[1, 2], [3, 2]], dtype=torch.int64, device="cuda")
    assert pa.pa_validate_copy_pairs(pa._ptr(pairs), 2, 8, s) == 6
    pairs = torch.tensor([[1, 2], [2, 3]], dtype=torch.int64, device="cuda")
    assert pa.pa_validate_copy_pairs(pa._ptr(pairs), 2, 8, s) == 6
    pairs = torch.tensor([[1, 2], [1, 3]], dtype=torch.int64, device="cuda")
    assert pa.pa_validate_copy_pairs(pa._ptr(pairs), 2, 8, s) == 0
    w = small("tiny")
    bt = torch.from_numpy(w.block_tables).cuda()
    cl = torch.from_numpy(w.context_lens).cuda()
    assert pa.pa_validate_block_tables(pa._ptr(bt), bt.shape[1], pa._ptr(cl), 4, 63, 16, 64, s) == 0
    bt[3, 2] = -1
    assert pa.pa_validate_block_tables(pa._ptr(bt), bt.shape[1], pa._ptr(cl), 4, 63, 16, 64, s) == 5


# ---------------------------------------------- benchmark sizes, sampled

def test_benchmark_workload_sampled_against_oracle(pa):
    """The Llama-3-70B-shaped layer at full size (256 x 4096 tokens, bf16)
    in the launch configuration the benchmark times; 12 sequences checked."""
    w = W.make("llama70b_gqa", device="cuda")
    out, _, _ = gpu_step(pa, w)
    seqs = [0, 1, 37, 100, 128, 129, 200, 254, 255, 64, 65, 3]
    ref = compact_oracle_step(w, seqs)
    assert_attention_close(as_f64(out)[seqs], ref, "llama70b_gqa full size")
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("name", ["fp8_longtail_bs16", "fp8_longtail_bs32", "llama13b_mha"])
def test_full_size_workloads_against_oracle(pa, name):
    w = W.make(name, device="cuda")
    out, _, _ = gpu_step(pa, w)
    rng = np.random.default_rng(0)
    seqs = sorted(set(rng.choice(w.num_seqs, size=16, replace=False).tolist()) |
                  {int(np.argmax(w.context_lens))})
    ref = compact_oracle_step(w, seqs)
    assert_attention_close(as_f64(out)[seqs], ref, f"{name} full size")


def test_automatic_split_follows_the_batch_total(pa):
    """With split_tokens == 0 the planning kernel lengthens the ranges to
    about (sum of the lengths) x kv heads / I tokens, I = 15/16 of 148 SMs
    times the kernel's resident blocks per SM, in whole blocks and never
    below pa_decode_split_tokens (which sizes the workspace): on the FP8
    long-tail batch (177,982 tokens, longest 7,305) well above the host's
    1,024.  The length used, left in the workspace, reproduces the output
    bit for bit when passed explicitly."""
    w = W.make("fp8_longtail_bs16", device="cuda")
    dev = "cuda"
    kp, vp = w.k_pool.to(dev).clone(), w.v_pool.to(dev).clone()
    pa.write_kv(w.new_k.to(dev).contiguous(), w.new_v.to(dev).contiguous(),
                torch.from_numpy(w.slot_mapping).to(dev), kp, vp, w.k_scale, w.v_scale)
    q = w.q.to(dev).contiguous()
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    bs = w.block_size
    floor = pa.decode_split_tokens(w.num_seqs, w.num_kv_heads, bs, w.max_context_len)
    nbytes = pa.decode_workspace_size(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, bs,
                                      w.max_context_len)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    out = pa.decode(q, kp, vp, bt, cl, w.scale, w.max_context_len, k_scale=w.k_scale,
                    v_scale=w.v_scale, workspace=ws)
    pa.sync_status()
    used = int(ws[8:12].view(torch.int32).item())
    units = w.num_kv_heads * -(-(w.num_q_heads // w.num_kv_heads) // 8)
    total = int(w.context_lens.sum())

    def rule(per_sm):
        items = 148 * per_sm * 15 // 16
        want = -(-total * units // items)
        return max(floor, min(-(-want // bs), -(-w.max_context_len // bs)) * bs)

    assert floor == 1024 and used > floor
    assert used in {rule(k) for k in range(1, 9)}
    # the work order in the workspace: every sequence cut into
    # n = ceil(len / used) ranges of whole blocks differing by at most one
    # block, none longer than `used`, listed longest first
    B = w.num_seqs
    nranges = int(ws[4:8].view(torch.int32).item()) // units
    off = 256 + -(-(B + 1) * 4 // 256) * 256
    order = ws[off:off + 16 * nranges].view(torch.int32).reshape(-1, 4).cpu().numpy()
    nblk = (order[:, 3] - order[:, 2] + bs - 1) // bs
    assert (np.diff(nblk) <= 0).all()
    for sq in range(B):
        rows = order[order[:, 0] == sq]
        rows = rows[np.argsort(rows[:, 1] & 0xFFFF)]
        n = max(1, -(-int(w.context_lens[sq]) // used))
        assert len(rows) == n and ((rows[:, 1] >> 16) == n).all()
        assert ((rows[:, 1] & 0xFFFF) == np.arange(n)).all()
        assert rows[0, 2] == 0 and rows[-1, 3] == w.context_lens[sq]
        assert (rows[1:, 2] == rows[:-1, 3]).all() and (rows[:, 2] % bs == 0).all()
        nb = (rows[:, 3] - rows[:, 2] + bs - 1) // bs
        assert nb.max() - nb.min() <= 1 and (rows[:, 3] - rows[:, 2] <= used).all()
    again = pa.decode(q, kp, vp, bt, cl, w.scale, w.max_context_len, k_scale=w.k_scale,
                      v_scale=w.v_scale, split_tokens=used)
    pa.sync_status()
    assert torch.equal(again, out)
    seqs = [int(np.argmax(w.context_lens)), 0, 5, 77]
    ref = compact_oracle_step(w, seqs)
    assert_attention_close(as_f64(out)[seqs], ref, "fp8 long tail, lengthened split")


@pytest.mark.parametrize("cache", ["bf16", "e4m3"])
def test_decode_short_contexts_many_sequences(pa, cache):
    """2-8 keys per sequence concentrate the softmax weights, so outputs are
    formed by cancellation between O(1) terms and rounding of the weights
    shows directly; 1024 sequences x 64 heads give many chances to."""
    rng = np.random.default_rng(41)
    lens = rng.integers(2, 9, size=1024)
    w = W._generic("short", lens, 64, 8, 128, 16, "bf16", cache, seed=41, device="cpu")
    out, _, _ = gpu_step(pa, w)
    ref, _, _ = oracle_step(w)
    assert_attention_close(as_f64(out), ref, f"short contexts {cache}")


def test_unplanned_small_batch_equals_the_planned_large_one(pa):
    """A batch whose unsplit items fit the resident CTAs runs without the
    planning kernel (each CTA forms its item from the context length); the
    same sequences inside a batch too large for that go through the plan and
    its work queue.  Both compute each (sequence, kv head) item the same way,
    so the outputs agree bit for bit; the small batch also matches the oracle."""
    rng = np.random.default_rng(43)
    lens = rng.integers(1, 200, size=1000)
    w = W._generic("planned", lens, 32, 8, 128, 16, "bf16", "bf16", seed=43, device="cpu")
    kp, vp = w.k_pool.cuda().clone(), w.v_pool.cuda().clone()
    pa.write_kv(w.new_k.cuda().contiguous(), w.new_v.cuda().contiguous(),
                torch.from_numpy(w.slot_mapping).cuda(), kp, vp, w.k_scale, w.v_scale)
    q = w.q.cuda().contiguous()
    bt = torch.from_numpy(w.block_tables).cuda()
    cl = torch.from_numpy(w.context_lens).cuda()
    B, hq, d = q.shape
    ws_big = torch.zeros(pa.decode_workspace_size(B, hq, 8, d, 16, w.max_context_len), dtype=torch.uint8,
                         device="cuda")
    big = pa.decode(q, kp, vp, bt, cl, w.scale, w.max_context_len, workspace=ws_big)
    pa.sync_status()
    n = 40  # 40 x 8 items: fewer than the resident CTAs
    ws_small = torch.zeros(pa.decode_workspace_size(n, hq, 8, d, 16, w.max_context_len), dtype=torch.uint8,
                           device="cuda")
    small_out = pa.decode(q[:n].contiguous(), kp, vp, bt[:n].contiguous(), cl[:n].contiguous(), w.scale,
                          w.max_context_len, workspace=ws_small)
    pa.sync_status()
    # the plan wrote the item total (byte offset 4); the unplanned call did not
    assert int(ws_big[4:8].view(torch.int32).item()) == B * 8
    assert int(ws_small[4:8].view(torch.int32).item()) == 0
    # both wrote the range length they used (byte offset 8): no split
    assert int(ws_small[8:12].view(torch.int32).item()) >= w.max_context_len
    assert torch.equal(small_out, big[:n])
    ref, _, _ = oracle_step(w, seqs=range(n))
    assert_attention_close(as_f64(small_out), ref[:n], "unplanned small batch")


@pytest.mark.parametrize("hq,hkv,cache,split", [(96, 8, "bf16", 0), (128, 8, "bf16", 64),
                                                (16, 1, "e4m3", 32), (48, 4, "f16", 0)])
def test_decode_more_than_eight_query_heads_per_kv_head(pa, hq, hkv, cache, split):
    """12 and 16 query heads per kv head: the heads are taken 8 at a time, each
    group its own work item over the kv head's blocks (split ranges merged
    per group)."""
    rng = np.random.default_rng(hq + hkv)
    lens = rng.integers(1, 300, size=9)
    qd = "f16" if cache == "f16" else "bf16"
    w = W._generic("wide_groups", lens, hq, hkv, 128, 16, qd, cache, seed=hq, device="cpu")
    out, _, _ = gpu_step(pa, w, split_tokens=split)
    ref, _, _ = oracle_step(w)
    assert_attention_close(as_f64(out), ref, f"{hq}/{hkv} {cache} split {split}")


@pytest.mark.parametrize("name", ["fp8_longtail_bs16", "llama70b_gqa_ragged"])
def test_decode_step_replays_in_a_cuda_graph(pa, name):
    """The step (copy-on-write, write, decode: the planning kernel and the
    attention kernel launched behind it) captured once in a CUDA graph and
    replayed on fresh pools gives the bytes of the direct calls."""
    w = small(name)
    direct, dkp, dvp = gpu_step(pa, w)
    k0, v0 = w.k_pool.cuda().clone(), w.v_pool.cuda().clone()
    kp, vp = k0.clone(), v0.clone()
    q = w.q.cuda().contiguous()
    nk, nv = w.new_k.cuda().contiguous(), w.new_v.cuda().contiguous()
    slots = torch.from_numpy(w.slot_mapping).cuda()
    tables = torch.from_numpy(w.block_tables).cuda()
    lens = torch.from_numpy(w.context_lens).cuda()
    pairs = torch.from_numpy(w.cow_pairs).cuda() if len(w.cow_pairs) else None
    out = torch.empty_like(q)
    B, hq, d = q.shape
    _, bs, hkv, _ = kp.shape
    ws = torch.empty(max(256, pa.decode_workspace_size(B, hq, hkv, d, bs, w.max_context_len, 0)),
                     dtype=torch.uint8, device="cuda")

    def step():
        if pairs is not None:
            pa.copy_blocks(kp, vp, pairs)
        pa.write_kv(nk, nv, slots, kp, vp, w.k_scale, w.v_scale)
        pa.decode(q, kp, vp, tables, lens, w.scale, w.max_context_len, k_scale=w.k_scale,
                  v_scale=w.v_scale, out=out, workspace=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    pa.sync_status()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        kp.copy_(k0)
        vp.copy_(v0)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        pa.sync_status()
        assert torch.equal(out, direct)
        assert torch.equal(kp.view(torch.uint8), dkp.view(torch.uint8))
        assert torch.equal(vp.view(torch.uint8), dvp.view(torch.uint8))
    del g
