"""Chained block hashes for prefix caching: the oracle pinned to the FNV-1a
specification's vectors and to the chain's properties; the host allocator's
prefix reuse; and (GPU) pa_hash_blocks bit-exact against the oracle."""

import json
import os

import numpy as np
import pytest
import torch

from oracle.prefix_hash import block_hashes, fnv1a64
from paged_kv_cache_416_b200.alloc import BlockAllocator

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fnv1a64_vectors.json")


def test_fnv1a64_matches_the_specification_vectors():
    g = json.load(open(GOLDEN))
    for v in g["vectors"]:
        assert fnv1a64(v["input"].encode()) == int(v["fnv1a64"], 16)


def test_chain_properties():
    rng = np.random.default_rng(1)
    bs = 16
    a = rng.integers(0, 50000, size=200)
    b = a.copy()
    b[100] += 1                     # token 100 lives in block 6
    ha, hb = block_hashes(a, 200, bs), block_hashes(b, 200, bs)
    assert len(ha) == 200 // bs == 12
    assert ha[:6] == hb[:6]         # equal prefixes hash equal
    assert all(x != y for x, y in zip(ha[6:], hb[6:]))  # the change and every later block differ
    # a block's hash depends on its parent: same tokens after a different prefix differ
    c = np.concatenate([a[16:32], a[16:32]])
    hc = block_hashes(c, 32, bs)
    assert hc[0] != hc[1]
    # ragged tail: only full blocks are hashed
    assert block_hashes(a, 47, bs) == ha[:2]
    assert block_hashes(a, 15, bs) == []


def test_allocator_reuses_cached_prefix_blocks():
    bs = 4
    alloc = BlockAllocator(32, bs)
    prompt = list(range(100, 114))                # 14 tokens: 3 full blocks + 2
    alloc.allocate(0, len(prompt))
    alloc.register_prefix(0, block_hashes(prompt, len(prompt), bs))
    other = prompt[:8] + [7, 7, 7, 7, 7]          # shares the first 2 blocks
    table, shared = alloc.allocate_cached(1, len(other), block_hashes(other, len(other), bs))
    assert shared == 2 and table[:2] == alloc.tables[0][:2]
    assert table[2:] != alloc.tables[0][2:4]
    assert alloc.refcount[alloc.tables[0][0]] == 2
    # a write into a shared block would copy it first (copy-on-write)
    alloc.free_seq(0)
    assert alloc.refcount[table[0]] == 1 and len(alloc.cached) == 2
    alloc.free_seq(1)
    assert alloc.used_blocks() == 0 and not alloc.cached


@pytest.mark.gpu
def test_gpu_block_hashes_match_the_oracle(pa):
    rng = np.random.default_rng(5)
    B, L, bs = 9, 700, 16
    toks = rng.integers(-2**31, 2**31 - 1, size=(B, L), dtype=np.int64).astype(np.int32)
    toks[7, :320] = toks[5, :320]                 # a shared 20-block prefix
    lens = np.array([700, 333, 16, 15, 0, 640, 17, 512, 699], dtype=np.int32)
    got = pa.hash_blocks(torch.from_numpy(toks).cuda(), torch.from_numpy(lens).cuda(), bs,
                         max_blocks=L // bs)
    pa.sync_status()
    got = got.cpu().numpy().view(np.uint64)
    for s in range(B):
        ref = block_hashes(toks[s].astype(np.int64), int(lens[s]), bs)
        assert [int(x) for x in got[s, :len(ref)]] == ref
        assert not got[s, len(ref):].any()
    assert (got[7, :20] == got[5, :20]).all() and got[7, 20] != got[5, 20]


@pytest.mark.gpu
@pytest.mark.parametrize("bs", [16, 32])
def test_gpu_block_hashes_across_chunks_of_256_blocks(pa, bs):
    # the kernel hashes a sequence's blocks 256 at a time: exactly one
    # chunk, one block past it, several chunks, and a ragged tail
    rng = np.random.default_rng(6)
    full = [256, 257, 600, 3]
    L = max(full) * bs + bs
    toks = rng.integers(-2**31, 2**31 - 1, size=(len(full), L), dtype=np.int64).astype(np.int32)
    lens = np.array([f * bs + (s % 2) * (bs - 1) for s, f in enumerate(full)], dtype=np.int32)
    got = pa.hash_blocks(torch.from_numpy(toks).cuda(), torch.from_numpy(lens).cuda(), bs,
                         max_blocks=L // bs)
    pa.sync_status()
    got = got.cpu().numpy().view(np.uint64)
    for s in range(len(full)):
        ref = block_hashes(toks[s].astype(np.int64), int(lens[s]), bs)
        assert len(ref) == full[s]
        assert [int(x) for x in got[s, :len(ref)]] == ref
        assert not got[s, len(ref):].any()


def test_planted_unchained_hash_is_caught(monkeypatch):
    """A block hash that leaves out its parent (each block hashed alone) fails
    the chain pin: equal blocks after different prefixes would hash equal."""
    import oracle.prefix_hash as ph

    def unchained(token_ids, num_tokens, block_size):
        toks = np.asarray(token_ids, dtype=np.int64)[: int(num_tokens)]
        return [fnv1a64(b"".join(int(t & 0xFFFFFFFF).to_bytes(4, "little")
                                 for t in toks[j * block_size:(j + 1) * block_size]))
                for j in range(int(num_tokens) // block_size)]
    monkeypatch.setitem(globals(), "block_hashes", unchained)
    monkeypatch.setattr(ph, "block_hashes", unchained)
    with pytest.raises(AssertionError):
        test_chain_properties()
