"""pa_swap_blocks: blocks moved between the device pool and pinned host
memory in one launch, bit-exact against the oracle's indexed copy."""

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_416_b200 import workloads as W
from paged_kv_cache_416_b200.workloads import raw

pytestmark = pytest.mark.gpu


def _pool(n, bs, hkv, d, dt, gen, device="cpu"):
    if dt == "e4m3":
        return torch.randint(0, 255, (n, bs, hkv, d), generator=gen, dtype=torch.uint8).view(torch.float8_e4m3fn).to(device)
    return torch.randint(-30000, 30000, (n, bs, hkv, d), generator=gen, dtype=torch.int16).view(W.TORCH_DTYPE[dt]).to(device)


@pytest.mark.parametrize("dt,bs,hkv,d", [("bf16", 16, 8, 128), ("e4m3", 32, 8, 128), ("f16", 16, 4, 64)])
def test_swap_out_then_in_is_bit_exact(pa, dt, bs, hkv, d):
    g = torch.Generator().manual_seed(11)
    dev_k, dev_v = _pool(300, bs, hkv, d, dt, g, "cuda"), _pool(300, bs, hkv, d, dt, g, "cuda")
    host_k, host_v = _pool(120, bs, hkv, d, dt, g).pin_memory(), _pool(120, bs, hkv, d, dt, g).pin_memory()
    src = torch.randperm(300, generator=g)[:100]
    dst = torch.randperm(120, generator=g)[:100]
    out_pairs = torch.stack([src, dst], 1).to(torch.int64)
    ok_, ov_ = raw(host_k).copy(), raw(host_v).copy()
    oracle.swap_blocks(raw(dev_k), raw(dev_v), ok_, ov_, out_pairs.numpy())
    pa.swap_blocks(dev_k, dev_v, host_k, host_v, out_pairs.cuda())
    pa.sync_status()
    assert np.array_equal(raw(host_k), ok_) and np.array_equal(raw(host_v), ov_)
    # back in, to other device slots
    back = torch.randperm(300, generator=g)[:100]
    in_pairs = torch.stack([dst, back], 1).to(torch.int64)
    dk, dv = raw(dev_k).copy(), raw(dev_v).copy()
    oracle.swap_blocks(raw(host_k), raw(host_v), dk, dv, in_pairs.numpy())
    pa.swap_blocks(host_k, host_v, dev_k, dev_v, in_pairs.cuda())
    pa.sync_status()
    assert np.array_equal(raw(dev_k), dk) and np.array_equal(raw(dev_v), dv)


def test_swapped_blocks_decode_like_the_originals(pa):
    """Evict every block of a workload to host memory and back into new
    device slots (tables remapped): the decode output is bit-identical."""
    w = W.make("fp8_longtail_bs16", num_seqs=6, max_len=3000)
    dev_k, dev_v = w.k_pool.cuda(), w.v_pool.cuda()
    bt = torch.from_numpy(w.block_tables).cuda()
    cl = torch.from_numpy(w.context_lens).cuda()
    ref = pa.decode(w.q.cuda(), dev_k, dev_v, bt, cl, w.scale, w.max_context_len,
                    k_scale=w.k_scale, v_scale=w.v_scale)
    N = w.num_blocks
    host_k = torch.empty((N,) + tuple(w.k_pool.shape[1:]), dtype=w.k_pool.dtype).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    ids = torch.arange(N, dtype=torch.int64)
    pa.swap_blocks(dev_k, dev_v, host_k, host_v, torch.stack([ids, ids], 1).cuda())
    new_k, new_v = torch.zeros_like(dev_k), torch.zeros_like(dev_v)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(5))
    pa.swap_blocks(host_k, host_v, new_k, new_v, torch.stack([ids, perm], 1).cuda())
    bt2 = w.block_tables.copy()
    m = bt2 >= 0
    bt2[m] = perm.numpy()[bt2[m]]
    out = pa.decode(w.q.cuda(), new_k, new_v, torch.from_numpy(bt2).cuda(), cl, w.scale,
                    w.max_context_len, k_scale=w.k_scale, v_scale=w.v_scale)
    pa.sync_status()
    assert torch.equal(out, ref)


def test_pageable_host_memory_is_refused(pa):
    dev = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    pageable = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    with pytest.raises(pa.PagedAttnError) as e:
        pa.swap_blocks(dev, dev.clone(), pageable, pageable.clone(), pairs)
    assert e.value.status == 11
    with pytest.raises(pa.PagedAttnError):
        pa.swap_blocks(dev, dev.clone(), dev.clone(), dev.clone(),
                       torch.tensor([[0, 9]], dtype=torch.int64, device="cuda"))
        pa.sync_status()


def test_swap_benchmark_size_bit_exact(pa):
    """The benchmark's swap: 2048 scattered blocks of an 8192-block bf16
    pool (bs 16, 8 kv heads, D 128) out to pinned host memory and back into
    their original slots, byte for byte against the oracle's indexed copy."""
    nb, n_dev, shape = 2048, 8192, (16, 8, 128)
    g = torch.Generator().manual_seed(3)
    dev_k = torch.randint(-30000, 30000, (n_dev,) + shape, generator=g, dtype=torch.int16).view(torch.bfloat16).cuda()
    dev_v = torch.randint(-30000, 30000, (n_dev,) + shape, generator=g, dtype=torch.int16).view(torch.bfloat16).cuda()
    host_k = torch.zeros((nb,) + shape, dtype=torch.bfloat16).pin_memory()
    host_v = torch.zeros((nb,) + shape, dtype=torch.bfloat16).pin_memory()
    src = torch.randperm(n_dev, generator=g)[:nb]
    dst = torch.randperm(nb, generator=g)
    out_pairs = torch.stack([src, dst], 1).to(torch.int64)
    dk0, dv0 = raw(dev_k), raw(dev_v)
    hk, hv = raw(host_k).copy(), raw(host_v).copy()
    oracle.swap_blocks(dk0, dv0, hk, hv, out_pairs.numpy())
    pa.swap_blocks(dev_k, dev_v, host_k, host_v, out_pairs.cuda())
    pa.sync_status()
    assert np.array_equal(raw(host_k), hk) and np.array_equal(raw(host_v), hv)
    dev_k[src.cuda()] = 0  # evicted
    dev_v[src.cuda()] = 0
    in_pairs = torch.stack([dst, src], 1).to(torch.int64)
    pa.swap_blocks(host_k, host_v, dev_k, dev_v, in_pairs.cuda())
    pa.sync_status()
    assert np.array_equal(raw(dev_k), dk0) and np.array_equal(raw(dev_v), dv0)
