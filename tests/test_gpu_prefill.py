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


def test_prefill_rejects_unsupported_shapes(pa):
    pw = W.prefill(ctxs=(40,), nqs=(40,), hq=12, hkv=4, bs=16, dtype="bf16")  # G = 3
    with pytest.raises(pa.PagedAttnError) as e:
        run(pa, pw)
    assert e.value.status == 4
