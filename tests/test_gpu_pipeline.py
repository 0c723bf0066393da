"""DecodePipeline (host-fed steps with overlapped copies) gives exactly the
outputs of the same calls made one after another."""

import numpy as np
import pytest
import torch

from paged_kv_cache_416_b200 import workloads as W
from paged_kv_cache_416_b200.pipeline import DecodePipeline

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["shared_prefix_fork", "fp8_longtail_bs16"])
def test_pipeline_matches_direct_calls(pa, name):
    w = W.make(name, **({"prompts": 3} if name.startswith("shared") else {"num_seqs": 12}))
    dev = torch.device("cuda", 0)
    kp, vp = w.k_pool.to(dev).clone(), w.v_pool.to(dev).clone()
    host = {"q": w.q, "new_k": w.new_k, "new_v": w.new_v,
            "slots": torch.from_numpy(w.slot_mapping), "tables": torch.from_numpy(w.block_tables),
            "lens": torch.from_numpy(w.context_lens), "pairs": torch.from_numpy(w.cow_pairs)}
    host = {k: t.contiguous().pin_memory() for k, t in host.items()}
    # direct: one step (the step is idempotent: the same writes every time)
    kd, vd = kp.clone(), vp.clone()
    if len(w.cow_pairs):
        pa.copy_blocks(kd, vd, host["pairs"].to(dev))
    pa.write_kv(host["new_k"].to(dev), host["new_v"].to(dev), host["slots"].to(dev), kd, vd,
                w.k_scale, w.v_scale)
    ref = pa.decode(host["q"].to(dev), kd, vd, host["tables"].to(dev), host["lens"].to(dev),
                    w.scale, w.max_context_len, k_scale=w.k_scale, v_scale=w.v_scale)
    pa.sync_status()
    pipe = DecodePipeline(kp, vp, w.scale, w.max_context_len, w.k_scale, w.v_scale)
    outs = [torch.empty(ref.shape, dtype=ref.dtype, pin_memory=True) for _ in range(2)]
    for i in range(5):
        pipe.submit(host, outs[i % 2])
    pipe.drain()
    torch.cuda.synchronize()
    pa.sync_status()
    for o in outs:
        assert torch.equal(o, ref.cpu()), f"{name}: pipelined output differs"
    # the pools hold NaN poison in unused slots: compare their bytes
    raw = lambda t: t.contiguous().view(torch.uint8).cpu()
    assert torch.equal(raw(kp), raw(kd)) and torch.equal(raw(vp), raw(vd))
