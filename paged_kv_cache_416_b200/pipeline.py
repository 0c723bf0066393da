"""Decode steps fed from host memory, with the copies overlapped.

A serving loop keeps each step's inputs on the host (query vectors, the new
tokens' K/V, the slot mapping, block tables, context lengths, copy-on-write
pairs) and needs each step's output back on the host.  ``DecodePipeline``
runs step n's device work (pa_copy_blocks, pa_write_kv, pa_decode) on the
compute stream while one copy stream moves step n+1's inputs in and another
moves step n-1's output out.  Two device buffer sets alternate, and events
keep every copy off the memory a running step uses:

* inputs of step n go into set n % 2 once step n-2 (the set's last user)
  has finished;
* step n starts once its inputs have arrived and step n-2's output has been
  read out of the set's output buffer;
* step n's output is read back once step n has finished.

Every step still moves all of its inputs in and its output out; only their
order relative to the device work of other steps changes.  The cache pools
and the decode workspace are shared by all steps, whose device work stays in
order on the compute stream.
"""

from __future__ import annotations

from typing import Dict, Optional

import torch

from . import pagedattn as pa

INPUTS = ("q", "new_k", "new_v", "slots", "tables", "lens", "pairs")


class DecodePipeline:
    def __init__(self, k_pool: torch.Tensor, v_pool: torch.Tensor, scale: float,
                 max_context_len: int, k_scale: float = 1.0, v_scale: float = 1.0,
                 workspace: Optional[torch.Tensor] = None):
        self.kp, self.vp = k_pool, v_pool
        self.scale, self.max_ctx = float(scale), int(max_context_len)
        self.k_scale, self.v_scale = float(k_scale), float(v_scale)
        self.device = k_pool.device
        self.workspace = workspace
        self.compute = torch.cuda.current_stream(self.device)
        self.h2d = torch.cuda.Stream(self.device)
        self.d2h = torch.cuda.Stream(self.device)
        self.sets = [None, None]
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]
        self.in_ready, self.step_done, self.out_read = ev(), ev(), ev()
        self.n = 0

    def _set(self, b: int, host: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
        if self.sets[b] is None:
            bufs = {k: torch.empty_like(t, device=self.device) for k, t in host.items()}
            bufs["out"] = torch.empty_like(bufs["q"])
            self.sets[b] = bufs
        return self.sets[b]

    def start_after(self, event: torch.cuda.Event) -> None:
        """Order the copy streams' next work after `event` (e.g. a timer)."""
        self.h2d.wait_event(event)
        self.d2h.wait_event(event)

    def submit(self, host: Dict[str, torch.Tensor], out_host: torch.Tensor) -> None:
        """Enqueue one step.  `host` maps the names in INPUTS to pinned CPU
        tensors ("pairs" may be absent or empty); `out_host` is a pinned CPU
        tensor of q's shape that receives the step's output."""
        b = self.n % 2
        bufs = self._set(b, host)
        if self.n >= 2:  # the set's previous step has finished with its inputs
            self.h2d.wait_event(self.step_done[b])
        with torch.cuda.stream(self.h2d):
            for k, t in host.items():
                if t.numel():
                    bufs[k].copy_(t, non_blocking=True)
        self.in_ready[b].record(self.h2d)
        self.compute.wait_event(self.in_ready[b])
        if self.n >= 2:  # and its output has been read back
            self.compute.wait_event(self.out_read[b])
        with torch.cuda.stream(self.compute):
            pairs = bufs.get("pairs")
            if pairs is not None and pairs.numel():
                pa.copy_blocks(self.kp, self.vp, pairs)
            pa.write_kv(bufs["new_k"], bufs["new_v"], bufs["slots"], self.kp, self.vp,
                        self.k_scale, self.v_scale)
            pa.decode(bufs["q"], self.kp, self.vp, bufs["tables"], bufs["lens"], self.scale,
                      self.max_ctx, k_scale=self.k_scale, v_scale=self.v_scale, out=bufs["out"],
                      workspace=self.workspace)
        self.step_done[b].record(self.compute)
        self.d2h.wait_event(self.step_done[b])
        with torch.cuda.stream(self.d2h):
            out_host.copy_(bufs["out"], non_blocking=True)
        self.out_read[b].record(self.d2h)
        self.n += 1

    def drain(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Make `stream` (default: the compute stream) wait for every copy
        submitted so far."""
        s = self.compute if stream is None else stream
        s.wait_event(self.out_read[(self.n - 1) % 2])
        if self.n >= 2:
            s.wait_event(self.out_read[self.n % 2])
