"""Closed-form memory arithmetic that the pages print.

TEST INFRASTRUCTURE ONLY (see the package docstring).

* KV bytes: every layer keeps, per token, one key and one value vector per KV
  head ("PagedAttention", Ultralytics glossary, §Çözdüğü Bellek Sorunu, which
  puts one LLaMA-13B sequence at up to 1.7 GB; gyaansetu, §مشکل حافظه, which
  puts one 4096-token Llama-3.1-70B sequence near 1.3 GB).
* Unused slots: a contiguous reservation wastes ``reserved - used`` slots
  (the sketch's 2008 of 2048; gyaansetu's 950 of 1000 and 93% of 4096 when
  300 are used); paging wastes only the unfilled tail of the last block
  (the sketch's 8 for 40 tokens in blocks of 16).
"""

from __future__ import annotations

import numpy as np


def blocks_needed(num_tokens: int, block_size: int) -> int:
    """ceil(num_tokens / block_size): blocks a request of that length holds."""
    return -(-int(num_tokens) // int(block_size))


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """K and V of one token over all layers: layers * 2 * Hkv * D * e bytes."""
    return int(num_layers) * 2 * int(num_kv_heads) * int(head_dim) * int(elem_bytes)


def kv_bytes(num_tokens: int, num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """KV-cache bytes of a sequence of ``num_tokens`` tokens."""
    return int(num_tokens) * kv_bytes_per_token(num_layers, num_kv_heads, head_dim, elem_bytes)


def reservation_unused_slots(used: int, reserved: int) -> int:
    """Slots left empty by one contiguous reservation of ``reserved`` tokens."""
    return int(reserved) - int(used)


def paged_unused_slots(context_lens, block_size: int) -> int:
    """Slots left empty by paging: the unfilled tail of each last block."""
    lens = np.asarray(context_lens, dtype=np.int64)
    nb = -(-lens // int(block_size))
    return int((nb * int(block_size) - lens).sum())
