"""Plain fp64 CPU oracle for the paged decode-attention hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import anything under ``oracle/``.  The product package
(``paged_kv_cache_416_b200``) never imports it, and this package imports
nothing from the product: the two share no code.  Inputs reach both sides
from the seeded generators in ``paged_kv_cache_416_b200.workloads``, which
hold none of the method's arithmetic.

What is computed, and where the pages define it
-----------------------------------------------
Sources are three web pages on PagedAttention:

* "PagedAttention" (Ultralytics glossary, Turkish), sections
  "Çözdüğü Bellek Sorunu" (the memory problem), "Sayfalama Nasıl Çalışır"
  (how paging works, with a PyTorch sketch of a block pool, a free list,
  a block table, slot writes and a gather), "Diziler Arasında Blokları
  Paylaşma" (sharing blocks, copy-on-write) and "İlgili Teknikler"
  (FlashAttention-style kernels, grouped-query attention, FP8 caches).
* "حافظه KV و PagedAttention" (gyaansetu, Persian), sections "مشکل حافظه"
  (memory arithmetic) and the fragmentation sections of its second article.

The method reaches exactly the plain softmax-attention result through a
different memory layout, so the oracle is that plain definition written
out (``paged.decode``): gather every sequence's blocks into a contiguous
fp64 cache through its block table, then run naive softmax attention.

Pins (tests/test_oracle_pins.py, all ``-m "not gpu"``):
every function here is pinned to something other than itself -- the
pages' worked example, closed forms, a library routine, brute force or an
exhaustive enumeration.  No function is "parity unpinned".
"""

from .codecs import (
    bf16_bits_to_f64,
    f16_bits_to_f64,
    e4m3_decode,
    e4m3_encode_f32,
    e4m3_finite_values,
    decode_cache,
)
from .paged import (
    slot_of,
    write_kv,
    copy_blocks,
    swap_blocks,
    gather,
    attention_weights,
    decode,
    decode_one,
    prefill,
    shared_prefix_blocks,
    partial_attention,
    merge_partials,
    shared_prefix_decode,
)
from .memory import (
    kv_bytes_per_token,
    kv_bytes,
    reservation_unused_slots,
    paged_unused_slots,
    blocks_needed,
)

__all__ = [
    "bf16_bits_to_f64", "f16_bits_to_f64", "e4m3_decode", "e4m3_encode_f32",
    "e4m3_finite_values", "decode_cache", "slot_of", "write_kv", "copy_blocks",
    "swap_blocks", "gather", "attention_weights", "decode", "decode_one", "prefill", "kv_bytes_per_token",
    "kv_bytes", "reservation_unused_slots", "paged_unused_slots", "blocks_needed",
    "shared_prefix_blocks", "partial_attention", "merge_partials", "shared_prefix_decode",
]
