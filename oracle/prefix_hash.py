"""Chained block hashes for prefix caching, in plain Python integers.

TEST INFRASTRUCTURE ONLY (see the package docstring).

"PagedAttention" (Ultralytics glossary), §Diziler Arasında Blokları Paylaşma:
taking a hash of every block carries block sharing across requests, which
is how vLLM implements prompt caching.  The pages name no hash function, so
the reading taken here is:

* a block is hashed only when it is full (bs tokens);
* its hash covers its own token ids AND its parent block's hash, so two
  blocks hash equal only when the whole prefix up to them is equal;
* the hash is 64-bit FNV-1a (Fowler / Noll / Vo; offset basis
  0xcbf29ce484222325, prime 0x100000001b3, per byte: xor, then multiply
  mod 2^64), restated here from its published definition;
* inner_j = FNV-1a over the block's token ids, each as 4 little-endian bytes
  of its int32 value; hash_j = FNV-1a over (hash_{j-1} as 8 little-endian
  bytes, then inner_j as 8 little-endian bytes), with hash_{-1} = 0.

Pins: the FNV-1a-64 test vectors of its specification (empty string, "a",
"foobar"), and the chain's properties (equal prefixes hash equal, one changed
token changes its block and every later one, placement does not matter).
"""

from __future__ import annotations

import numpy as np

FNV64_OFFSET = 0xCBF29CE484222325
FNV64_PRIME = 0x100000001B3
MASK64 = (1 << 64) - 1


def fnv1a64(data: bytes, h: int = FNV64_OFFSET) -> int:
    for b in data:
        h ^= b
        h = (h * FNV64_PRIME) & MASK64
    return h


def block_hashes(token_ids, num_tokens: int, block_size: int) -> list:
    """Hashes of the full blocks of one sequence, in logical order."""
    toks = np.asarray(token_ids, dtype=np.int64)[: int(num_tokens)]
    out = []
    parent = 0
    for j in range(int(num_tokens) // block_size):
        chunk = toks[j * block_size:(j + 1) * block_size]
        inner = fnv1a64(b"".join(int(t & 0xFFFFFFFF).to_bytes(4, "little") for t in chunk))
        parent = fnv1a64(parent.to_bytes(8, "little") + inner.to_bytes(8, "little"))
        out.append(parent)
    return out
