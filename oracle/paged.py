"""The paged KV cache and decode attention, written out plainly in fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Layouts (the pages' sketch keeps ``key_pool[block, slot, dim]`` for one
head; the head axis is inserted before the dimension axis):

* pools:        raw words ``[num_blocks, block_size, num_kv_heads, head_dim]``
* block_tables: int ``[num_seqs, max_blocks_per_seq]``, logical block i of a
  sequence lives in physical block ``block_tables[s, i]``
* q:            raw words ``[num_seqs, num_q_heads, head_dim]``
* new k / v:    raw words ``[num_tokens, num_kv_heads, head_dim]``
* slot_mapping: int ``[num_tokens]``, slot = physical_block * block_size + offset

Sources: "PagedAttention" (Ultralytics glossary), §Sayfalama Nasıl Çalışır
and its PyTorch sketch (slot writes through the block table, the gather
``key_pool[block_table].reshape(-1, D)[:len]``), §Diziler Arasında Blokları
Paylaşma (several tables may name one physical block; a block still used by
others is copied before it is written), §İlgili Teknikler (grouped-query
attention shares K/V heads among query heads).
"""

from __future__ import annotations

import numpy as np

from .codecs import decode_cache, e4m3_encode_f32, f16_bits_to_f64, bf16_bits_to_f64


def slot_of(block_table, pos: int, block_size: int) -> int:
    """Slot of token position ``pos``: its logical block's physical id times
    the block size, plus the offset inside the block (the sketch's write
    ``key_pool[block_table[pos // block_size], pos % block_size]``)."""
    return int(block_table[pos // block_size]) * block_size + pos % block_size


def write_kv(k_raw, v_raw, in_dtype: str, slot_mapping, k_pool, v_pool,
             cache_dtype: str, k_scale: float = 1.0, v_scale: float = 1.0):
    """Scatter new tokens into the pools, in place; returns (k_pool, v_pool).

    For each token t with slot >= 0: ``pool[slot // bs, slot % bs] = x[t]``.
    A negative slot marks a padding token and is skipped.  For a 16-bit cache
    the input words are stored unchanged (the cache dtype must equal the
    input dtype); for an e4m3 cache each element is quantised as
    ``e4m3(fp32(x) / fp32(scale))`` (see ``codecs``).
    """
    bs = k_pool.shape[1]
    slot_mapping = np.asarray(slot_mapping, dtype=np.int64)
    if cache_dtype == "e4m3":
        to_f64 = f16_bits_to_f64 if in_dtype == "f16" else bf16_bits_to_f64
        k_val = to_f64(k_raw).astype(np.float32)  # exact: 16-bit -> fp32
        v_val = to_f64(v_raw).astype(np.float32)
        k_enc = e4m3_encode_f32(k_val / np.float32(k_scale))
        v_enc = e4m3_encode_f32(v_val / np.float32(v_scale))
    else:
        if cache_dtype != in_dtype:
            raise ValueError("a 16-bit cache stores its input words unchanged")
        k_enc, v_enc = np.asarray(k_raw), np.asarray(v_raw)
    for t, slot in enumerate(slot_mapping):
        if slot < 0:
            continue
        b, o = divmod(int(slot), bs)
        k_pool[b, o] = k_enc[t]
        v_pool[b, o] = v_enc[t]
    return k_pool, v_pool


def copy_blocks(k_pool, v_pool, pairs):
    """Copy-on-write block copy, in place: ``pool[dst] = pool[src]`` for every
    (src, dst) pair, for K and V.  All pairs read the state before any copy."""
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    k_src = k_pool.copy()
    v_src = v_pool.copy()
    for src, dst in pairs:
        k_pool[dst] = k_src[src]
        v_pool[dst] = v_src[src]
    return k_pool, v_pool


def swap_blocks(src_k, src_v, dst_k, dst_v, pairs):
    """Move blocks between two pools, in place on the destination:
    ``dst[d] = src[s]`` for every (s, d) pair, for K and V (gyaansetu, first
    article: fine-grained eviction moves small pages, not whole sequences,
    to the CPU when memory is full)."""
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    for src, dst in pairs:
        dst_k[dst] = src_k[src]
        dst_v[dst] = src_v[src]
    return dst_k, dst_v


def gather(pool_values, block_table_row, context_len: int) -> np.ndarray:
    """A sequence's contiguous cache ``[context_len, H, D]`` from its blocks:
    the blocks named by the first ceil(len / bs) table entries, concatenated
    in logical order and cut to ``context_len`` tokens.  Entries past those
    are never read."""
    bs = pool_values.shape[1]
    nb = -(-int(context_len) // bs)
    ids = np.asarray(block_table_row[:nb], dtype=np.int64)
    blocks = pool_values[ids]  # [nb, bs, H, D]
    return blocks.reshape(nb * bs, *pool_values.shape[2:])[:context_len]


def attention_weights(q_vec: np.ndarray, keys: np.ndarray, scale: float) -> np.ndarray:
    """Softmax weights of one query against ``keys [n, D]``, fp64:
    ``w = exp(z - max z) / sum exp(z - max z)`` with ``z = scale * keys @ q``."""
    z = float(scale) * (keys @ q_vec)
    z = z - z.max()
    e = np.exp(z)
    return e / e.sum()


def decode_one(q_f64: np.ndarray, k_vals: np.ndarray, v_vals: np.ndarray,
               table_row, context_len: int, scale: float, num_kv_heads: int) -> np.ndarray:
    """Decode attention of one sequence: ``q_f64 [Hq, D]`` against the
    decoded pools -> ``[Hq, D]`` fp64.  Query head h reads KV head
    ``h // (Hq / Hkv)`` (consecutive grouping).  An empty context gives 0."""
    hq, d = q_f64.shape
    out = np.zeros((hq, d), dtype=np.float64)
    if context_len <= 0:
        return out
    group = hq // num_kv_heads
    K = gather(k_vals, table_row, context_len)  # [n, Hkv, D]
    V = gather(v_vals, table_row, context_len)
    for h in range(hq):
        kv = h // group
        w = attention_weights(q_f64[h], K[:, kv, :], scale)
        out[h] = w @ V[:, kv, :]
    return out


def decode(q_raw, q_dtype: str, k_pool, v_pool, cache_dtype: str, block_tables,
           context_lens, scale: float, num_kv_heads: int,
           k_scale: float = 1.0, v_scale: float = 1.0, seqs=None) -> np.ndarray:
    """Paged decode attention for every sequence (or the listed ``seqs``).

    Returns fp64 ``[num_seqs, Hq, D]`` (rows not listed in ``seqs`` are 0).
    Only the blocks each sequence names are decoded, so a large pool with a
    small sample of sequences stays cheap.
    """
    q = decode_cache(q_raw, q_dtype)
    B, hq, d = q.shape
    out = np.zeros((B, hq, d), dtype=np.float64)
    bs = k_pool.shape[1]
    seqs = range(B) if seqs is None else seqs
    for s in seqs:
        n = int(context_lens[s])
        if n <= 0:
            continue
        nb = -(-n // bs)
        ids = np.asarray(block_tables[s][:nb], dtype=np.int64)
        # decode only this sequence's blocks; renumber them 0..nb-1
        kv_k = decode_cache(k_pool[ids], cache_dtype, k_scale)
        kv_v = decode_cache(v_pool[ids], cache_dtype, v_scale)
        out[s] = decode_one(q[s], kv_k, kv_v, np.arange(nb), n, scale, num_kv_heads)
    return out


def prefill(q_raw, q_dtype: str, k_pool, v_pool, cache_dtype: str, block_tables, context_lens,
            query_start, scale: float, num_kv_heads: int, k_scale: float = 1.0,
            v_scale: float = 1.0, seqs=None) -> np.ndarray:
    """Paged prefill (chunked prefill) attention, fp64.

    Sequence s has ``n = query_start[s+1] - query_start[s]`` new query tokens
    ``q[query_start[s] + i]`` at positions ``context_lens[s] - n + i`` (their
    K/V already in the cache).  Token i attends causally to cached tokens
    0..its position, gathered through the block table ("PagedAttention",
    §İlgili Teknikler: FlashAttention-style kernels read the paged blocks).
    Returns ``[total_q, Hq, D]``; rows of sequences not in ``seqs`` are 0.
    """
    q = decode_cache(q_raw, q_dtype)
    total, hq, d = q.shape
    out = np.zeros((total, hq, d), dtype=np.float64)
    bs = k_pool.shape[1]
    group = hq // num_kv_heads
    qs = np.asarray(query_start, dtype=np.int64)
    seqs = range(len(qs) - 1) if seqs is None else seqs
    for s in seqs:
        n = int(qs[s + 1] - qs[s])
        ctx = int(context_lens[s])
        if n <= 0 or ctx <= 0:
            continue
        nb = -(-ctx // bs)
        ids = np.asarray(block_tables[s][:nb], dtype=np.int64)
        K = gather(decode_cache(k_pool[ids], cache_dtype, k_scale), np.arange(nb), ctx)
        V = gather(decode_cache(v_pool[ids], cache_dtype, v_scale), np.arange(nb), ctx)
        for i in range(n):
            nk = visible_keys(ctx, n, i)
            for h in range(hq):
                kv = h // group
                w = attention_weights(q[qs[s] + i, h], K[:nk, kv, :], scale)
                out[qs[s] + i, h] = w @ V[:nk, kv, :]
    return out


def visible_keys(context_len: int, num_new: int, i: int) -> int:
    """Keys new token i of a chunk of ``num_new`` sees: it sits at position
    ``context_len - num_new + i`` (the chunk is the end of the context) and
    attends causally to positions 0 .. that position."""
    return context_len - num_new + i + 1


def shared_prefix_blocks(block_tables, context_lens, members, block_size: int) -> int:
    """Blocks a group of sequences shares at the head of their tables: the
    longest run of leading table entries equal in every member's row, cut
    so that each member keeps at least one token of its own (the prefix
    lies inside every member's context and ends before its last token).
    A group of fewer than two members shares nothing.

    ("PagedAttention", §Diziler Arasında Blokları Paylaşma: sequences forked
    from one prompt -- parallel sampling, beam search, a common prompt --
    name the same physical blocks in their tables.)"""
    members = [int(m) for m in members]
    if len(members) < 2:
        return 0
    limit = min((int(context_lens[m]) - 1) // block_size for m in members)
    lead = block_tables[members[0]]
    p = 0
    while p < limit and all(int(block_tables[m][p]) == int(lead[p]) for m in members):
        p += 1
    return max(p, 0)


def partial_attention(q_vec: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float):
    """Attention of one query over one part of its context, kept as the
    pair (log-sum-exp of the scores, normalised output): ``lse = log sum
    exp(z)``, ``o = softmax(z) @ values`` with ``z = scale * keys @ q``.
    An empty part gives (-inf, 0)."""
    if keys.shape[0] == 0:
        return -np.inf, np.zeros(values.shape[-1])
    z = float(scale) * (keys @ q_vec)
    m = z.max()
    e = np.exp(z - m)
    return m + np.log(e.sum()), (e / e.sum()) @ values


def merge_partials(parts):
    """Combine the (lse, o) pairs of disjoint parts of one context into the
    attention over their union: weights ``exp(lse_i - max lse)``,
    ``out = sum_i w_i o_i / sum_i w_i``."""
    lses = np.array([p[0] for p in parts], dtype=np.float64)
    M = lses.max()
    if M == -np.inf:
        return np.zeros_like(parts[0][1])
    w = np.exp(lses - M)
    return sum(wi * p[1] for wi, p in zip(w, parts)) / w.sum()


def shared_prefix_decode(q_raw, q_dtype: str, k_pool, v_pool, cache_dtype: str, block_tables,
                         context_lens, group_start, group_seqs, scale: float, num_kv_heads: int,
                         k_scale: float = 1.0, v_scale: float = 1.0):
    """Decode attention with shared prefixes taken apart (cascade form), fp64.

    For every group g (sequences ``group_seqs[group_start[g]:group_start[g+1]]``)
    the shared blocks (``shared_prefix_blocks``) are attended once per member
    query as one part, the member's remaining tokens as a second part, and
    the two partial results are merged by log-sum-exp (``merge_partials``).
    Sequences in no group are one part.  The result is the plain decode
    attention of every sequence (``decode``), a sum split in two.
    Returns (out ``[B, Hq, D]``, shared blocks per sequence ``[B]``).
    """
    q = decode_cache(q_raw, q_dtype)
    B, hq, d = q.shape
    bs = k_pool.shape[1]
    group = hq // num_kv_heads
    pre = np.zeros(B, dtype=np.int64)
    gs = np.asarray(group_start, dtype=np.int64)
    for g in range(len(gs) - 1):
        members = list(group_seqs[gs[g]:gs[g + 1]])
        p = shared_prefix_blocks(block_tables, context_lens, members, bs)
        for m in members:
            pre[int(m)] = p
    out = np.zeros((B, hq, d), dtype=np.float64)
    for s in range(B):
        n = int(context_lens[s])
        if n <= 0:
            continue
        nb = -(-n // bs)
        ids = np.asarray(block_tables[s][:nb], dtype=np.int64)
        K = gather(decode_cache(k_pool[ids], cache_dtype, k_scale), np.arange(nb), n)
        V = gather(decode_cache(v_pool[ids], cache_dtype, v_scale), np.arange(nb), n)
        cut = int(pre[s]) * bs
        for h in range(hq):
            kv = h // group
            head = partial_attention(q[s, h], K[:cut, kv], V[:cut, kv], scale)
            tail = partial_attention(q[s, h], K[cut:, kv], V[cut:, kv], scale)
            out[s, h] = merge_partials([head, tail])
    return out, pre
