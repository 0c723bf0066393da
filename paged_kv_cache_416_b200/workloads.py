"""Seeded synthetic inputs for the paged decode path.

These generators feed both the CUDA path and the CPU oracle.  They hold
none of the method's arithmetic: they draw values with library generators
(numpy / torch), round them to the storage dtype with library casts, and
lay sequences out through :class:`~paged_kv_cache_416_b200.alloc.BlockAllocator`.

Recipe (every workload):

* q, K, V ~ N(0, 1) drawn in fp32 by ``torch.Generator(device).manual_seed``
  and rounded to the storage dtype by torch's round-to-nearest-even casts;
  an e4m3 cache stores ``clamp(x / s, -448, 448)`` cast by
  ``torch.float8_e4m3fn`` with the per-tensor scale ``s = max|x| / 448``;
* structure (lengths, free-list order, prefix lengths) from
  ``numpy.random.default_rng(seed)``;
* physical block ids: the free list is a seeded permutation of the pool, so
  every sequence's blocks are scattered;
* pool = blocks in use + 10% spare (the tiny workload: 64 blocks);
* every slot no sequence uses (spare blocks, the tail of each last block) is
  poisoned with NaN (e4m3: code 0x7F), and tables are padded with -1, so a
  kernel that reads past a sequence's tokens shows it;
* one decode step writes each sequence's newest token (position len-1)
  with ``pa_write_kv`` and then attends over all ``len`` tokens.

Workloads (sizes as in the five benchmark configurations):

``tiny``                 4 seqs, lens [40,16,1,63], 4/4 heads, D 64, fp16, bs 16, 64 blocks
``llama13b_mha``         64 seqs, lens U{128..2048}, 40/40 heads, D 128, fp16, bs 16
``llama70b_gqa``         256 seqs, all lens 4096, 64/8 heads, D 128, bf16, bs 16
``shared_prefix_fork``   32 prompts x 4 samples sharing a 1024 + r tokens prefix
                         (r ~ U{1..15}, so the last prefix block is partial);
                         the step copies that block for 3 of 4 samples
                         (copy-on-write, 96 pairs), writes each sample's first
                         own token and decodes; 32/8 heads, D 128, bf16
``shared_prefix_tails``  the same batch later: each sample has T ~ U{0..512}
                         own tokens after the fork; the step writes the next
                         token and decodes
``fp8_longtail_bs16/32`` 128 seqs, lens lognormal(ln 1024, 1) clipped to
                         [1, 32768], 32/8 heads, D 128, q bf16, e4m3 cache
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

from .alloc import BlockAllocator

TORCH_DTYPE = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn}
ELEM_BYTES = {"f16": 2, "bf16": 2, "e4m3": 1}
E4M3_MAX = 448.0


@dataclass
class Workload:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    q_dtype: str
    cache_dtype: str
    num_blocks: int
    scale: float
    k_scale: float
    v_scale: float
    context_lens: np.ndarray          # int32 [B]
    block_tables: np.ndarray          # int32 [B, W], padded with -1
    q: torch.Tensor                   # [B, Hq, D] q dtype
    k_pool: torch.Tensor              # [N, bs, Hkv, D] cache dtype
    v_pool: torch.Tensor
    new_k: torch.Tensor               # [T, Hkv, D] q dtype
    new_v: torch.Tensor
    slot_mapping: np.ndarray          # int64 [T]
    cow_pairs: np.ndarray             # int64 [P, 2]
    meta: Dict = field(default_factory=dict)

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if len(self.context_lens) else 0

    @property
    def kv_bytes(self) -> int:
        """Algorithmic K+V bytes one decode reads: sum(len) * Hkv * D * 2 * e."""
        return int(self.context_lens.astype(np.int64).sum()) * self.num_kv_heads * \
            self.head_dim * 2 * ELEM_BYTES[self.cache_dtype]

    @property
    def seq_tokens(self) -> int:
        return int(self.context_lens.astype(np.int64).sum())


def raw(t: torch.Tensor) -> np.ndarray:
    """Raw storage words of a tensor as numpy (uint16 for 16-bit, uint8 for
    8-bit), copied to the host."""
    t = t.detach().contiguous().cpu()
    if t.element_size() == 2:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.element_size() == 1:
        return t.view(torch.uint8).numpy()
    raise TypeError("expected a 16-bit or 8-bit tensor")


def _randn(shape, gen, device):
    """fp32 N(0,1) draw from the seeded generator."""
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _to_storage(x32: torch.Tensor, dtype: str, scale: float = 1.0) -> torch.Tensor:
    if dtype == "e4m3":
        return (x32 / scale).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return x32.to(TORCH_DTYPE[dtype])


def _fill_pool(num_blocks, bs, hkv, d, dtype, valid, gen, device, scale=None):
    """Pool [N, bs, Hkv, D] with N(0,1) values in valid slots and NaN poison
    elsewhere.  Returns (pool, scale) where scale is the e4m3 per-tensor
    scale (max |x| / 448 over the drawn values) or 1.0."""
    pool = torch.empty((num_blocks, bs, hkv, d), dtype=TORCH_DTYPE[dtype], device=device)
    # draw in slabs of blocks to bound the fp32 temporary
    slab = max(1, (1 << 26) // (bs * hkv * d))
    amax = 0.0
    draws = []
    for b0 in range(0, num_blocks, slab):
        b1 = min(num_blocks, b0 + slab)
        x = _randn((b1 - b0, bs, hkv, d), gen, device)
        if dtype == "e4m3":
            amax = max(amax, float(x.abs().max()))
            draws.append((b0, b1, x.cpu() if device == "cpu" else x))
        else:
            pool[b0:b1] = x.to(TORCH_DTYPE[dtype])
    if dtype == "e4m3":
        scale = amax / E4M3_MAX if scale is None else scale
        for b0, b1, x in draws:
            pool[b0:b1] = _to_storage(x.to(device), "e4m3", scale)
    else:
        scale = 1.0
    vmask = torch.from_numpy(valid).to(device)  # [N, bs] bool
    bad = ~vmask
    if bool(bad.any()):
        if dtype == "e4m3":
            pool.view(torch.uint8)[bad] = 0x7F
        else:
            pool[bad] = float("nan")
    return pool, float(scale)


def _valid_slots(num_blocks, bs, tables: List[List[int]], lens: List[int]) -> np.ndarray:
    valid = np.zeros((num_blocks, bs), dtype=bool)
    for t, n in zip(tables, lens):
        if n <= 0:
            continue
        nb = -(-n // bs)
        if nb > 1:
            valid[np.asarray(t[: nb - 1], dtype=np.int64)] = True
        valid[t[nb - 1], : n - (nb - 1) * bs] = True
    return valid


def _generic(name, lens, hq, hkv, d, bs, q_dtype, cache_dtype, seed, device,
             num_blocks=None, spare=0.10, shuffle=True) -> Workload:
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in lens]
    need = sum(-(-n // bs) for n in lens)
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(need * (1.0 + spare))))
    free = rng.permutation(num_blocks) if shuffle else np.arange(num_blocks)
    alloc = BlockAllocator(num_blocks, bs, free_list=free.tolist())
    B = len(lens)
    for s, n in enumerate(lens):
        alloc.allocate(s, n)
    tables = alloc.table_array(list(range(B)))
    gen = torch.Generator(device=device).manual_seed(int(seed))
    valid = _valid_slots(num_blocks, bs, [alloc.tables[s] for s in range(B)], lens)
    k_pool, k_scale = _fill_pool(num_blocks, bs, hkv, d, cache_dtype, valid, gen, device)
    v_pool, v_scale = _fill_pool(num_blocks, bs, hkv, d, cache_dtype, valid, gen, device)
    q = _to_storage(_randn((B, hq, d), gen, device), q_dtype)
    new_k = _to_storage(_randn((B, hkv, d), gen, device), q_dtype)
    new_v = _to_storage(_randn((B, hkv, d), gen, device), q_dtype)
    # the newest token of every sequence sits at position len - 1; a sequence
    # of length 0 has no token to write (slot -1 is skipped)
    slots = np.array([alloc.slot(s, n - 1) if n > 0 else -1 for s, n in enumerate(lens)], dtype=np.int64)
    return Workload(
        name=name, num_seqs=B, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, block_size=bs,
        q_dtype=q_dtype, cache_dtype=cache_dtype, num_blocks=num_blocks,
        scale=1.0 / math.sqrt(d), k_scale=k_scale, v_scale=v_scale,
        context_lens=np.asarray(lens, dtype=np.int32), block_tables=tables,
        q=q, k_pool=k_pool, v_pool=v_pool, new_k=new_k, new_v=new_v,
        slot_mapping=slots, cow_pairs=np.zeros((0, 2), dtype=np.int64),
        meta={"seed": int(seed), "allocator": alloc},
    )


def _lens_tiny(lens=(40, 16, 1, 63)):
    return np.asarray(lens, dtype=np.int64)


def _lens_llama13b(seed, num_seqs=64, max_len=2048, min_len=128):
    rng = np.random.default_rng(seed + 1000)
    return rng.integers(min_len, max_len + 1, size=num_seqs)


def _lens_llama70b(num_seqs=256, context_len=4096):
    return np.full(num_seqs, context_len, dtype=np.int64)


def _lens_fp8(seed, num_seqs=128, max_len=32768):
    rng = np.random.default_rng(seed + 1000)
    return np.clip(np.rint(rng.lognormal(math.log(1024.0), 1.0, size=num_seqs)), 1,
                   max_len).astype(np.int64)


def tiny(seed=1, device="cpu", **kw) -> Workload:
    """4 sequences, lens [40,16,1,63], 4/4 heads, D 64, fp16, bs 16, a 64-block
    pool whose free list is a seeded shuffle (9 blocks used)."""
    lens = _lens_tiny(kw.pop("lens", (40, 16, 1, 63)))
    return _generic("tiny", lens, 4, 4, 64, 16, "f16", "f16", seed, device, num_blocks=64, **kw)


def llama13b_mha(seed=2, device="cpu", num_seqs=64, max_len=2048, min_len=128, **kw) -> Workload:
    """LLaMA-13B-shaped MHA layer: 40/40 heads, D 128, fp16, bs 16,
    lens U{min_len..max_len}."""
    lens = _lens_llama13b(seed, num_seqs, max_len, min_len)
    return _generic("llama13b_mha", lens, 40, 40, 128, kw.pop("block_size", 16), "f16", "f16",
                    seed, device, **kw)


def llama70b_gqa(seed=3, device="cpu", num_seqs=256, context_len=4096, **kw) -> Workload:
    """Llama-3-70B-shaped GQA layer: 64/8 heads, D 128, bf16, bs 16, every
    sequence ``context_len`` tokens."""
    lens = _lens_llama70b(num_seqs, context_len)
    return _generic("llama70b_gqa", lens, 64, 8, 128, kw.pop("block_size", 16), "bf16", "bf16",
                    seed, device, **kw)


def fp8_longtail(seed=5, device="cpu", num_seqs=128, block_size=16, max_len=32768, **kw) -> Workload:
    """Llama-3-8B-shaped layer, e4m3 cache: 32/8 heads, D 128, q bf16, lens
    lognormal(ln 1024, 1) rounded and clipped to [1, max_len]."""
    lens = _lens_fp8(seed, num_seqs, max_len)
    w = _generic(f"fp8_longtail_bs{block_size}", lens, 32, 8, 128, block_size, "bf16", "e4m3",
                 seed, device, **kw)
    return w


def e4m3_uniform(seed=5, device="cpu", num_seqs=128, context_len=4096, **kw) -> Workload:
    """Diagnostic companion of the fp8 long-tail batch: the same layer shape
    and cache format (32/8 heads, D 128, e4m3 cache, bf16 q, bs 16) with every
    sequence ``context_len`` tokens, so the per-byte cost of the e4m3 path
    can be told apart from the cost of a long-tailed length mix."""
    lens = _lens_llama70b(num_seqs, context_len)
    return _generic("e4m3_uniform", lens, 32, 8, 128, kw.pop("block_size", 16), "bf16", "e4m3",
                    seed, device, **kw)


def _sample_groups(prompts: int, samples: int) -> Dict:
    """The samples of one prompt form a group: group_seqs lists sequences
    p * samples + i group by group, group_start[g] is where group g starts."""
    return {"group_start": np.arange(prompts + 1, dtype=np.int32) * samples,
            "group_seqs": np.arange(prompts * samples, dtype=np.int32)}


def _shared_prefix_draws(seed, prompts, samples, prefix, max_tail, bs):
    """Prompt lengths (prefix + r, r ~ U{1..bs-1}) and own-token counts
    T ~ U{0..max_tail} per sample, and the generator that drew them (the
    batch draws its free-list order from it next)."""
    rng = np.random.default_rng(seed + 1000)
    extra = rng.integers(1, bs, size=prompts)
    tails = rng.integers(0, max_tail + 1, size=(prompts, samples))
    return rng, prefix + extra, tails


def _lens_shared_prefix(phase, seed, prompts=32, samples=4, prefix=1024, max_tail=512, bs=16,
                        **_):
    """Context lengths of the shared-prefix batch: the prompt and the fork
    step's token; later also T own tokens and the step's token."""
    _, plen, tails = _shared_prefix_draws(seed, prompts, samples, prefix, max_tail, bs)
    first = np.repeat(plen + 1, samples)
    return first if phase == "fork" else first + tails.reshape(-1) + 1


def _shared_prefix(phase, seed, device, prompts=32, samples=4, prefix=1024,
                   max_tail=512, hq=32, hkv=8, d=128, bs=16, cache="bf16") -> Workload:
    """Parallel sampling over a shared prompt (see the module docstring);
    queries and new tokens bf16, the cache bf16 or e4m3 (per-tensor scales
    from the prompt's values, later tokens quantised with the same scales)."""
    rng, plen, tails = _shared_prefix_draws(seed, prompts, samples, prefix, max_tail, bs)
    B = prompts * samples
    # pool: shared prompt blocks once, plus every sample's own blocks
    own = 0
    for p in range(prompts):
        for i in range(samples):
            own += -(-(int(plen[p]) + 2 + int(tails[p, i])) // bs) - int(plen[p]) // bs
    need = sum(-(-int(n) // bs) for n in plen) + own
    num_blocks = int(math.ceil(need * 1.1))
    alloc = BlockAllocator(num_blocks, bs, free_list=rng.permutation(num_blocks).tolist())
    gen = torch.Generator(device=device).manual_seed(int(seed))
    seq = lambda p, i: p * samples + i
    for p in range(prompts):
        alloc.allocate(seq(p, 0), int(plen[p]))
        for i in range(1, samples):
            alloc.fork(seq(p, 0), seq(p, i))
    prompt_valid = _valid_slots(num_blocks, bs, [alloc.tables[seq(p, 0)] for p in range(prompts)],
                                [int(n) for n in plen])
    # each sample's first own token: the shared partial block is copied for
    # every sample but the last one to write (copy-on-write)
    pairs, first_slots = [], []
    for p in range(prompts):
        for i in range(samples):
            slot, cow = alloc.append_token(seq(p, i))
            first_slots.append(slot)
            if cow is not None:
                pairs.append(cow)
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    k_pool, k_scale = _fill_pool(num_blocks, bs, hkv, d, cache, prompt_valid, gen, device)
    v_pool, v_scale = _fill_pool(num_blocks, bs, hkv, d, cache, prompt_valid, gen, device)
    q = _to_storage(_randn((B, hq, d), gen, device), "bf16")
    first_k = _to_storage(_randn((B, hkv, d), gen, device), "bf16")
    first_v = _to_storage(_randn((B, hkv, d), gen, device), "bf16")
    if phase == "fork":
        lens = np.array([alloc.lengths[seq(p, i)] for p in range(prompts) for i in range(samples)],
                        dtype=np.int32)
        tables = alloc.table_array(list(range(B)))
        return Workload(
            name="shared_prefix_fork", num_seqs=B, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
            block_size=bs, q_dtype="bf16", cache_dtype=cache, num_blocks=num_blocks,
            scale=1.0 / math.sqrt(d), k_scale=k_scale, v_scale=v_scale, context_lens=lens,
            block_tables=tables, q=q, k_pool=k_pool, v_pool=v_pool, new_k=first_k, new_v=first_v,
            slot_mapping=np.asarray(first_slots, dtype=np.int64), cow_pairs=pairs,
            meta={"seed": int(seed), "allocator": alloc, "prompt_lens": plen, "samples": samples,
                  **_sample_groups(prompts, samples)},
        )
    # tails phase: lay the state after the fork step and T own tokens down
    # directly (copied prompt rows in the copied blocks, fresh values for the
    # own tokens), then the step writes the next token of every sample
    if len(pairs):
        src = torch.from_numpy(pairs[:, 0]).to(device)
        dst = torch.from_numpy(pairs[:, 1]).to(device)
        k_pool[dst] = k_pool[src]
        v_pool[dst] = v_pool[src]
    fs = torch.from_numpy(np.asarray(first_slots, dtype=np.int64)).to(device)
    k_pool.view(-1, hkv, d)[fs] = _to_storage(first_k.float(), cache, k_scale)
    v_pool.view(-1, hkv, d)[fs] = _to_storage(first_v.float(), cache, v_scale)
    tail_slots = []
    for p in range(prompts):
        for i in range(samples):
            for _ in range(int(tails[p, i])):
                slot, cow = alloc.append_token(seq(p, i))
                assert cow is None  # every sample owns its last block after the fork step
                tail_slots.append(slot)
    if tail_slots:
        ts = torch.from_numpy(np.asarray(tail_slots, dtype=np.int64)).to(device)
        n = len(tail_slots)
        k_pool.view(-1, hkv, d)[ts] = _to_storage(_randn((n, hkv, d), gen, device), cache, k_scale)
        v_pool.view(-1, hkv, d)[ts] = _to_storage(_randn((n, hkv, d), gen, device), cache, v_scale)
    step_slots = []
    for p in range(prompts):
        for i in range(samples):
            slot, cow = alloc.append_token(seq(p, i))
            assert cow is None
            step_slots.append(slot)
    lens = np.array([alloc.lengths[seq(p, i)] for p in range(prompts) for i in range(samples)],
                    dtype=np.int32)
    tables = alloc.table_array(list(range(B)))
    new_k = _to_storage(_randn((B, hkv, d), gen, device), "bf16")
    new_v = _to_storage(_randn((B, hkv, d), gen, device), "bf16")
    return Workload(
        name="shared_prefix_tails", num_seqs=B, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
        block_size=bs, q_dtype="bf16", cache_dtype=cache, num_blocks=num_blocks,
        scale=1.0 / math.sqrt(d), k_scale=k_scale, v_scale=v_scale, context_lens=lens,
        block_tables=tables, q=q, k_pool=k_pool, v_pool=v_pool, new_k=new_k, new_v=new_v,
        slot_mapping=np.asarray(step_slots, dtype=np.int64), cow_pairs=np.zeros((0, 2), np.int64),
        meta={"seed": int(seed), "allocator": alloc, "prompt_lens": plen, "tails": tails,
              "samples": samples, **_sample_groups(prompts, samples)},
    )


def shared_prefix_fork(seed=4, device="cpu", **kw) -> Workload:
    return _shared_prefix("fork", seed, device, **kw)


def shared_prefix_tails(seed=4, device="cpu", **kw) -> Workload:
    return _shared_prefix("tails", seed, device, **kw)


@dataclass
class PrefillWorkload:
    """Chunked prefill: sequence s has context_lens[s] cached tokens, of which
    the last query_start[s+1] - query_start[s] are the new query tokens."""
    base: Workload                    # pools, tables, lengths (its q/new_k unused)
    q: torch.Tensor                   # [total_q, Hq, D]
    query_start: np.ndarray           # int32 [B + 1]

    @property
    def max_query_len(self) -> int:
        return int(np.diff(self.query_start).max()) if len(self.query_start) > 1 else 0

    @property
    def flops(self) -> int:
        """Causal attention flops: 4 * D * Hq * sum over new tokens of the keys each sees."""
        b = self.base
        tot = 0
        for s in range(b.num_seqs):
            n = int(self.query_start[s + 1] - self.query_start[s])
            c = int(b.context_lens[s])
            tot += n * (c - n) + n * (n + 1) // 2
        return 4 * b.head_dim * b.num_q_heads * tot


def prefill(seed=6, device="cpu", ctxs=(200, 300, 1, 77), nqs=(200, 77, 1, 50), hq=32, hkv=8,
            d=128, bs=16, dtype="bf16", **kw) -> PrefillWorkload:
    """Paged prefill inputs: the cache holds every token (the new ones
    included, as pa_write_kv leaves it); q holds the new tokens, packed."""
    assert all(n <= c for n, c in zip(nqs, ctxs))
    base = _generic("prefill", list(ctxs), hq, hkv, d, bs, dtype, dtype, seed, device, **kw)
    qs = np.concatenate([[0], np.cumsum(nqs)]).astype(np.int32)
    gen = torch.Generator(device=device).manual_seed(int(seed) + 77)
    q = _to_storage(_randn((int(qs[-1]), hq, d), gen, device), dtype)
    return PrefillWorkload(base=base, q=q, query_start=qs)


# (kv heads, head_dim, bytes per cache element) and the length rule of each
# workload, for sizes without building pools
_SHAPES = {"tiny": (4, 64, 2), "llama13b_mha": (40, 128, 2), "llama70b_gqa": (8, 128, 2),
           "shared_prefix_fork": (8, 128, 2), "shared_prefix_tails": (8, 128, 2),
           "fp8_longtail_bs16": (8, 128, 1), "fp8_longtail_bs32": (8, 128, 1),
           "e4m3_uniform": (8, 128, 1)}
_DEFAULT_SEEDS = {"tiny": 1, "llama13b_mha": 2, "llama70b_gqa": 3, "shared_prefix_fork": 4,
                  "shared_prefix_tails": 4, "fp8_longtail_bs16": 5, "fp8_longtail_bs32": 5,
                  "e4m3_uniform": 5}


def default_seed(name: str) -> int:
    """The seed of a workload's configuration (1..5, by configuration)."""
    return _DEFAULT_SEEDS[name]


def context_lens(name: str, seed: Optional[int] = None, **kw) -> np.ndarray:
    """The context lengths :func:`make` gives for the same arguments, without
    building the pools."""
    seed = _DEFAULT_SEEDS[name] if seed is None else seed
    if name == "tiny":
        return _lens_tiny(kw.get("lens", (40, 16, 1, 63)))
    if name == "llama13b_mha":
        return _lens_llama13b(seed, **{k: kw[k] for k in ("num_seqs", "max_len", "min_len") if k in kw})
    if name == "llama70b_gqa":
        return _lens_llama70b(**{k: kw[k] for k in ("num_seqs", "context_len") if k in kw})
    if name == "e4m3_uniform":
        return _lens_llama70b(kw.get("num_seqs", 128), kw.get("context_len", 4096))
    if name.startswith("fp8_longtail"):
        return _lens_fp8(seed, **{k: kw[k] for k in ("num_seqs", "max_len") if k in kw})
    return _lens_shared_prefix(name.split("_")[-1], seed, **kw)


def kv_bytes_of(name: str, seed: Optional[int] = None, **kw) -> int:
    """Algorithmic K+V bytes one decode of the workload reads (as
    ``make(name, seed, **kw).kv_bytes``), from the lengths alone."""
    hkv, d, e = _SHAPES[name]
    return int(context_lens(name, seed, **kw).astype(np.int64).sum()) * hkv * d * 2 * e


REGISTRY = {
    "tiny": tiny,
    "llama13b_mha": llama13b_mha,
    "llama70b_gqa": llama70b_gqa,
    "shared_prefix_fork": shared_prefix_fork,
    "shared_prefix_tails": shared_prefix_tails,
    "fp8_longtail_bs16": lambda seed=5, device="cpu", **kw: fp8_longtail(seed, device, block_size=16, **kw),
    "fp8_longtail_bs32": lambda seed=5, device="cpu", **kw: fp8_longtail(seed, device, block_size=32, **kw),
    "e4m3_uniform": e4m3_uniform,
}


def make(name: str, seed: Optional[int] = None, device="cpu", **kw) -> Workload:
    fn = REGISTRY[name]
    return fn(device=device, **kw) if seed is None else fn(seed=seed, device=device, **kw)
