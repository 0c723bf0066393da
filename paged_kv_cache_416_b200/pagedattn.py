"""ctypes binding of libpagedattn.so (the C ABI in include/pagedattn.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  Importing this module loads the library and raises if it is
missing -- there is no CPU fallback.  torch supplies device memory and
streams.

Two layers:
* ``pa_*``: the C entry points themselves, with ctypes signatures (raw
  pointers, sizes, dtype codes, stream handles);
* ``write_kv``, ``copy_blocks``, ``decode``, ``decode_workspace_size``,
  ``decode_shared_prefix``, ``shared_prefix_workspace_size``, ``prefill``,
  ``swap_blocks``, ``hash_blocks``, ``sync_status``: the same calls taking
  torch tensors, which read pointers, sizes and dtypes off the tensors and
  pass the current torch stream.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "pagedattn.h")

PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2
STATUS_NAMES = {
    0: "PA_OK", 1: "PA_ERR_NULL", 2: "PA_ERR_DTYPE", 3: "PA_ERR_SHAPE", 4: "PA_ERR_HEADS",
    5: "PA_ERR_RANGE", 6: "PA_ERR_ALIAS", 7: "PA_ERR_CUDA", 8: "PA_ERR_DEVICE_BOUNDS",
    9: "PA_ERR_WORKSPACE", 10: "PA_ERR_TIMEOUT", 11: "PA_ERR_MEMORY",
}
_TORCH_TO_PA = {torch.float16: PA_F16, torch.bfloat16: PA_BF16, torch.float8_e4m3fn: PA_FP8_E4M3}


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Set the ctypes signatures of the C entry points on a loaded library."""
    P, I32, I64, F, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sig = {
        "pa_write_kv": (I32, [P, P, I32, P, I32, P, P, I32, I32, I32, I32, I32, F, F, P]),
        "pa_copy_blocks": (I32, [P, P, I32, I32, I32, I32, I32, P, I32, P]),
        "pa_swap_blocks": (I32, [P, P, I32, P, P, I32, I32, I32, I32, I32, P, I32, P]),
        "pa_hash_blocks": (I32, [P, I64, P, I32, I32, P, I32, P]),
        "pa_prefill": (I32, [P, P, I32, P, P, I32, P, I32, P, P, I32, I32, I32, I32, I32, I32,
                             I32, I32, F, P]),
        "pa_decode_split_tokens": (I32, [I32, I32, I32, I32, I32]),
        "pa_decode_workspace_size": (SZ, [I32, I32, I32, I32, I32, I32, I32]),
        "pa_decode": (I32, [P, P, I32, P, P, I32, P, I32, P, I32, I32, I32, I32, I32, I32, I32,
                            F, F, F, I32, P, SZ, P]),
        "pa_decode_shared_prefix_workspace_size": (SZ, [I32, I32, I32, I32, I32, I32, I32]),
        "pa_decode_shared_prefix": (I32, [P, P, I32, P, P, I32, P, I32, P, I32, P, P, I32, I32,
                                          I32, I32, I32, I32, I32, F, F, F, I32, P, SZ, P]),
        "pa_sync_status": (I32, [P]),
        "pa_last_error": (ctypes.c_char_p, []),
        "pa_validate_slot_mapping": (I32, [P, I32, I32, I32, P]),
        "pa_validate_copy_pairs": (I32, [P, I32, I32, P]),
        "pa_validate_block_tables": (I32, [P, I32, P, I32, I32, I32, I32, P]),
        "pa_decode_noalloc": (I32, [P, P, I32, P, P, I32, P, I32, P, I32, I32, I32, I32, I32, I32,
                                    I32, F, F, F, I32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with `python -m paged_kv_cache_416_b200.build` "
            "(there is no CPU fallback)")
    return declare(ctypes.CDLL(LIB_PATH))


_lib = _load()

# the C entry points, unchanged
pa_write_kv = _lib.pa_write_kv
pa_copy_blocks = _lib.pa_copy_blocks
pa_swap_blocks = _lib.pa_swap_blocks
pa_hash_blocks = _lib.pa_hash_blocks
pa_prefill = _lib.pa_prefill
pa_decode_split_tokens = _lib.pa_decode_split_tokens
pa_decode_workspace_size = _lib.pa_decode_workspace_size
pa_decode = _lib.pa_decode
pa_decode_shared_prefix_workspace_size = _lib.pa_decode_shared_prefix_workspace_size
pa_decode_shared_prefix = _lib.pa_decode_shared_prefix
pa_sync_status = _lib.pa_sync_status
pa_last_error = _lib.pa_last_error
pa_validate_slot_mapping = _lib.pa_validate_slot_mapping
pa_validate_copy_pairs = _lib.pa_validate_copy_pairs
pa_validate_block_tables = _lib.pa_validate_block_tables
# pa_decode for callers that cannot allocate device memory: the scratch comes
# from an array the library reserves when it is loaded (see the header)
pa_decode_noalloc = _lib.pa_decode_noalloc


def _header_size_define(name: str) -> int:
    """Value of a `#define NAME (a * b * ...)` size constant of the C header,
    so that the binding and the library take it from one source."""
    import re
    with open(HEADER_PATH) as f:
        text = f.read()
    m = re.search(r"#define\s+" + name + r"\s+\(([^)]*)\)", text)
    if m is None:
        raise ImportError(f"{name} is not defined in {HEADER_PATH}")
    value = 1
    for factor in m.group(1).split("*"):
        value *= int(factor.strip().rstrip("uUlL"))
    return value


NOALLOC_SCRATCH_BYTES = _header_size_define("PA_DECODE_NOALLOC_SCRATCH_BYTES")

ENTRY_POINTS = [
    "pa_write_kv", "pa_copy_blocks", "pa_swap_blocks", "pa_hash_blocks", "pa_decode_split_tokens", "pa_decode_workspace_size",
    "pa_decode", "pa_prefill", "pa_sync_status", "pa_last_error", "pa_validate_slot_mapping",
    "pa_validate_copy_pairs", "pa_validate_block_tables", "pa_decode_noalloc",
    "pa_decode_shared_prefix_workspace_size", "pa_decode_shared_prefix",
]


def library() -> ctypes.CDLL:
    return _lib


def check(status: int) -> None:
    """Raise PagedAttnError for a non-zero status, with pa_last_error()."""
    if status != 0:
        msg = _lib.pa_last_error()
        raise PagedAttnError(status, msg.decode() if msg else "")


# ----------------------------------------------------------- tensor helpers
def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t: torch.Tensor, override: Optional[int] = None) -> int:
    if override is not None:
        return override
    if t.dtype not in _TORCH_TO_PA:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _TORCH_TO_PA[t.dtype]


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def write_kv(k, v, slot_mapping, k_pool, v_pool, k_scale: float = 1.0, v_scale: float = 1.0,
             stream=None) -> None:
    """pa_write_kv on tensors: k, v [T, Hkv, D] (f16/bf16), slot_mapping int64 [T],
    pools [N, bs, Hkv, D] (k's dtype, or float8_e4m3fn)."""
    _contig(k, v, slot_mapping, k_pool, v_pool)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    N, bs, hkv, d = k_pool.shape
    check(pa_write_kv(_ptr(k), _ptr(v), _dtype(k), _ptr(slot_mapping), k.shape[0], _ptr(k_pool),
                      _ptr(v_pool), _dtype(k_pool), N, bs, hkv, d, float(k_scale), float(v_scale),
                      _stream(stream)))


def copy_blocks(k_pool, v_pool, pairs, stream=None) -> None:
    """pa_copy_blocks on tensors: pairs int64 [P, 2] of (src, dst) block ids."""
    _contig(k_pool, v_pool, pairs)
    if pairs.dtype != torch.int64:
        raise TypeError("pairs must be int64")
    N, bs, hkv, d = k_pool.shape
    check(pa_copy_blocks(_ptr(k_pool), _ptr(v_pool), _dtype(k_pool), N, bs, hkv, d, _ptr(pairs),
                         pairs.shape[0], _stream(stream)))


def swap_blocks(src_k, src_v, dst_k, dst_v, pairs, stream=None) -> None:
    """pa_swap_blocks on tensors: pools [N, bs, Hkv, D] of one dtype, on the
    device or in pinned host memory; pairs int64 [P, 2] (src id, dst id) on
    the device."""
    _contig(src_k, src_v, dst_k, dst_v, pairs)
    if pairs.dtype != torch.int64:
        raise TypeError("pairs must be int64")
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype != dst_k.dtype:
        raise ValueError("the pools must share block shape and dtype")
    N, bs, hkv, d = src_k.shape
    check(pa_swap_blocks(_ptr(src_k), _ptr(src_v), N, _ptr(dst_k), _ptr(dst_v), dst_k.shape[0],
                         _dtype(src_k), bs, hkv, d, _ptr(pairs), pairs.shape[0], _stream(stream)))


def hash_blocks(token_ids, num_tokens, block_size: int, max_blocks: Optional[int] = None,
                out=None, stream=None) -> torch.Tensor:
    """pa_hash_blocks on tensors: token_ids int32 [B, L], num_tokens int32 [B]
    -> int64 [B, max_blocks] (the uint64 hash bits)."""
    _contig(token_ids, num_tokens)
    if token_ids.dtype != torch.int32 or num_tokens.dtype != torch.int32:
        raise TypeError("token_ids and num_tokens must be int32")
    B, L = token_ids.shape
    mb = max(1, L // block_size) if max_blocks is None else int(max_blocks)
    if out is None:
        out = torch.empty((B, mb), dtype=torch.int64, device=token_ids.device)
    check(pa_hash_blocks(_ptr(token_ids), L, _ptr(num_tokens), B, block_size, _ptr(out), mb,
                         _stream(stream)))
    return out


def decode_split_tokens(num_seqs, num_kv_heads, block_size, max_context_len, split_tokens=0) -> int:
    return int(pa_decode_split_tokens(num_seqs, num_kv_heads, block_size, max_context_len,
                                      split_tokens))


def decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                          max_context_len, split_tokens=0) -> int:
    return int(pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                        max_context_len, split_tokens))


_ws_cache = {}


def workspace_for(device, nbytes: int) -> torch.Tensor:
    """A cached device byte buffer of at least nbytes (torch-allocated), one
    per device, grown when a call needs more.  Calls that use it share it, so
    they must not overlap on the GPU: calls on several streams at once pass
    their own `workspace`."""
    key = torch.device(device)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=key)
        _ws_cache[key] = buf
    return buf


def decode(q, k_pool, v_pool, block_tables, context_lens, scale: float, max_context_len: int,
           k_scale: float = 1.0, v_scale: float = 1.0, split_tokens: int = 0, out=None,
           workspace=None, stream=None) -> torch.Tensor:
    """pa_decode on tensors.  q [B, Hq, D]; pools [N, bs, Hkv, D]; block_tables
    int32 [B, W]; context_lens int32 [B].  Returns out [B, Hq, D] (q's dtype)."""
    _contig(q, k_pool, v_pool, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    B, hq, d = q.shape
    N, bs, hkv, d2 = k_pool.shape
    if out is None:
        out = torch.empty_like(q)
    nbytes = decode_workspace_size(B, hq, hkv, d, bs, max_context_len, split_tokens)
    if workspace is None:
        workspace = workspace_for(q.device, nbytes)
    check(pa_decode(_ptr(out), _ptr(q), _dtype(q), _ptr(k_pool), _ptr(v_pool), _dtype(k_pool),
                    _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                    int(max_context_len), B, hq, hkv, d, bs, N, float(scale), float(k_scale),
                    float(v_scale), int(split_tokens), _ptr(workspace), workspace.numel(),
                    _stream(stream)))
    return out


def shared_prefix_workspace_size(num_seqs, hq, hkv, head_dim, bs, max_context_len,
                                 split_tokens=0) -> int:
    return int(pa_decode_shared_prefix_workspace_size(num_seqs, hq, hkv, head_dim, bs,
                                                      int(max_context_len), int(split_tokens)))


def decode_shared_prefix(q, k_pool, v_pool, block_tables, context_lens, group_start, group_seqs,
                         scale: float, max_context_len: int, k_scale: float = 1.0,
                         v_scale: float = 1.0, split_tokens: int = 0, out=None,
                         workspace=None, stream=None) -> torch.Tensor:
    """pa_decode_shared_prefix on tensors: pa_decode's arguments plus the
    groups (group_start int32 [G + 1], group_seqs int32 [group_start[G]]).
    Returns out [B, Hq, D]."""
    _contig(q, k_pool, v_pool, block_tables, context_lens, group_start, group_seqs)
    for t in (block_tables, context_lens, group_start, group_seqs):
        if t.dtype != torch.int32:
            raise TypeError("block_tables, context_lens and the group arrays must be int32")
    B, hq, d = q.shape
    N, bs, hkv, _ = k_pool.shape
    if out is None:
        out = torch.empty_like(q)
    nbytes = shared_prefix_workspace_size(B, hq, hkv, d, bs, max_context_len, split_tokens)
    if workspace is None:
        workspace = workspace_for(q.device, nbytes)
    check(pa_decode_shared_prefix(
        _ptr(out), _ptr(q), _dtype(q), _ptr(k_pool), _ptr(v_pool), _dtype(k_pool),
        _ptr(block_tables), block_tables.shape[1], _ptr(context_lens), int(max_context_len),
        _ptr(group_start), _ptr(group_seqs), group_start.shape[0] - 1, B, hq, hkv, d, bs, N,
        float(scale), float(k_scale), float(v_scale), int(split_tokens), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return out


def prefill(q, k_pool, v_pool, block_tables, context_lens, query_start, scale: float,
            max_query_len: int, max_context_len: int, out=None, stream=None) -> torch.Tensor:
    """pa_prefill on tensors.  q [total_q, Hq, D] packed by query_start
    (int32 [B + 1]); pools [N, bs, Hkv, D]; block_tables int32 [B, W];
    context_lens int32 [B].  Returns out [total_q, Hq, D]."""
    _contig(q, k_pool, v_pool, block_tables, context_lens, query_start)
    for t in (block_tables, context_lens, query_start):
        if t.dtype != torch.int32:
            raise TypeError("block_tables, context_lens and query_start must be int32")
    total, hq, d = q.shape
    N, bs, hkv, _ = k_pool.shape
    if out is None:
        out = torch.empty_like(q)
    check(pa_prefill(_ptr(out), _ptr(q), _dtype(q), _ptr(k_pool), _ptr(v_pool), _dtype(k_pool),
                     _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                     _ptr(query_start), context_lens.shape[0], int(max_query_len),
                     int(max_context_len), hq, hkv, d, bs, N, float(scale), _stream(stream)))
    return out


def sync_status(stream=None) -> None:
    """pa_sync_status: synchronise and raise if a kernel reported an error."""
    check(pa_sync_status(_stream(stream)))
