/*
 * pagedattn.h -- C ABI of the paged KV-cache decode-attention library
 * (libpagedattn.so, hand-written CUDA for sm_100a / B200).
 *
 * The method: a KV cache split into fixed-size physical blocks that sit
 * wherever they were free in one shared pool, addressed per sequence by a
 * block table that maps logical block i to a physical block id; the attention
 * kernel follows the table to gather keys and values block by block, so a
 * sequence's cache need not be contiguous ("PagedAttention", Ultralytics
 * glossary, section "Sayfalama Nasil Calisir" and its PyTorch sketch).  Blocks
 * may be shared by several sequences and are copied before a write while
 * others still use them (same page, section "Diziler Arasinda Bloklari
 * Paylasma").  Grouped-query attention and FP8 caches are named as companion
 * techniques (same page, section "Ilgili Teknikler").
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees, retains or allocates device memory.
 *  - Every tensor is dense and row-major with the layout stated below.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and the call returns without synchronising.
 *  - Arguments are validated on the host before any launch; a failed check
 *    returns a PA_ERR_* code, launches nothing and sets pa_last_error().
 *  - Kernels never trap: an out-of-range index met on the device (a block id
 *    outside the pool, a slot outside the pool, a context length above the
 *    stated maximum) skips that access and records PA_ERR_DEVICE_BOUNDS in a
 *    device error word that pa_sync_status() reports.
 *  - Nothing throws across the ABI.
 *
 * Layouts (B = num_seqs, Hq = num_q_heads, Hkv = num_kv_heads, D = head_dim,
 * bs = block_size, N = num_blocks, T = num_tokens):
 *   q, out        [B, Hq, D]          q dtype (out has q's dtype)
 *   k, v (write)  [T, Hkv, D]
 *   k_pool/v_pool [N, bs, Hkv, D]     the sketch's key_pool[block, slot, dim]
 *                                     with the head axis before dim
 *   block_tables  int32 [B, max_blocks_per_seq]; entries at or past
 *                 ceil(context_lens[s] / bs) are never read
 *   context_lens  int32 [B]
 *   slot_mapping  int64 [T]; slot = physical_block * bs + offset; < 0 skips
 *   src_dst_pairs int64 [P, 2]
 *
 * Supported: D in {64, 128}; bs in {16, 32}; Hq a multiple of Hkv with
 * Hq / Hkv <= 64 for pa_decode (a kv head's query heads are taken 8 at a
 * time: more than 8 read its blocks once per group of 8), <= 16 for the
 * shared-prefix decode; cache dtype f16 (q f16), bf16 (q bf16) or e4m3 (q f16 or
 * bf16).  With an e4m3 cache the tensor-core products run in fp16: each
 * head's query is first scaled by a power of two that brings its largest
 * component into [2^14, 2^15), and the factor is taken back out of that
 * head's scores, so any finite f16 or bf16 query is accepted (a component
 * below 2^-28 of its head's largest falls into fp16's subnormal range, where
 * it is kept to an absolute precision of 2^-39 of that largest component).
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (the same object as cudaStream_t / CUstream). */
typedef struct CUstream_st* pa_stream_t;

typedef enum pa_dtype {
  PA_F16 = 0,      /* IEEE binary16 */
  PA_BF16 = 1,     /* bfloat16 */
  PA_FP8_E4M3 = 2  /* OCP 8-bit E4M3 ("fn": no infinities, 0x7F/0xFF NaN, max 448) */
} pa_dtype;

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_NULL = 1,          /* a required pointer is NULL */
  PA_ERR_DTYPE = 2,         /* unsupported dtype or dtype combination */
  PA_ERR_SHAPE = 3,         /* unsupported or inconsistent size */
  PA_ERR_HEADS = 4,         /* Hq not a multiple of Hkv, or too many query heads per kv head */
  PA_ERR_RANGE = 5,         /* an index is out of range (pa_validate_*) */
  PA_ERR_ALIAS = 6,         /* duplicate destinations, or a destination that is
                               also a source (pa_validate_*) */
  PA_ERR_CUDA = 7,          /* a CUDA runtime call failed; see pa_last_error() */
  PA_ERR_DEVICE_BOUNDS = 8, /* a kernel met an out-of-range index and skipped it */
  PA_ERR_WORKSPACE = 9,     /* workspace missing or smaller than required */
  PA_ERR_TIMEOUT = 10,      /* a kernel gave up waiting for an asynchronous copy
                               (about one second) and skipped that block */
  PA_ERR_MEMORY = 11        /* a buffer the device cannot reach (pageable host
                               memory) */
} pa_status;

/*
 * pa_write_kv -- scatter new keys and values into the pools by slot.
 * Defined by the pages' sketch, where token `pos` of a request is stored at
 * key_pool[block_table[pos // bs], pos % bs]; the caller folds the table into
 * slot = block_table[pos // bs] * bs + pos % bs ("Sayfalama Nasil Calisir").
 *
 * For each token t with slot_mapping[t] >= 0 and every kv head h:
 *   k_pool[slot / bs][slot % bs][h][:] = enc(k[t][h][:])   (same for v)
 * enc is the identity when cache_dtype == in_dtype (f16 or bf16), and for an
 * e4m3 cache enc(x) = e4m3_rne_satfinite(fp32(x) / k_scale) (v: v_scale),
 * with the division in IEEE fp32.  Tokens with slot < 0 are padding and are
 * skipped.  A slot >= num_blocks * bs is skipped and reported as
 * PA_ERR_DEVICE_BOUNDS.  Two tokens with the same slot race (undefined which
 * value lands); pa_validate_slot_mapping() detects that case.
 * k_scale / v_scale are ignored for 16-bit caches and must be finite and
 * > 0 for e4m3.
 */
pa_status pa_write_kv(const void* k, const void* v, pa_dtype in_dtype,
                      const int64_t* slot_mapping, int32_t num_tokens,
                      void* k_pool, void* v_pool, pa_dtype cache_dtype,
                      int32_t num_blocks, int32_t block_size,
                      int32_t num_kv_heads, int32_t head_dim,
                      float k_scale, float v_scale, pa_stream_t stream);

/*
 * pa_copy_blocks -- copy-on-write block copy ("Diziler Arasinda Bloklari
 * Paylasma": a block that others still use is copied before it is written).
 * For each pair p: k_pool[dst] = k_pool[src] and v_pool[dst] = v_pool[src],
 * all bs * Hkv * D elements, with (src, dst) = src_dst_pairs[p].
 * Pairs must not chain or collide (no dst equal to another pair's src or
 * dst); pa_validate_copy_pairs() checks that.  An id outside [0, num_blocks)
 * skips the pair and reports PA_ERR_DEVICE_BOUNDS.  num_pairs == 0 is a no-op.
 */
pa_status pa_copy_blocks(void* k_pool, void* v_pool, pa_dtype cache_dtype,
                         int32_t num_blocks, int32_t block_size,
                         int32_t num_kv_heads, int32_t head_dim,
                         const int64_t* src_dst_pairs, int32_t num_pairs,
                         pa_stream_t stream);

/*
 * pa_swap_blocks -- move blocks between two pools of the same block shape,
 * e.g. out of the device pool into pinned host memory when device memory is
 * full and back in when they are needed again: the pages' fine-grained
 * eviction, which moves small pages instead of whole sequences to the CPU
 * (gyaansetu, first article, the fine-grained eviction bullet of how
 * PagedAttention solves the memory problem).
 * For each pair p: dst_k[dst] = src_k[src] and dst_v[dst] = src_v[src], all
 * bs * Hkv * D elements, with (src, dst) = src_dst_pairs[p] (src indexes the
 * source pool, dst the destination pool).  Each pool pointer is device memory
 * or host memory the device can address (pinned by cudaHostAlloc /
 * cudaHostRegister under unified addressing); pageable host memory is
 * refused with PA_ERR_MEMORY.  src_dst_pairs lives in device memory.  One
 * launch moves all pairs; bytes cross the host link once.  Ids outside their
 * pool skip the pair and report PA_ERR_DEVICE_BOUNDS.  Destinations must be
 * distinct, and the two pools must not overlap.
 */
pa_status pa_swap_blocks(const void* src_k, const void* src_v, int32_t src_blocks,
                         void* dst_k, void* dst_v, int32_t dst_blocks,
                         pa_dtype cache_dtype, int32_t block_size,
                         int32_t num_kv_heads, int32_t head_dim,
                         const int64_t* src_dst_pairs, int32_t num_pairs,
                         pa_stream_t stream);

/*
 * pa_hash_blocks -- chained hashes of full blocks of token ids, the key of a
 * prefix cache: hashing every block carries block sharing across requests
 * ("PagedAttention", Ultralytics glossary, section "Diziler Arasinda
 * Bloklari Paylasma": this is how vLLM implements prompt caching).  A block's
 * hash covers its own tokens and its parent block's hash, so equal hashes
 * mean equal prefixes (up to 64-bit collisions; a caller may compare tokens
 * on a hit).
 * For sequence s (token ids token_ids[s * token_stride ...], num_tokens[s] of
 * them) and every full block j < num_tokens[s] / block_size:
 *   inner_j = FNV1a64(the block's block_size ids, 4 little-endian bytes each)
 *   hash_j  = FNV1a64(hash_{j-1} as 8 LE bytes, inner_j as 8 LE bytes),
 *   hash_{-1} = 0,
 * with FNV1a64 the 64-bit FNV-1a hash (offset basis 0xcbf29ce484222325,
 * prime 0x100000001b3).  block_hashes[s * max_blocks + j] = hash_j; entries
 * of blocks that are not full are 0.  A length above token_stride, or more
 * full blocks than max_blocks, is clamped and reported as
 * PA_ERR_DEVICE_BOUNDS.  All pointers are device pointers.
 */
pa_status pa_hash_blocks(const int32_t* token_ids, int64_t token_stride,
                         const int32_t* num_tokens, int32_t num_seqs,
                         int32_t block_size, uint64_t* block_hashes,
                         int32_t max_blocks, pa_stream_t stream);

/*
 * pa_decode_split_tokens -- the context-split length that sizes pa_decode's
 * workspace for these sizes: the automatic choice when split_tokens == 0,
 * else split_tokens rounded up to a multiple of block_size and raised, if
 * needed, so that no sequence has more than 1024 ranges.  A value >=
 * max_context_len means every (sequence, kv head) is one work item and
 * nothing is merged.  With split_tokens == 0 and a value below
 * max_context_len, pa_decode's planning kernel may lengthen the ranges on
 * the device, from the lengths it reads, to about
 *   (sum of the valid context_lens) * num_kv_heads * ceil(G / 8) / I
 * tokens (G = query heads per kv head; I = 15/16 of 148 SMs times the decode
 * kernel's resident blocks per SM), in whole blocks, never below this value
 * and never past max_context_len, so that a batch of a few long and many
 * short contexts is cut by its total rather than by its longest context; the
 * length used is left in the workspace (see pa_decode).  Returns 0 on
 * invalid arguments.
 */
int32_t pa_decode_split_tokens(int32_t num_seqs, int32_t num_kv_heads,
                               int32_t block_size, int32_t max_context_len,
                               int32_t split_tokens);

/*
 * pa_decode_workspace_size -- bytes of device workspace pa_decode needs for
 * these sizes (work counter, per-sequence item offsets, and the split
 * partials: one fp32 log-sum-exp and one fp32 [D] vector per (item, q head)).
 * Returns 0 on invalid arguments.  With split_tokens == 0 the automatic
 * split grows with num_seqs, so a smaller batch can need MORE workspace
 * than a larger one: a caller that keeps one workspace for many batch
 * sizes takes the largest size over them, or passes a fixed split_tokens
 * (then the size grows with num_seqs).  pa_decode refuses a smaller
 * workspace with PA_ERR_WORKSPACE before any launch.
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_context_len,
                                int32_t split_tokens);

/*
 * pa_decode -- single-query decode attention over the paged cache.
 * The attention kernel follows each sequence's block table to gather keys and
 * values block by block ("Sayfalama Nasil Calisir"), in the tiled
 * FlashAttention style that never writes the score matrix to memory ("Ilgili
 * Teknikler", Flash Attention bullet), with the query heads of one KV head
 * packed together (same section, grouped-query attention bullet).
 *
 * For every sequence s and query head h (kv head kvh = h / (Hq / Hkv)), with
 * n = context_lens[s] and K_s, V_s the first n token rows gathered through
 * block_tables[s]:
 *   z_t    = scale * k_scale * <q[s][h], K_s[t][kvh]>          t < n
 *   out[s][h] = v_scale * sum_t softmax(z)_t * V_s[t][kvh]
 * (k_scale = v_scale = 1 for 16-bit caches), accumulated in fp32 and
 * rounded to q's dtype (round to nearest even).  n == 0 gives zeros.
 *
 * A context longer than the split length S (split_tokens, or the automatic
 * choice when it is 0, see pa_decode_split_tokens) is cut into
 * n = ceil(len / S) ranges of whole blocks, as equal as blocks allow (the
 * first ceil-share ranges one block longer), none longer than S; each range
 * writes a partial (log-sum-exp, normalised vector) into the workspace, and
 * the kernel that finishes a sequence's last range combines them
 * (log-sum-exp merge).
 * Results depend only on the arguments (not on the grid or on timing): the
 * same call gives bit-identical outputs.
 *
 * max_context_len must bound every context_lens[s]; a larger length, or one
 * above max_blocks_per_seq * bs, makes that sequence's output zero and
 * reports PA_ERR_DEVICE_BOUNDS.  A table entry outside [0, num_blocks) is
 * skipped (its tokens left out) and reported the same way.  The pools must be
 * 16-byte aligned (they are read through TMA tensor maps).
 * workspace: device memory of at least pa_decode_workspace_size(...) bytes,
 * 256-byte aligned, used only during the call (stream-ordered).  When the
 * call has completed, the int32 at byte offset 8 of the workspace holds the
 * range length it used; passing that value as split_tokens reproduces the
 * output bit for bit.
 * The call enqueues two kernels on `stream`: a one-block planning kernel,
 * then the attention kernel, launched with programmatic stream
 * serialization so that its blocks set up while the plan runs and read the
 * plan only once it has completed.  When no context is split and the work
 * items (sequences x kv heads x groups of up to 8 query heads) fit the
 * GPU's resident attention blocks at once, there is no queue to plan: the
 * attention kernel runs alone, block c on item c.  Work before and after
 * the call on the stream is ordered as usual; the call can be captured in
 * a CUDA graph.
 */
pa_status pa_decode(void* out, const void* q, pa_dtype q_dtype,
                    const void* k_pool, const void* v_pool, pa_dtype cache_dtype,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t max_context_len,
                    int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                    int32_t head_dim, int32_t block_size, int32_t num_blocks,
                    float scale, float k_scale, float v_scale,
                    int32_t split_tokens,
                    void* workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode_shared_prefix_workspace_size -- bytes of device workspace
 * pa_decode_shared_prefix needs for these sizes (planning arrays, the work
 * list and the per-range partials).  Returns 0 on invalid arguments.
 */
size_t pa_decode_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                              int32_t num_kv_heads, int32_t head_dim,
                                              int32_t block_size, int32_t max_context_len,
                                              int32_t split_tokens);

/*
 * pa_decode_shared_prefix -- decode attention for sequences whose block
 * tables share leading blocks (samples forked from one prompt, beams, a
 * common system prompt: "PagedAttention", Ultralytics glossary, section
 * "Diziler Arasinda Bloklari Paylasma", where several tables name the same
 * physical blocks).  The result is pa_decode's (same formula, same
 * arguments; up to fp32 rounding order, within the attention tolerance),
 * but the shared blocks are read from memory once per group instead of
 * once per member:
 *   - group g lists its sequences in group_seqs[group_start[g] ..
 *     group_start[g+1]) (device int32 arrays; group_start has num_groups + 1
 *     entries, non-decreasing from 0, group_seqs group_start[num_groups]).
 *     Sequences in no group are decoded on their own.  A sequence listed
 *     twice, or outside [0, num_seqs), makes its group(s) decode unshared
 *     and is reported as PA_ERR_RANGE at the next pa_sync_status.
 *   - the shared part of a group is found on the device: the longest run of
 *     leading table entries equal in every member's row, cut so that each
 *     member keeps at least one token of its own.  Groups of one member, or
 *     with a length outside [1, max_context_len], share nothing.
 *   - up to 16 / (Hq/Hkv) members form a chunk whose query heads are the
 *     rows of one tile: the shared blocks are attended once by all rows,
 *     each member's own blocks by its own heads, in ranges of blocks whose
 *     partial results are merged by log-sum-exp.  With more than 8 query
 *     heads per kv head a chunk is one member (its heads fill the tile).
 * Supported: as pa_decode's caches (f16 with q f16, bf16 with q bf16, e4m3
 * with q f16 or bf16 and the per-tensor k_scale / v_scale, which are ignored
 * for 16-bit caches), head_dim 64 or 128, block_size 16 or 32, Hq / Hkv <= 16.
 * split_tokens: 0 = automatic, else the shortest range in tokens.
 * workspace: at least pa_decode_shared_prefix_workspace_size(...) bytes,
 * 256-byte aligned, stream-ordered use only.  Other errors as pa_decode.
 */
pa_status pa_decode_shared_prefix(void* out, const void* q, pa_dtype q_dtype,
                                  const void* k_pool, const void* v_pool, pa_dtype cache_dtype,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t max_context_len,
                                  const int32_t* group_start, const int32_t* group_seqs,
                                  int32_t num_groups, int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t num_blocks, float scale, float k_scale, float v_scale,
                                  int32_t split_tokens, void* workspace, size_t workspace_bytes,
                                  pa_stream_t stream);

/*
 * pa_prefill -- paged prefill / chunked-prefill attention on the 5th-
 * generation tensor cores.  Several new query tokens per sequence attend
 * causally to the sequence's cached keys and values, gathered block by block
 * through its block table by FlashAttention-style tiles ("PagedAttention",
 * Ultralytics glossary, section "Ilgili Teknikler": current engines run
 * FlashAttention-style kernels that read from paged blocks).
 * Sequence s has n_s = query_start[s+1] - query_start[s] new tokens, rows
 * query_start[s] .. +n_s of q and out ([total_q, Hq, D], packed), at positions
 * context_lens[s] - n_s .. context_lens[s] - 1; their K/V must already be in
 * the cache (pa_write_kv).  Token i at position p, query head h (kv head
 * h / (Hq / Hkv)):
 *   out = sum_{t <= p} softmax_t(scale * <q, K_s[t]>) V_s[t]
 * accumulated in fp32, rounded to q's dtype.  query_start is int32 [B + 1],
 * device memory.  Supported: head_dim 64 or 128; q and cache both f16 or both
 * bf16; G = Hq / Hkv <= 128 (a CTA takes floor(128 / G) new tokens);
 * block_size 16 or 32.  max_query_len must
 * bound every n_s (rows past it are not computed) and max_context_len every
 * context length; a length below n_s or above the maxima zeroes that
 * sequence's rows and reports PA_ERR_DEVICE_BOUNDS.  No workspace.
 */
pa_status pa_prefill(void* out, const void* q, pa_dtype q_dtype,
                     const void* k_pool, const void* v_pool, pa_dtype cache_dtype,
                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* context_lens, const int32_t* query_start,
                     int32_t num_seqs, int32_t max_query_len, int32_t max_context_len,
                     int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t block_size, int32_t num_blocks, float scale,
                     pa_stream_t stream);

/*
 * pa_sync_status -- synchronise `stream`, then read and clear the device
 * error word of the current device.  Returns PA_OK, PA_ERR_DEVICE_BOUNDS,
 * PA_ERR_TIMEOUT or PA_ERR_CUDA (an asynchronous CUDA error).
 */
pa_status pa_sync_status(pa_stream_t stream);

/* Message of the last failing call on this host thread ("" if none).  The
 * pointer stays valid until the next call on this thread. */
const char* pa_last_error(void);

/*
 * Debug checks of index contents (they copy the indices to the host and
 * synchronise `stream`; not for the hot path):
 *  pa_validate_slot_mapping: every slot < num_blocks * bs, no slot twice
 *    (negative slots ignored)                -> PA_ERR_RANGE / PA_ERR_ALIAS
 *  pa_validate_copy_pairs: ids in [0, num_blocks), no dst twice, no dst that
 *    is also a src                           -> PA_ERR_RANGE / PA_ERR_ALIAS
 *  pa_validate_block_tables: 0 <= context_lens[s] <= max_context_len,
 *    ceil(len / bs) <= max_blocks_per_seq, and every entry the sequence
 *    reads in [0, num_blocks)                -> PA_ERR_RANGE
 */
pa_status pa_validate_slot_mapping(const int64_t* slot_mapping, int32_t num_tokens,
                                   int32_t num_blocks, int32_t block_size,
                                   pa_stream_t stream);
pa_status pa_validate_copy_pairs(const int64_t* src_dst_pairs, int32_t num_pairs,
                                 int32_t num_blocks, pa_stream_t stream);
pa_status pa_validate_block_tables(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* context_lens, int32_t num_seqs,
                                   int32_t max_context_len, int32_t block_size,
                                   int32_t num_blocks, pa_stream_t stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device
 * memory.  (The pages have no counterpart to this call; it exists for
 * library users.)
 *
 * Some callers may not call cudaMalloc at all: a kernel plugin inside a host
 * framework that owns every device allocation and hands the plugin only its
 * inputs and outputs, or a serving loop whose memory is budgeted up front and
 * where an allocation call could block until the device is idle.  Such a
 * caller still passes q, the pools, the tables and `out`, but no workspace:
 * this entry point takes pa_decode's scratch (work counter, range offsets,
 * split partials) from one array of PA_DECODE_NOALLOC_SCRATCH_BYTES bytes
 * that the library reserves in device memory; every GPU that loads the
 * library holds that array until the process exits.
 *
 * Arguments and results are exactly those of pa_decode without `workspace`
 * and `workspace_bytes`.  A call whose scratch need
 * (pa_decode_workspace_size of the same sizes) exceeds
 * PA_DECODE_NOALLOC_SCRATCH_BYTES is refused with PA_ERR_WORKSPACE before any
 * launch; a larger split_tokens (fewer context ranges) lowers the need.
 * The first call on a device looks up the array's device address with
 * cudaGetSymbolAddress (once per device, with that device current); make
 * that first call before any stream capture begins.  The address is kept
 * per CUDA context: after cudaDeviceReset, or under another context of the
 * same device, the next call looks it up again (so make that call, too,
 * before a capture).  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 * Every call shares the one array and finds the previous call's contents in
 * it; the work counter that must start at zero is cleared by the call's own
 * first kernel.  Calls that overlap on the GPU (other streams, other host
 * threads) race on the array: order them on one stream.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
pa_status pa_decode_noalloc(void* out, const void* q, pa_dtype q_dtype,
                            const void* k_pool, const void* v_pool, pa_dtype cache_dtype,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t max_context_len,
                            int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            float scale, float k_scale, float v_scale,
                            int32_t split_tokens, pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H_ */
