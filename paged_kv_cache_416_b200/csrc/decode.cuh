// Paged single-query decode attention for sm_100a.
//
// Method ("PagedAttention", Ultralytics glossary): a sequence's keys and
// values live in fixed-size blocks scattered through one pool; the kernel
// follows the sequence's block table and gathers them block by block
// (section "Sayfalama Nasil Calisir"), computing attention tile by tile so
// the score matrix never reaches memory (section "Ilgili Teknikler", Flash
// Attention bullet), with the G = Hq / Hkv query heads of one KV head
// packed together so every cache byte is read once (same section, grouped-
// query attention bullet).
//
// Work decomposition
//   item  = (sequence, context range, kv head, group of <= 8 of its q heads)
//   CTA   = 4 warps; a persistent grid pulls items from an atomic counter
//   warp  = takes every 4th block of the item's range; each warp owns a ring
//           of kStages shared-memory stages, one stage = the K tile and the V
//           tile of one block for one kv head, each tile filled by ONE tiled
//           TMA copy (cp.async.bulk.tensor through a tensor map over the
//           pool, box = bs token rows of one head, 128B/64B swizzle so that
//           ldmatrix is free of bank conflicts; completion counted in bytes
//           on an mbarrier; no multicast)
// Per block and warp, with the packed heads as the MMA's N = 8 columns:
//   S^T[t, g] = K[t, :] . Q[g, :]        m16n8k16, A = K rows (ldmatrix)
//   online softmax over t per column g   (exp2, running max and sum)
//   O^T[d, g] += V^T[d, t] P^T[t, g]     A = V (ldmatrix.trans), B = P^T
//                                         (S^T fragment transposed in
//                                         registers with movmatrix)
// The warps' partial (max, sum, O) are merged through shared memory at the
// end of an item; a split item writes (log-sum-exp, O / sum) to the
// workspace, and the CTA that finishes the last range of a (sequence, kv
// head) combines them (log-sum-exp merge) and writes the output.
#pragma once

#include <cuda.h>  // CUtensorMap

#include "common.cuh"

namespace pa {

enum CacheKind : int { kCacheF16 = 0, kCacheBF16 = 1, kCacheE4M3 = 2 };

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kMaxGroup = 8;          // packed query heads per work item (MMA N); a kv
                                      // head with more query heads is several items
constexpr int kBarrierBytes = 256;    // mbarrier area at the start of smem
constexpr int kTileAlign = 1024;      // swizzled tiles start on this boundary
constexpr int kMaxRanges = 1024;      // context ranges per sequence (fused merge uses smem)

template <int CK, int D, int BS>
struct DecodeCfg {
  static constexpr int kBS = BS;
  static constexpr int kElem = (CK == kCacheE4M3) ? 1 : 2;
  static constexpr int kRowBytes = D * kElem;                    // one token row of one head
  static constexpr int kSwzBytes = kRowBytes >= 128 ? 128 : 64;  // bytes per swizzle row
  static constexpr int kHalves = kRowBytes / kSwzBytes;          // swizzle rows per token row
  static constexpr int kSwzMask = kSwzBytes == 128 ? 7 : 3;      // 128B / 64B swizzle
  static constexpr int kTileBytes = BS * kRowBytes;              // one tensor, one block
  static constexpr int kStageBytes = 2 * kTileBytes;             // K tile then V tile
  // stage memory per CTA: 70 KB lets three CTAs share an SM; e4m3 tiles of
  // 16-token blocks take 48 KB (3 stages per warp) so four fit (the e4m3
  // kernel needs 116 registers): 82.2 vs 86.2 us on the fp8 long-tail batch
  static constexpr int kBudget = (CK == kCacheE4M3 && BS == 16 && D == 128 ? 48 : 70) * 1024;
  static constexpr int kStagesRaw = kBudget / (kDecodeWarps * kStageBytes);
  static constexpr int kStages = kStagesRaw < 1 ? 1 : (kStagesRaw > 6 ? 6 : kStagesRaw);
  static constexpr int kWarpBytes = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarrierBytes + kTileAlign + kDecodeWarps * kWarpBytes;
  static constexpr int kTokTiles = BS / 16;
  static constexpr int kDimTiles = D / 16;
  static constexpr bool kMmaBF16 = (CK == kCacheBF16);
  // merge scratch of one warp: O[8][D] fp32, then max[8], sum[8]
  static constexpr int kScratchBytes = (kMaxGroup * D + 2 * kMaxGroup) * 4;
  static_assert(kWarpBytes >= kScratchBytes, "warp ring too small for the merge scratch");
  static_assert(kDecodeWarps * kStages <= kBarrierBytes / 8, "too many mbarriers");
  static_assert(kRowBytes == 64 || kRowBytes % 128 == 0, "unsupported row size");
  static_assert(kTileBytes % (8 * kSwzBytes) == 0, "tiles must hold whole swizzle atoms");
  static_assert(kWarpBytes % kTileAlign == 0 || kDecodeWarps == 1, "rings keep tiles aligned");
  static_assert(kDecodeWarps * kWarpBytes >= (kMaxRanges + 1) * kMaxGroup * 4,
                "the rings must hold the fused merge's weights");
};

// Byte offset of (token row t, byte b of the row) inside a swizzled tile.
// The tile holds kHalves groups of BS rows of kSwzBytes bytes; the TMA
// swizzle XORs the 16-byte chunk index with address bits 7.. (mask 7 for
// 128B, 3 for 64B), which the tile's kTileAlign alignment makes equal to the
// offset's bits.
template <class C>
__device__ __forceinline__ uint32_t tile_off(int t, int b) {
  const int row = (b / C::kSwzBytes) * C::kBS + t;
  const uint32_t o = static_cast<uint32_t>(row * C::kSwzBytes);
  const uint32_t chunk = static_cast<uint32_t>((b % C::kSwzBytes) >> 4);
  return o + ((chunk ^ ((o >> 7) & C::kSwzMask)) << 4);
}

// Tiled TMA load of a 5-D box: tensor map coordinates (x innermost).
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, int c4, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(c4), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

struct DecodeArgs {
  // Tensor maps over the pools, viewed as 5-D bytes (x, token, half, kv head,
  // block) = (kSwzBytes, bs, kHalves, Hkv, N); box (kSwzBytes, bs, kHalves, 1, 1).
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int32_t* counter;        // workspace: work-queue counter (zeroed by plan_kernel)
  const int32_t* total;    // workspace: number of items (written by plan_kernel)
  const int32_t* seq_off;  // workspace: [B + 1] first range index of each sequence
  const int4* order;       // workspace: [ranges] (sequence, range | ranges of the
                           // sequence << 16, first token, end token), longest range first
  int32_t* arrived;        // workspace: [B * Hkv] ranges finished per (sequence, kv head)
  float* lse_part;         // workspace: [ranges * Hq]
  float* o_part;           // workspace: [ranges * Hq * D]
  int num_seqs, hq, hkv, group, max_blocks, num_blocks, max_ctx;
  int ncg;                 // column groups per kv head: ceil(group / 8) items read its blocks
  float sl2;               // scale * k_scale * log2(e)
  float out_scale;         // v_scale
  // direct = 1: no planning kernel ran (unsplit contexts, one item per CTA):
  // CTA c takes item c, whose descriptor it forms from the context length,
  // and CTA 0 writes split_len to *split_out as the plan would
  int direct;
  int split_len;
  int32_t* split_out;
};

// ---------------------------------------------------------------- planning
constexpr int kPlanBuckets = 256;  // range-length classes of the longest-first order

// One CTA of 1024 threads, once per decode call:
//  0. with adapt_items > 0 (the automatic split), lengthens the range
//     length S to about (sum of the valid lengths) x units / adapt_items
//     tokens, rounded up to whole blocks (never below S, whose ranges the
//     workspace holds, never past one range per sequence); writes the length
//     used to *split_out;
//  1. validates the context lengths (an out-of-range length counts as 0 and
//     is reported), counts each sequence's ranges n = max(1, ceil(len / S))
//     and writes their exclusive prefix sum seq_off (where a sequence's
//     partials go) and the item total (ranges * Hkv); zeroes the work
//     counter.  A sequence's nb blocks are dealt out evenly: its first
//     nb % n ranges take floor(nb / n) + 1 blocks, the others floor(nb / n)
//     (never more than S tokens), so no short remnant range of a split
//     sequence, with the merge it triggers, is left for the end of the queue;
//  2. writes the work order: every (sequence, range) pair with the range's
//     first and end token and the sequence's range count, longest range first
//     (counting sort over kPlanBuckets length classes), so that the
//     short ranges fill the end of the persistent grid's queue.  The order
//     inside a class is whatever the atomics give: outputs do not depend on
//     it, because every item writes its own output or partial slot.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ ctx_lens, int B,
                                                    int max_ctx, int max_blocks, int bs, int S,
                                                    int adapt_items, int hkv, int32_t* counter,
                                                    int32_t* total, int32_t* split_out,
                                                    int32_t* seq_off, int4* order,
                                                    int32_t* arrived) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  __shared__ int hist[kPlanBuckets];
  __shared__ long long warp_sum[32];
  __shared__ int s_split;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_launch_dependents();  // the decode grid may set up while the plan runs
  auto valid_len = [&](int s) {
    const int c = ctx_lens[s];
    return (c < 0 || c > max_ctx || c > max_blocks * bs) ? -1 : c;
  };
  // the thread's first sequence (s = tid) is read once and kept for every pass
  const int c_own = tid < B ? valid_len(tid) : 0;
  auto len_of = [&](int s) { return s == tid ? c_own : valid_len(s); };
  if (adapt_items > 0) {
    long long sum = 0;
    for (int s = tid; s < B; s += 1024) sum += max(0, len_of(s));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) warp_sum[warp] = sum;
    __syncthreads();
    if (warp == 0) {
      sum = warp_sum[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const long long want = (sum * hkv + adapt_items - 1) / adapt_items;
        const long long blocks = (want + bs - 1) / bs;
        const long long cap = (static_cast<long long>(max_ctx) + bs - 1) / bs;  // one range
        s_split = static_cast<int>(max(static_cast<long long>(S), min(blocks, cap) * bs));
      }
    }
    __syncthreads();
    S = s_split;
  }
  const int max_nb = (min(S, max_ctx) + bs - 1) / bs;  // blocks of the longest range
  auto bucket = [&](int nb) {  // longer ranges -> higher class
    return max_nb < kPlanBuckets ? nb : static_cast<int>((static_cast<int64_t>(nb) * (kPlanBuckets - 1)) / max_nb);
  };
  if (tid == 0) {
    carry = 0;
    *counter = 0;
    *split_out = S;
  }
  if (tid < kPlanBuckets) hist[tid] = 0;
  if (arrived != nullptr)
    for (int i = tid; i < B * hkv; i += 1024) arrived[i] = 0;
  __syncthreads();
  for (int base = 0; base < B; base += 1024) {
    const int s = base + tid;
    int n = 0;
    if (s < B) {
      int c = len_of(s);
      if (c < 0) {
        record_error(PA_ERR_DEVICE_BOUNDS);
        c = 0;
      }
      n = c > 0 ? (c + S - 1) / S : 1;
      const int nb = (c + bs - 1) / bs;
      const int q = nb / n, ex = nb % n;  // ex ranges of q + 1 blocks, n - ex of q
      if (ex > 0) atomicAdd(&hist[bucket(q + 1)], ex);
      atomicAdd(&hist[bucket(q)], n - ex);
    }
    int x = n;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int incl = x + (warp > 0 ? warp_tot[warp - 1] : 0) + carry;
    if (s < B) seq_off[s] = incl - n;
    __syncthreads();
    if (tid == 1023) carry = incl;
    __syncthreads();
  }
  if (tid == 0) {
    seq_off[B] = carry;
    *total = carry * hkv;
  }
  // class starts, longest class first: start[b] = sum of hist[b'] for b' > b
  if (warp == 0) {
    constexpr int kPer = kPlanBuckets / 32;
    int v[kPer], sum = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {  // lane owns classes from the top down
      v[i] = hist[kPlanBuckets - 1 - (lane * kPer + i)];
      sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      hist[kPlanBuckets - 1 - (lane * kPer + i)] = run;  // becomes the class's cursor
      run += v[i];
    }
  }
  __syncthreads();
  for (int s = tid; s < B; s += 1024) {
    int c = len_of(s);
    if (c < 0) c = 0;
    const int n = c > 0 ? (c + S - 1) / S : 1;
    const int nb = (c + bs - 1) / bs;
    const int q = nb / n, ex = nb % n;
    const int p1 = ex > 0 ? atomicAdd(&hist[bucket(q + 1)], ex) : 0;
    const int p0 = atomicAdd(&hist[bucket(q)], n - ex);
    for (int r = 0; r < n; ++r) {
      const int b0 = r * q + min(r, ex);     // first block of range r
      const int b1 = b0 + q + (r < ex ? 1 : 0);
      order[r < ex ? p1 + r : p0 + r - ex] = make_int4(s, r | (n << 16), b0 * bs, min(c, b1 * bs));
    }
  }
}

// Keep the halves of a 32-bit fragment register whose token is valid:
// low half <- token t, high half <- token t + 1.
__device__ __forceinline__ uint32_t pair_mask(bool lo_ok, bool hi_ok) {
  return (lo_ok ? 0x0000ffffu : 0u) | (hi_ok ? 0xffff0000u : 0u);
}

// ------------------------------------------------------------ main kernel
template <int CK, bool kQBF16, int D, int BS>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const __grid_constant__ DecodeArgs a) {
  using C = DecodeCfg<CK, D, BS>;
  constexpr bool kMmaBF16 = C::kMmaBF16;
  constexpr int kStages = C::kStages;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_item;   // the CTA's next item ...
  __shared__ int4 s_desc;  // ... and its descriptor (a.order entry)
  __shared__ int s_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;    // fragment row group
  const int tig = lane & 3;   // thread in group

  // stage rings start on a kTileAlign boundary after the mbarriers
  const uint32_t smem_s = smem_addr(smem);
  const uint32_t ring_s = (smem_s + kBarrierBytes + kTileAlign - 1) & ~uint32_t(kTileAlign - 1);
  const uint32_t wbase_s = ring_s + warp * C::kWarpBytes;
  uint8_t* const ring = smem + (ring_s - smem_s);
  uint8_t* const wbase = ring + warp * C::kWarpBytes;
  const uint32_t bar0 = smem_s + warp * kStages * 8;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&a.tmap_k);
    prefetch_tensormap(&a.tmap_v);
  }
  // launched behind plan_kernel (or, direct, behind whatever wrote the cache):
  // nothing from global memory before it is done
  grid_dependency_wait();
  __syncthreads();

  const int total = a.direct ? a.num_seqs * a.hkv * a.ncg : *a.total;
  uint32_t n_issued = 0, n_consumed = 0;  // warp-uniform ring counters
  uint32_t skip_stage = 0;                // stages holding a block with a bad table entry
  bool failed = false;                    // a wait timed out: stop issuing / computing

  // the next item and its descriptor, fetched by thread 0: CTA c starts on
  // item c (no atomic on the path to the first tile); later items come from
  // the counter, past the grid's first ones
  auto fetch_next = [&](bool first) {
    const int it = first ? static_cast<int>(blockIdx.x)
                   : a.direct ? total  // one item per CTA
                              : static_cast<int>(gridDim.x) + atomicAdd(a.counter, 1);
    s_item = it;
    if (it < total) {
      if (a.direct) {  // the whole context as one range, validated as the plan does
        const int seq = it / (a.hkv * a.ncg);
        int c = a.context_lens[seq];
        if (c < 0 || c > a.max_ctx || c > a.max_blocks * BS) {
          if (it % (a.hkv * a.ncg) == 0) record_error(PA_ERR_DEVICE_BOUNDS);
          c = 0;
        }
        s_desc = make_int4(seq, 1 << 16, 0, c);
      } else {
        s_desc = a.order[it / (a.hkv * a.ncg)];
      }
    }
    if (a.direct && first && blockIdx.x == 0) *a.split_out = a.split_len;
  };
  if (threadIdx.x == 0) fetch_next(true);
  __syncthreads();

  for (;;) {
    const int item = s_item;
    if (item >= total) break;

    // ---- item -> (sequence, range, kv head); kv heads innermost, so the
    // heads of one range run side by side and share the table's cache lines
    // the kv head's query heads are cut into column groups of at most 8 (the
    // MMA's N); each group is its own item over the same blocks
    const int kvh_cg = item % (a.hkv * a.ncg);
    const int kvh = kvh_cg / a.ncg, cg = kvh_cg % a.ncg;
    const int ncols = min(kMaxGroup, a.group - cg * kMaxGroup);  // heads of this item
    const int4 desc = s_desc;
    const int seq = desc.x;
    const int split = desc.y & 0xffff;  // range index ...
    const int nsplit = desc.y >> 16;    // ... of this many
    const int t0 = desc.z;  // first token of the range (a block boundary) ...
    const int t1 = desc.w;  // ... and its end (both validated by plan_kernel)
    const int jb0 = t0 / BS;
    const int nblk = t1 > t0 ? (t1 + BS - 1) / BS - jb0 : 0;
    const int nb_w = nblk > warp ? (nblk - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
    const int32_t* table = a.block_tables + static_cast<int64_t>(seq) * a.max_blocks;
    const int h0 = kvh * a.group + cg * kMaxGroup;

    // ---- block-table entries of the warp's blocks, prefetched in registers:
    // lane l holds the entry of the warp's block (32 * chunk + l); tab_cur is
    // the chunk the issue cursor is in, tab_nxt the one after it, so the
    // table read never sits on the path from one block to the next
    auto load_chunk = [&](int c) -> int {
      const int i = c * 32 + lane;
      return i < nb_w ? table[jb0 + warp + i * kDecodeWarps] : -1;
    };
    int tab_chunk = 0;
    int tab_cur = load_chunk(0);
    int tab_nxt = load_chunk(1);

    // ---- issue the two tile loads of the warp's i-th block of this item
    // (i increases by at most one chunk between calls)
    auto issue = [&](int i) {
      const int st = n_issued % kStages;
      const uint32_t bar = bar0 + 8 * st;
      const uint32_t sK = wbase_s + st * C::kStageBytes;
      if ((i >> 5) != tab_chunk) {
        tab_chunk = i >> 5;
        tab_cur = tab_nxt;
        tab_nxt = load_chunk(tab_chunk + 1);
      }
      const int phys = __shfl_sync(0xffffffffu, tab_cur, i & 31);
      const bool ok = phys >= 0 && phys < a.num_blocks;
      skip_stage = ok ? (skip_stage & ~(1u << st)) : (skip_stage | (1u << st));
      fence_proxy_async_smem();  // this lane's earlier generic accesses of the stage first
      __syncwarp();
      if (lane == 0) {
        if (ok) {
          mbar_arrive_expect_tx(bar, 2u * C::kTileBytes + PA_TEST_STAGE_EXTRA_TX);
          tma_load_5d(sK, &a.tmap_k, 0, 0, 0, kvh, phys, bar);
          tma_load_5d(sK + C::kTileBytes, &a.tmap_v, 0, 0, 0, kvh, phys, bar);
        } else {
          record_error(PA_ERR_DEVICE_BOUNDS);  // the block's tokens are left out
          mbar_arrive_expect_tx(bar, 0u);
        }
      }
      ++n_issued;
    };

    if (!failed) {
      const int pro = min(kStages, nb_w);
      for (int i = 0; i < pro; ++i) issue(i);
    }

    // ---- query fragments (B operand of S^T = K Q^T): rows = dims, cols = heads.
    // With an e4m3 cache the products run in fp16, so each head's query is
    // first scaled by a power of two 2^-e that brings its largest |q| into
    // [2^14, 2^15): any f16 or bf16 query fits, and 2^e goes back into that
    // head's softmax scale (exact: a power of two scales every product and
    // partial sum of the fp32 accumulation exactly).
    uint32_t qf[C::kDimTiles][2];
    float sl2c[2] = {a.sl2, a.sl2};  // softmax scale of heads 2tig, 2tig+1 (log2 units)
    {
      const bool hv = g < ncols;
      const uint16_t* qrow = reinterpret_cast<const uint16_t*>(a.q) +
                             (static_cast<int64_t>(seq) * a.hq + h0 + (hv ? g : 0)) * D;
      if constexpr (CK == kCacheE4M3) {
        // dims 16ks + 4tig .. +3 (the order ldmatrix gives 8-bit K rows)
        uint2 qw[C::kDimTiles];
        float amax = 0.f;
#pragma unroll
        for (int ks = 0; ks < C::kDimTiles; ++ks) {
          qw[ks] = hv ? *reinterpret_cast<const uint2*>(qrow + ks * 16 + 4 * tig) : make_uint2(0u, 0u);
          amax = fmax3(amax, fabsf(to_float<kQBF16>(qw[ks].x & 0xffff)),
                       fabsf(to_float<kQBF16>(qw[ks].x >> 16)));
          amax = fmax3(amax, fabsf(to_float<kQBF16>(qw[ks].y & 0xffff)),
                       fabsf(to_float<kQBF16>(qw[ks].y >> 16)));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));  // the head's 4 threads
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        // e in [-126, 126]; 0 for a zero (or non-finite) query
        const int e = (amax > 0.f && amax < INFINITY) ? max(-126, min(126, ilogbf(amax) - 14)) : 0;
        const float down = __int_as_float((127 - e) << 23);  // 2^-e
#pragma unroll
        for (int ks = 0; ks < C::kDimTiles; ++ks) {
          qf[ks][0] = pack_f16x2(to_float<kQBF16>(qw[ks].x & 0xffff) * down,
                                 to_float<kQBF16>(qw[ks].x >> 16) * down);
          qf[ks][1] = pack_f16x2(to_float<kQBF16>(qw[ks].y & 0xffff) * down,
                                 to_float<kQBF16>(qw[ks].y >> 16) * down);
        }
        // columns 2tig and 2tig+1 of the score tile are heads 2tig, 2tig+1,
        // whose exponents sit in row groups 2tig and 2tig+1
        const int e0 = __shfl_sync(0xffffffffu, e, 8 * tig);
        const int e1 = __shfl_sync(0xffffffffu, e, 8 * tig + 4);
        sl2c[0] = a.sl2 * __int_as_float((127 + e0) << 23);
        sl2c[1] = a.sl2 * __int_as_float((127 + e1) << 23);
      } else {
#pragma unroll
        for (int ks = 0; ks < C::kDimTiles; ++ks) {
          qf[ks][0] = hv ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * tig) : 0u;
          qf[ks][1] = hv ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * tig) : 0u;
        }
      }
    }

    float acc[C::kDimTiles][4];
#pragma unroll
    for (int dt = 0; dt < C::kDimTiles; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[dt][e] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};  // heads 2tig, 2tig+1 (log2 units)
    float l_run[2] = {0.f, 0.f};              // this thread's share of the sums

    const int li = lane >> 3;  // which 8x8 matrix of an ldmatrix.x4 this lane addresses
    for (int i = 0; i < nb_w; ++i) {
      const int st = n_consumed % kStages;
      const uint32_t par = (n_consumed / kStages) & 1u;
      if (!failed) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar0 + 8 * st, par));
        if (!ok) {
          failed = true;  // warp-uniform
          if (lane == 0) record_error(PA_ERR_TIMEOUT);
        }
      }
      if (!failed && !((skip_stage >> st) & 1u)) {
        const int j = jb0 + warp + i * kDecodeWarps;
        const int tbase = j * BS;
        const bool partial = tbase + BS > t1;  // rows past the range hold other data
        const uint32_t sK = wbase_s + st * C::kStageBytes;
        const uint32_t sV = sK + C::kTileBytes;

        // ---- S^T = K Q^T  (rows: tokens, cols: packed heads)
        float s[C::kTokTiles][4];
#pragma unroll
        for (int mt = 0; mt < C::kTokTiles; ++mt) {
          float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
          float s2[4] = {0.f, 0.f, 0.f, 0.f}, s3[4] = {0.f, 0.f, 0.f, 0.f};
          if constexpr (CK == kCacheE4M3) {
            const int tok = mt * 16 + (lane & 7) + (li & 1) * 8;
#pragma unroll
            for (int cp = 0; cp < C::kDimTiles / 2; ++cp) {
              uint32_t r0, r1, r2, r3;
              ldsm_x4(sK + tile_off<C>(tok, (2 * cp + (li >> 1)) * 16), r0, r1, r2, r3);
              const uint32_t a0[4] = {e4m3x2_to_f16x2(r0 & 0xffff), e4m3x2_to_f16x2(r1 & 0xffff),
                                      e4m3x2_to_f16x2(r0 >> 16), e4m3x2_to_f16x2(r1 >> 16)};
              const uint32_t a1[4] = {e4m3x2_to_f16x2(r2 & 0xffff), e4m3x2_to_f16x2(r3 & 0xffff),
                                      e4m3x2_to_f16x2(r2 >> 16), e4m3x2_to_f16x2(r3 >> 16)};
              if (cp & 1) {
                mma_16816<false>(s2, a0, qf[2 * cp][0], qf[2 * cp][1]);
                mma_16816<false>(s3, a1, qf[2 * cp + 1][0], qf[2 * cp + 1][1]);
              } else {
                mma_16816<false>(s0, a0, qf[2 * cp][0], qf[2 * cp][1]);
                mma_16816<false>(s1, a1, qf[2 * cp + 1][0], qf[2 * cp + 1][1]);
              }
            }
          } else {
            const int row = mt * 16 + (lane & 7) + (li & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < C::kDimTiles; ++ks) {
              uint32_t af[4];
              ldsm_x4(sK + tile_off<C>(row, (ks * 16 + (li >> 1) * 8) * 2), af[0], af[1], af[2],
                      af[3]);
              if ((ks & 3) == 0) mma_16816<kMmaBF16>(s0, af, qf[ks][0], qf[ks][1]);
              else if ((ks & 3) == 1) mma_16816<kMmaBF16>(s1, af, qf[ks][0], qf[ks][1]);
              else if ((ks & 3) == 2) mma_16816<kMmaBF16>(s2, af, qf[ks][0], qf[ks][1]);
              else mma_16816<kMmaBF16>(s3, af, qf[ks][0], qf[ks][1]);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = tbase + mt * 16 + g + (e >> 1) * 8;
            const float x = ((s0[e] + s1[e]) + (s2[e] + s3[e])) * sl2c[e & 1];
            s[mt][e] = tok < t1 ? x : -INFINITY;
          }
        }

        // ---- online softmax per head column
        float alpha[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float bm = -INFINITY;
#pragma unroll
          for (int mt = 0; mt < C::kTokTiles; ++mt) bm = fmaxf(bm, fmaxf(s[mt][c], s[mt][2 + c]));
          bm = shfl_xor_max(bm);
          const float mn = fmaxf(m_run[c], bm);
          alpha[c] = fast_exp2(m_run[c] - mn);
          m_run[c] = mn;
          float ps = 0.f;
#pragma unroll
          for (int mt = 0; mt < C::kTokTiles; ++mt) {
            s[mt][c] = fast_exp2(s[mt][c] - mn);
            s[mt][2 + c] = fast_exp2(s[mt][2 + c] - mn);
            ps += s[mt][c] + s[mt][2 + c];
          }
          l_run[c] = l_run[c] * alpha[c] + ps;
        }
#pragma unroll
        for (int dt = 0; dt < C::kDimTiles; ++dt) {
          acc[dt][0] *= alpha[0];
          acc[dt][1] *= alpha[1];
          acc[dt][2] *= alpha[0];
          acc[dt][3] *= alpha[1];
        }

        // ---- P^T as the B operand: transpose the 8x8 (token, head) tiles
        // With a bf16 cache, P = P_hi + P_lo in bf16: one bf16 value keeps 8
        // significant bits (error up to 2^-9 of each weight), which outputs
        // formed by cancellation cannot absorb; fp16 P keeps 11 and stays one.
        uint32_t pb[C::kTokTiles][2];
        uint32_t pl[C::kTokTiles][2];
        constexpr bool kPBF16 = (CK == kCacheBF16);
#pragma unroll
        for (int mt = 0; mt < C::kTokTiles; ++mt) {
          const uint32_t h0 = pack2<kPBF16>(s[mt][0], s[mt][1]);
          const uint32_t h1 = pack2<kPBF16>(s[mt][2], s[mt][3]);
          pb[mt][0] = movmatrix_trans(h0);
          pb[mt][1] = movmatrix_trans(h1);
          if constexpr (kPBF16) {
            pl[mt][0] = movmatrix_trans(pack_bf16x2(s[mt][0] - to_float<true>(h0 & 0xffff),
                                                    s[mt][1] - to_float<true>(h0 >> 16)));
            pl[mt][1] = movmatrix_trans(pack_bf16x2(s[mt][2] - to_float<true>(h1 & 0xffff),
                                                    s[mt][3] - to_float<true>(h1 >> 16)));
          }
        }

        // ---- O^T += V^T P^T  (rows: dims, cols: packed heads).  In a partial
        // block the V rows past the range are zeroed in the fragments (their
        // P is 0, but the rows may hold anything, NaN included).
#pragma unroll
        for (int mt = 0; mt < C::kTokTiles; ++mt) {
          uint32_t m_lo = 0xffffffffu, m_hi = 0xffffffffu;  // tokens 2tig(+1), 2tig+8(+9)
          if (partial) {
            const int tk = tbase + mt * 16 + 2 * tig;
            m_lo = pair_mask(tk < t1, tk + 1 < t1);
            m_hi = pair_mask(tk + 8 < t1, tk + 9 < t1);
          }
          if constexpr (CK == kCacheE4M3) {
            const int tok = mt * 16 + (lane & 7) + (li & 1) * 8;
#pragma unroll
            for (int cp = 0; cp < C::kDimTiles / 2; ++cp) {
              uint32_t r0, r1, r2, r3;
              ldsm_x4_trans(sV + tile_off<C>(tok, (2 * cp + (li >> 1)) * 16), r0, r1, r2, r3);
              if (partial) {
                r0 &= m_lo; r1 &= m_hi; r2 &= m_lo; r3 &= m_hi;
              }
              // bytes (tok 2tig: dim 2g, 2g+1 | tok 2tig+1: dim 2g, 2g+1) -> pairs per dim
              const uint32_t p0 = __byte_perm(r0, 0, 0x3120), p1 = __byte_perm(r1, 0, 0x3120);
              const uint32_t p2 = __byte_perm(r2, 0, 0x3120), p3 = __byte_perm(r3, 0, 0x3120);
              const uint32_t a0[4] = {e4m3x2_to_f16x2(p0 & 0xffff), e4m3x2_to_f16x2(p0 >> 16),
                                      e4m3x2_to_f16x2(p1 & 0xffff), e4m3x2_to_f16x2(p1 >> 16)};
              const uint32_t a1[4] = {e4m3x2_to_f16x2(p2 & 0xffff), e4m3x2_to_f16x2(p2 >> 16),
                                      e4m3x2_to_f16x2(p3 & 0xffff), e4m3x2_to_f16x2(p3 >> 16)};
              mma_16816<false>(acc[2 * cp], a0, pb[mt][0], pb[mt][1]);
              mma_16816<false>(acc[2 * cp + 1], a1, pb[mt][0], pb[mt][1]);
            }
          } else {
            const int tok = mt * 16 + (lane & 7) + (li >> 1) * 8;
#pragma unroll
            for (int dt = 0; dt < C::kDimTiles; ++dt) {
              uint32_t af[4];
              ldsm_x4_trans(sV + tile_off<C>(tok, (dt * 16 + (li & 1) * 8) * 2), af[0], af[1],
                            af[2], af[3]);
              if (partial) {
                af[0] &= m_lo; af[1] &= m_lo; af[2] &= m_hi; af[3] &= m_hi;
              }
              mma_16816<kMmaBF16>(acc[dt], af, pb[mt][0], pb[mt][1]);
              if constexpr (kPBF16) mma_16816<kMmaBF16>(acc[dt], af, pl[mt][0], pl[mt][1]);
            }
          }
        }
      }
      __syncwarp();
      ++n_consumed;
      if (!failed && i + kStages < nb_w) issue(i + kStages);
    }

    // ---- merge the warps' partial states through shared memory
    {
      float* scr = reinterpret_cast<float*>(wbase);
      const float lsum0 = shfl_xor_sum(l_run[0]);
      const float lsum1 = shfl_xor_sum(l_run[1]);
#pragma unroll
      for (int dt = 0; dt < C::kDimTiles; ++dt) {
        // C fragment rows: 16-bit path dims 16dt + g (+8); 8-bit path 16dt + 2g (+1)
        const int dlo = (CK == kCacheE4M3) ? dt * 16 + 2 * g : dt * 16 + g;
        const int dhi = (CK == kCacheE4M3) ? dlo + 1 : dlo + 8;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int h = 2 * tig + c;
          scr[h * D + dlo] = acc[dt][c];
          scr[h * D + dhi] = acc[dt][2 + c];
        }
      }
      if (g == 0) {
        scr[kMaxGroup * D + 2 * tig] = m_run[0];
        scr[kMaxGroup * D + 2 * tig + 1] = m_run[1];
        scr[kMaxGroup * D + kMaxGroup + 2 * tig] = lsum0;
        scr[kMaxGroup * D + kMaxGroup + 2 * tig + 1] = lsum1;
      }
    }
    __syncthreads();
    {
      constexpr int kVec = 8;
      const int units = ncols * (D / kVec);
      for (int u = threadIdx.x; u < units; u += kDecodeThreads) {
        const int h = u / (D / kVec);
        const int d0 = (u % (D / kVec)) * kVec;
        float mw[kDecodeWarps];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
          const float* scr = reinterpret_cast<const float*>(ring + w * C::kWarpBytes);
          mw[w] = scr[kMaxGroup * D + h];
          M = fmaxf(M, mw[w]);
        }
        float o[kVec];
#pragma unroll
        for (int v = 0; v < kVec; ++v) o[v] = 0.f;
        float L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kDecodeWarps; ++w) {
            const float* scr = reinterpret_cast<const float*>(ring + w * C::kWarpBytes);
            const float f = fast_exp2(mw[w] - M);
            L += f * scr[kMaxGroup * D + kMaxGroup + h];
            const float4 x0 = *reinterpret_cast<const float4*>(scr + h * D + d0);
            const float4 x1 = *reinterpret_cast<const float4*>(scr + h * D + d0 + 4);
            o[0] += f * x0.x; o[1] += f * x0.y; o[2] += f * x0.z; o[3] += f * x0.w;
            o[4] += f * x1.x; o[5] += f * x1.y; o[6] += f * x1.z; o[7] += f * x1.w;
          }
          const float inv = a.out_scale / L;
#pragma unroll
          for (int v = 0; v < kVec; ++v) o[v] *= inv;
        }
        const int64_t qh = static_cast<int64_t>(seq) * a.hq + h0 + h;
        if (nsplit == 1) {
          uint4 pk;
          pk.x = static_cast<uint32_t>(from_float<kQBF16>(o[0])) | (static_cast<uint32_t>(from_float<kQBF16>(o[1])) << 16);
          pk.y = static_cast<uint32_t>(from_float<kQBF16>(o[2])) | (static_cast<uint32_t>(from_float<kQBF16>(o[3])) << 16);
          pk.z = static_cast<uint32_t>(from_float<kQBF16>(o[4])) | (static_cast<uint32_t>(from_float<kQBF16>(o[5])) << 16);
          pk.w = static_cast<uint32_t>(from_float<kQBF16>(o[6])) | (static_cast<uint32_t>(from_float<kQBF16>(o[7])) << 16);
          *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.out) + qh * D + d0) = pk;
        } else {
          const int64_t pi = static_cast<int64_t>(a.seq_off[seq] + split) * a.hq + h0 + h;
          float* op = a.o_part + pi * D + d0;
          *reinterpret_cast<float4*>(op) = make_float4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<float4*>(op + 4) = make_float4(o[4], o[5], o[6], o[7]);
          if (d0 == 0) a.lse_part[pi] = (M == -INFINITY) ? -INFINITY : M + log2f(L);
        }
      }
    }
    if (nsplit > 1) {
      // The CTA that finishes the last range of this (sequence, kv head)
      // merges all its ranges: out = sum_i w_i o_i / sum_i w_i with
      // w_i = 2^(lse_i - max lse).  Partials are published with a fence
      // before the arrival count and read after it through L2.
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        const int prev = atomicAdd(&a.arrived[(seq * a.hkv + kvh) * a.ncg + cg], 1);
        s_flag = (prev == nsplit - 1) ? 1 : 0;
      }
      __syncthreads();
      if (s_flag) {
        __threadfence();
        // (1) every range's lse of every head into shared memory (the ring is
        // free: the warps' scratch was consumed above), (2) per head the max
        // and the weights w_i = 2^(lse_i - max), (3) the weighted sum of the
        // partial outputs, four ranges' loads at a time
        float* lse_s = reinterpret_cast<float*>(ring);           // [nsplit][group]
        float* wsum_s = lse_s + nsplit * ncols;                  // [ncols]
        const int64_t base = static_cast<int64_t>(a.seq_off[seq]) * a.hq + h0;
        const int npairs = nsplit * ncols;
        for (int k = threadIdx.x; k < npairs; k += kDecodeThreads) {
          const int i = k / ncols, h = k % ncols;
          lse_s[k] = __ldcg(a.lse_part + base + static_cast<int64_t>(i) * a.hq + h);
        }
        __syncthreads();
        for (int h = warp; h < ncols; h += kDecodeWarps) {
          float M = -INFINITY;
          for (int i = lane; i < nsplit; i += 32) M = fmaxf(M, lse_s[i * ncols + h]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
          float W = 0.f;
          for (int i = lane; i < nsplit; i += 32) {
            const float w = (M == -INFINITY) ? 0.f : fast_exp2(lse_s[i * ncols + h] - M);
            lse_s[i * ncols + h] = w;  // now the weight
            W += w;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
          if (lane == 0) wsum_s[h] = W;
        }
        __syncthreads();
        constexpr int kVec = 4;
        const int units = ncols * (D / kVec);
        for (int u = threadIdx.x; u < units; u += kDecodeThreads) {
          const int h = u / (D / kVec);
          const int d0 = (u % (D / kVec)) * kVec;
          float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
          const float* op = a.o_part + (base + h) * D + d0;
          // four ranges per pass, their loads issued together
          for (int i0 = 0; i0 < nsplit; i0 += 4) {
            float w[4];
            float4 x[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const bool in = i0 + k < nsplit;
              w[k] = in ? lse_s[(i0 + k) * ncols + h] : 0.f;
              x[k] = in ? __ldcg(reinterpret_cast<const float4*>(op + static_cast<int64_t>(i0 + k) * a.hq * D))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              o0 += w[k] * x[k].x; o1 += w[k] * x[k].y; o2 += w[k] * x[k].z; o3 += w[k] * x[k].w;
            }
          }
          const float W = wsum_s[h];
          const float inv = W > 0.f ? 1.f / W : 0.f;
          uint2 pk;
          pk.x = static_cast<uint32_t>(from_float<kQBF16>(o0 * inv)) | (static_cast<uint32_t>(from_float<kQBF16>(o1 * inv)) << 16);
          pk.y = static_cast<uint32_t>(from_float<kQBF16>(o2 * inv)) | (static_cast<uint32_t>(from_float<kQBF16>(o3 * inv)) << 16);
          *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.out) +
                                    (static_cast<int64_t>(seq) * a.hq + h0 + h) * D + d0) = pk;
        }
      }
    }
    // the next item is taken only now, when this CTA can start it at once,
    // so no CTA holds an item it cannot start while others run dry
    if (threadIdx.x == 0) fetch_next(false);
    __syncthreads();           // scratch (= stage memory) is free again ...
    fence_proxy_async_smem();  // ... and the next item's tile loads come after these accesses
  }

  // drain copies still in flight after a timeout (bounded again)
  if (failed) {
    while (n_consumed < n_issued) {
      const int st = n_consumed % kStages;
      mbar_wait_bounded(bar0 + 8 * st, (n_consumed / kStages) & 1u);
      ++n_consumed;
    }
  }
}

}  // namespace pa
