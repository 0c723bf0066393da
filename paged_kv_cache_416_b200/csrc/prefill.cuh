// Paged prefill (chunked-prefill) attention on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory), sm_100a.
//
// Method: the new query tokens of a sequence attend causally to its cached
// keys and values, gathered block by block through the block table
// ("PagedAttention", Ultralytics glossary, section "Sayfalama Nasil Calisir"),
// FlashAttention style: tiled, with an online softmax, so the score matrix
// never reaches memory (section "Ilgili Teknikler", Flash Attention bullet);
// the G query heads of a kv head are packed into the rows of one tile
// (grouped-query attention bullet).  Unlike single-query decode this is a
// dense contraction (128 query rows x 64 keys x 128 dims per tile pair), so
// both products run on tcgen05.mma:
//
//   CTA   = 6 warps on one (sequence, kv head, 128 query rows) tile, two
//           CTAs per SM.  Warps 0-3 own the rows: query row r = (token r / G,
//           head r % G) lives in TMEM lane r and thread r runs its softmax.
//           Warp 4 issues the MMAs (one lane) and zeroes values that must not
//           reach O; warp 5 issues the TMA loads.  They hand over through
//           mbarriers only (S done and O done, four of each, which also
//           free K and V stages; S read, P ready; K / V full per stage),
//           never a CTA-wide barrier inside the key loop.
//   TMEM  = S [0, 64) | P [64, 128) | O [128, 128 + D): S(kt) in fp32; P(kt)
//           with P_hi in the first 32 columns of P, P_lo (bf16 caches) in
//           the next 32, two 16-bit values per column.  S and P have
//           buffers of their own, so S(kt+1) waits only for the rows to have
//           read S(kt), never for O(kt-1): the MMA queue need not drain
//           between the products of consecutive tiles (the rows write P(kt)
//           once O(kt-1), the P buffer's last reader, is done)
//   per 64-key tile kt (K and V by TMA into two stages each, K one box per
//   (block, dim half), V one box per block; K(kt+2) is loaded once S(kt) is
//   done, V(kt+2) once O(kt) is done; the load warp reads the block ids 32 at
//   a time, a chunk ahead, and polls the stages without sleeping on either):
//     S            = Q K^T      tcgen05.mma, A = Q and B = K from shared memory
//                               (K-major), M128 N64, D/16 x K16; S(kt+1) is
//                               issued once the rows have read S(kt), so it
//                               runs under the softmax of tile kt
//     softmax      thread r: tcgen05.ld of its S row, causal and block masks
//                  (only on tiles that need them), online max / sum in packed
//                  fp32 pairs; with a bf16 cache P = P_hi + P_lo (two bf16
//                  parts, so P keeps ~16 significant bits), with fp16 one
//                  fp16 part, by tcgen05.st into TMEM
//     O           += P V        tcgen05.mma, A = P from TMEM, B = V from shared
//                               memory read MN-major (no transpose), M128 N=D,
//                               2 x 4 x K16, accumulated in TMEM across tiles
//   O is rescaled (tcgen05.ld, multiply, tcgen05.st) only when a row's
//   running max grows by more than 8 in log2 units; otherwise the weights
//   keep the stale max (they stay below 2^8) and the sum follows it, so the
//   normalised result is the same.
//
// Every shared-memory operand tile uses the 128-byte swizzle, rows of 128
// bytes, 8-row groups 1024 bytes apart.  Every wait is bounded.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode.cuh"  // tma_load_5d, prefetch_tensormap, pair helpers
#include "tcgen05.cuh"

namespace pa {

constexpr int kPfRowThreads = 128;  // warps 0-3: thread r owns query row r (TMEM lane r)
constexpr int kPfThreads = 192;     // + warp 4: MMA issue, warp 5: TMA loads
constexpr int kPfRows = 128;      // MMA M: (token, head) rows per CTA
constexpr int kPfKeys = 64;       // keys per tile
constexpr int kPfMaxD = 128;      // head_dim 64 or 128: one or two 64-dim (128-byte) halves
constexpr int kPfTmemCols = 256;  // S [0, 64), P [64, 128), O [128, 256)
constexpr float kPfRescaleLog2 = 8.f;  // rescale O when the max grows by more than this

template <int BS, int D>
struct PrefillCfg {
  static constexpr int kHalves = D / 64;                  // 128-byte dim halves of a row
  static constexpr int kQBytes = kPfRows * D * 2;         // [halves][128 rows][128 B]
  static constexpr int kKBytes = kPfKeys * D * 2;         // K: [halves][64 keys][128 B]
  static constexpr int kBlocksPerTile = kPfKeys / BS;
  static constexpr int kVBlockBytes = kHalves * BS * 128; // V: [blocks][halves][bs keys][128 B]
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;           // 2 stages
  static constexpr int kOffV = kOffK + 2 * kKBytes;       // 2 stages
  static constexpr int kTiles = kOffV + 2 * kKBytes;      // 96 KiB at D 128: two CTAs per SM
  static constexpr int kHead = 256;                       // 15 mbarriers, TMEM slot, block ids
  static constexpr int kSmemBytes = kTiles + kHead;
  static_assert(kPfKeys % BS == 0, "a key tile holds whole blocks");
};

struct PrefillArgs {
  // Pools viewed as 5-D bytes (x, token, half, kv head, block) =
  // (128, bs, D / 64, Hkv, N); a K box (128, bs, 1, 1, 1) is one dim half of
  // one block, a V box (128, bs, D / 64, 1, 1) the whole block
  CUtensorMap tmap_k;
  CUtensorMap tmap_v;
  void* out;                   // [total_q, Hq, D], q's dtype
  const void* q;               // [total_q, Hq, D]
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* query_start;  // [B + 1]
  int hq, hkv, group, max_blocks, num_blocks, max_ctx;
  float sl2;                   // scale * log2(e)
};

// Offset of 16-byte chunk `c` of row `r` in a 128B-swizzled tile of 128-byte rows.
__device__ __forceinline__ uint32_t swz128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

// One CTA per (query tile, kv head, sequence): grid (ceil(max_query_len / T),
// Hkv, B) with T = 128 / G tokens; CTAs past a sequence's new tokens exit.
// Blocks start in index order, x fastest, and block x takes query tile
// gridDim.x - 1 - x: within a (sequence, kv head) the tiles with the most
// keys under the causal mask start first, so the grid ends on short tiles
// (the tiles of one pair still run side by side and share its K / V in L2).
template <bool kBF16, int BS, int D>
__global__ void __launch_bounds__(kPfThreads, 2) prefill_kernel(const __grid_constant__ PrefillArgs a) {
  using C = PrefillCfg<BS, D>;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  extern __shared__ __align__(1024) uint8_t pf_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp >= kPfRowThreads / 32;     // warps 4 (MMA) and 5 (loads)
  const bool mma_warp = warp == kPfRowThreads / 32;
  const int s = blockIdx.z, kvh = blockIdx.y;
  const int G = a.group;
  const int T = kPfRows / G;  // query tokens per CTA
  const int q0 = a.query_start[s];
  const int n = a.query_start[s + 1] - q0;
  const int i0 = static_cast<int>(gridDim.x - 1 - blockIdx.x) * T;
  if (n <= 0 || i0 >= n) return;  // the whole CTA, before any TMEM use
  const int nt = min(T, n - i0);
  const int r = tid;                          // row of a row thread
  const int tok = r / G;
  const int hr = kvh * G + r % G;             // its query head
  const bool row_ok = !producer && tok < nt;
  const int ctx = a.context_lens[s];
  const int64_t orow_off = (static_cast<int64_t>(q0 + i0 + tok) * a.hq + hr) * (D * 2 / 16);
  if (ctx < n || ctx > a.max_ctx || ctx > a.max_blocks * BS) {
    if (tid == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    if (row_ok)
      for (int j = 0; j < D * 2 / 16; ++j)
        reinterpret_cast<uint4*>(a.out)[orow_off + j] = make_uint4(0, 0, 0, 0);
    return;
  }
  const int qfirst = ctx - n + i0;            // position of the CTA's first token
  const int qpos = qfirst + tok;              // this row's position
  const int kend = qfirst + nt;               // keys the CTA's rows see: [0, kend)
  const int nkt = (kend - 1) / kPfKeys + 1;
  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks;

  // [tiles (1024-aligned) | mbarriers | TMEM slot | block ids of 4 key tiles]
  const uint32_t base_s = smem_addr(pf_smem);
  uint8_t* const base = pf_smem;
  const uint32_t head_s = base_s + C::kTiles;
  const uint32_t full_k = head_s, full_v = head_s + 16;  // + 8 * stage, TMA
  // S(kt) done and O(kt) done: MMA commits to one of four barriers each, kt & 3,
  // waited with parity (kt >> 2) & 1.  The row warps wait on them, and so
  // does the load warp before it refills a stage (K(kt+2) after S(kt),
  // V(kt+2) after O(kt)): a barrier cannot run a phase ahead of the loader,
  // since its next phase, S(kt+4) or O(kt+4), needs the tile the loader has
  // yet to load, so no separate "stage empty" commits are needed
  const uint32_t bar_s = head_s + 32, bar_o = head_s + 64;  // + 8 * (kt & 3)
  const uint32_t s_free = head_s + 96, p_ready = head_s + 104;  // one arrival per row warp
  const uint32_t bar_done = head_s + 112;                        // the last O product
  const uint32_t tmem_slot_s = head_s + 120;  // tcgen05.alloc writes the TMEM address here
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(base + C::kTiles + 120);
  // the loader's block ids of key tile kt (K issue writes, V issue reads)
  int* const s_phys = reinterpret_cast<int*>(base + C::kTiles + 128);  // [4][kBlocksPerTile]
  const uint32_t sQ = base_s + C::kOffQ, sK = base_s + C::kOffK, sV = base_s + C::kOffV;
  if (base_s & 1023) {  // the swizzled tiles need a 1024-byte aligned start
    if (tid == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    return;
  }

  // physical block of slot b of key tile kt: -1 past the context, -2 for a
  // bad table entry (its keys are masked and its values zeroed)
  auto tile_block = [&](int kt, int b) -> int {
    const int j = kt * C::kBlocksPerTile + b;
    if (j * BS >= ctx) return -1;
    const int p = table[j];
    return (p >= 0 && p < a.num_blocks) ? p : -2;
  };
  // loader lane 0: TMA loads of one K or V tile into its stage (K: one box
  // per block and dim half, so that each half is one K-major tile; V: one
  // box per block, both halves); blocks past the context or with a bad
  // entry (phys < 0) are not loaded
  auto issue_tile = [&](int kt, bool is_v, const int* phys) {
    const int st = kt & 1;
    uint32_t bytes = 0;
#pragma unroll
    for (int b = 0; b < C::kBlocksPerTile; ++b)
      if (phys[b] >= 0) bytes += C::kHalves * BS * 128u;
    const uint32_t bar = (is_v ? full_v : full_k) + 8 * st;
    const uint32_t dst = (is_v ? sV : sK) + st * C::kKBytes;
    const CUtensorMap* map = is_v ? &a.tmap_v : &a.tmap_k;
    mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
    for (int b = 0; b < C::kBlocksPerTile; ++b) {
      if (phys[b] < 0) continue;
      if (is_v) {
        tma_load_5d(dst + b * C::kVBlockBytes, map, 0, 0, 0, kvh, phys[b], bar);
      } else {
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_5d(dst + hf * (kPfKeys * 128) + b * BS * 128, map, 0, 0, hf, kvh, phys[b], bar);
      }
    }
  };

  if (producer && !mma_warp && lane == 0) {
    for (int i = 0; i < 12; ++i) mbar_init(head_s + 8 * i, 1);  // full_k/v[2], bar_s[4], bar_o[4]
    mbar_init(s_free, kPfRowThreads / 32);
    mbar_init(p_ready, kPfRowThreads / 32);
    mbar_init(bar_done, 1);
    mbar_init_fence();
    prefetch_tensormap(&a.tmap_k);
    prefetch_tensormap(&a.tmap_v);
    for (int kt = 0; kt < 2 && kt < nkt; ++kt) {
      int phys[C::kBlocksPerTile];
#pragma unroll
      for (int b = 0; b < C::kBlocksPerTile; ++b) {
        phys[b] = tile_block(kt, b);
        s_phys[(kt & 3) * C::kBlocksPerTile + b] = phys[b];
      }
      issue_tile(kt, false, phys);
      issue_tile(kt, true, phys);
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot_s, kPfTmemCols);
    tmem_relinquish();
  }
  if (!producer) {  // Q tile: thread r writes its row (2 D bytes) into the dim halves
    const uint4* src = reinterpret_cast<const uint4*>(a.q) + orow_off;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const uint4 v = row_ok ? src[j] : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(base + C::kOffQ + (j >> 3) * (kPfRows * 128) + swz128(r, j & 7)) = v;
    }
    fence_proxy_async_smem();
  }
  // any bad table entry among the blocks this CTA loads (every block of its
  // key tiles inside the context, visible to its rows or not)?  (then every
  // tile takes the masked path and the bad blocks' values are zeroed;
  // otherwise only the tiles that cross the diagonal or the end of the
  // context are masked)
  int my_bad = 0;
  for (int j = tid; j * BS < min(nkt * kPfKeys, ctx); j += kPfThreads) {
    const int p = table[j];
    my_bad |= (p < 0 || p >= a.num_blocks);
  }
  tc_fence_before_sync();
  const bool any_bad = __syncthreads_or(my_bad) != 0;  // + Q tile, barriers, TMEM address
  tc_fence_after_sync();
  if (any_bad && tid == 0) record_error(PA_ERR_DEVICE_BOUNDS);
  const uint32_t tmem = *tmem_slot;
  // S(kt) in [0, 64); P(kt) in [64, 128), hi in its first 32 columns, lo in
  // the next 32; O in [128, 256)
  const uint32_t tS = tmem, tP = tmem + 64, tO = tmem + 128;
  bool failed = false;
  auto wait = [&](uint32_t bar, int parity) {
    if (!failed && !mbar_wait_bounded(bar, parity)) {
      failed = true;
      record_error(PA_ERR_TIMEOUT);
    }
  };
  auto bad_of = [&](int kt) {
    int m = 0;
    if (any_bad) {
#pragma unroll
      for (int b = 0; b < C::kBlocksPerTile; ++b) m |= (tile_block(kt, b) == -2) << b;
    }
    return m;
  };

  if (mma_warp) {
    // ======================= MMA warp (lane 0 issues) ====================
    constexpr uint32_t kIdescS = umma_idesc_f16(kPfRows, kPfKeys, kBF16);
    constexpr uint32_t kIdescO = umma_idesc_f16(kPfRows, D, kBF16, /*b_mn_major=*/true);
    auto issue_s = [&](int kt) {  // S(kt) = Q K(kt)^T; then K(kt)'s stage is free
      wait(full_k + 8 * (kt & 1), (kt >> 1) & 1);
      if (failed || lane != 0) return;
      tc_fence_after_sync();
      const uint32_t k_st = sK + (kt & 1) * C::kKBytes;
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        umma_f16(tS, umma_desc_k128(sQ + (k >> 2) * (kPfRows * 128) + (k & 3) * 32),
                 umma_desc_k128(k_st + (k >> 2) * (kPfKeys * 128) + (k & 3) * 32), kIdescS,
                 k > 0 ? 1u : 0u);
      umma_commit(bar_s + 8 * (kt & 3));  // S(kt) done: the rows read it, K(kt)'s stage is free
    };
    issue_s(0);
    for (int kt = 0; kt < nkt; ++kt) {
      const int st = kt & 1;
      if (kt + 1 < nkt) {
        wait(s_free, kt & 1);  // every row has read S(kt): S(kt+1) may overwrite it
        issue_s(kt + 1);
      }
      wait(p_ready, kt & 1);  // P(kt) in TMEM (the rows waited for O(kt-1) to write it)
      wait(full_v + 8 * st, (kt >> 1) & 1);
      // values of keys past the context or in bad blocks may hold anything
      // (0 * NaN would reach O): zero their rows of V(kt)
      const int bad = bad_of(kt);
      if ((kt + 1) * kPfKeys > ctx || bad) {
#pragma unroll
        for (int i = 0; i < 2 * C::kHalves; ++i) {  // (half, key) rows of the stage
          const int row = lane + 32 * i, key = row & (kPfKeys - 1), hf = row >> 6;
          if (kt * kPfKeys + key >= ctx || ((bad >> (key / BS)) & 1)) {
            uint4* dst = reinterpret_cast<uint4*>(base + C::kOffV + st * C::kKBytes +
                                                  (key / BS) * C::kVBlockBytes + hf * (BS * 128) +
                                                  (key % BS) * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0 && !failed) {  // O += (P_hi [+ P_lo]) V(kt): (2 x) 4 MMAs of K = 16
        tc_fence_after_sync();
        const uint32_t v_st = sV + st * C::kKBytes;
        // keys 16k .. 16k+15 lie in one block: rows of 128 bytes from
        // v_koff(k), the next dim half bs * 128 bytes further
        auto v_koff = [&](int k) {
          return static_cast<uint32_t>((k * 16 / BS) * C::kVBlockBytes + (k * 16 % BS) * 128);
        };
#pragma unroll
        for (int k = 0; k < kPfKeys / 16; ++k)
          umma_f16_ts(tO, tP + 8 * k, umma_desc_mn128(v_st + v_koff(k), BS * 128), kIdescO,
                      (kt > 0 || k > 0) ? 1u : 0u);
        if constexpr (kBF16) {
#pragma unroll
          for (int k = 0; k < kPfKeys / 16; ++k)
            umma_f16_ts(tO, tP + 32 + 8 * k, umma_desc_mn128(v_st + v_koff(k), BS * 128), kIdescO,
                        1u);
        }
        umma_commit(bar_o + 8 * (kt & 3));  // O(kt) done: P and V(kt)'s stage are free
      }
      __syncwarp();
    }
    if (lane == 0 && !failed) umma_commit(bar_done);
  } else if (producer) {
    // ======================= load warp (lane 0 issues) ===================
    // K(kt) waits for its stage (S(kt-2) done), V(kt) for its own (O(kt-2)
    // done); whichever is ready goes first.  The block ids of the next K
    // tile are read ahead, while the loader waits.
    int nk = min(2, nkt), nv = min(2, nkt);  // tiles 0 and 1 went out above
    // block ids in chunks of 32 (lane i holds entry 32 c + i of the table,
    // or -1 past the context), the next chunk loaded while the current one
    // is used, so no table read stands between two tile loads
    auto fetch_ids = [&](int c) {
      const int j = c * 32 + lane;
      int p = -1;
      if (j * BS < ctx) p = table[j];
      return p;
    };
    int tab_c = (nk * C::kBlocksPerTile) >> 5;
    int tab_cur = fetch_ids(tab_c), tab_nxt = fetch_ids(tab_c + 1);
    unsigned long long t_idle = global_timer_ns();
    while ((nk < nkt || nv < nkt) && !failed) {
      bool did = false;
      if (nv < nk && nv < nkt) {
        const int ready = __shfl_sync(
            0xffffffffu, lane == 0 ? (int)mbar_test_wait(bar_o + 8 * ((nv - 2) & 3), ((nv - 2) >> 2) & 1) : 0, 0);
        if (ready) {
          if (lane == 0) issue_tile(nv, true, s_phys + (nv & 3) * C::kBlocksPerTile);
          ++nv;
          did = true;
        }
      }
      if (nk < nkt) {
        const int ready = __shfl_sync(
            0xffffffffu, lane == 0 ? (int)mbar_test_wait(bar_s + 8 * ((nk - 2) & 3), ((nk - 2) >> 2) & 1) : 0, 0);
        if (ready) {
          const int j0 = nk * C::kBlocksPerTile;  // a tile never straddles two chunks
          if ((j0 >> 5) != tab_c) {
            ++tab_c;
            tab_cur = tab_nxt;
            tab_nxt = fetch_ids(tab_c + 1);
          }
          int phys[C::kBlocksPerTile];
#pragma unroll
          for (int b = 0; b < C::kBlocksPerTile; ++b) {  // as tile_block(nk, b)
            const int p = __shfl_sync(0xffffffffu, tab_cur, (j0 + b) & 31);
            phys[b] = (j0 + b) * BS >= ctx ? -1 : ((p >= 0 && p < a.num_blocks) ? p : -2);
          }
          if (lane == 0) {
#pragma unroll
            for (int b = 0; b < C::kBlocksPerTile; ++b)
              s_phys[(nk & 3) * C::kBlocksPerTile + b] = phys[b];
            issue_tile(nk, false, phys);
          }
          ++nk;
          did = true;
        }
      }
      const unsigned long long now = global_timer_ns();
      if (did) {
        t_idle = now;
      } else if (now - t_idle > kWaitLimitNs) {
        failed = true;
        if (lane == 0) record_error(PA_ERR_TIMEOUT);
      }
    }
  } else {
    // ======================= row warps ==================================
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;  // the warp's TMEM lanes
    const uint64_t sl2x2 = f2(a.sl2, a.sl2);
    float m_run = -INFINITY;  // running max of the raw scores
    float l_run = 0.f;        // sum of weights, relative to m_run
    for (int kt = 0; kt < nkt; ++kt) {
      wait(bar_s + 8 * (kt & 3), (kt >> 2) & 1);
      tc_fence_after_sync();
      uint32_t sv[kPfKeys];
      const uint32_t tb = tS + lane_off;
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        tmem_ld32(tb, lo);
        tmem_ld32(tb + 32, hi);
      }
      tmem_wait_ld();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      float x[kPfKeys];
#pragma unroll
      for (int c = 0; c < kPfKeys; ++c) x[c] = __uint_as_float(sv[c]);
      // keys past the diagonal, the context, or in a bad block get -inf;
      // tiles wholly below the CTA's first row need no mask
      const bool masked = any_bad || kt * kPfKeys + kPfKeys - 1 > qfirst;
      if (masked) {
        const int bad = bad_of(kt);
        const int lim = row_ok ? qpos - kt * kPfKeys : -1;  // keys c <= lim are visible
#pragma unroll
        for (int c = 0; c < kPfKeys; ++c)
          if (c > lim || ((bad >> (c / BS)) & 1)) x[c] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kPfKeys; c += 2) mx = fmax3(mx, x[c], x[c + 1]);
      const float m_new = fmaxf(m_run, mx);
      // rescale only when the max grew by more than 2^8 (in weight terms);
      // false while the row has seen no key (m_new = -inf)
      const bool resc = (m_new - m_run) * a.sl2 > kPfRescaleLog2;
      float alpha = 1.f;
      if (resc) {
        alpha = m_run == -INFINITY ? 0.f : fast_exp2((m_run - m_new) * a.sl2);
        m_run = m_new;
      }
      const float nm = m_run == -INFINITY ? 0.f : -m_run * a.sl2;
      const uint64_t nm2 = f2(nm, nm);
      // bf16: P = P_hi + P_lo, both bf16: rounding P to one bf16 value alone
      // (8 significant bits) errs by up to 2^-9 of each weight, which outputs
      // formed by cancellation cannot absorb.  fp16 keeps 11 bits: one part
      uint32_t ph[kPfKeys / 2], pl[kPfKeys / 2];
      uint64_t sum2 = f2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < kPfKeys; c += 2) {
        const float2 e = f2_split(f2_fma(f2(x[c], x[c + 1]), sl2x2, nm2));
        const float p0 = fast_exp2(e.x), p1 = fast_exp2(e.y);  // exp2(-inf) = 0
        const uint64_t pp = f2(p0, p1);
        sum2 = f2_add(sum2, pp);
        const uint32_t h = pack2<kBF16>(p0, p1);
        ph[c / 2] = h;
        if constexpr (kBF16) {
          const uint64_t hf = f2(__uint_as_float(h << 16), __uint_as_float(h & 0xffff0000u));
          const float2 d = f2_split(f2_sub(pp, hf));
          pl[c / 2] = pack2<true>(d.x, d.y);
        }
      }
      const float2 ss = f2_split(sum2);
      l_run = l_run * alpha + (ss.x + ss.y);
      // P(kt) takes the P buffer and a rescale touches O: wait for O(kt-1),
      // the last reader of both (O(kt) needs P(kt), so this wait cannot fall
      // two phases behind); by now it has long finished
      if (kt > 0) {
        wait(bar_o + 8 * ((kt - 1) & 3), ((kt - 1) >> 2) & 1);
        tc_fence_after_sync();
      }
      if (kt > 0 && __any_sync(0xffffffffu, resc)) {
        {  // tcgen05.ld / st are warp-wide
          const uint64_t al2 = f2(alpha, alpha);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ot[32];
            tmem_ld32(tO + lane_off + 32 * c, ot);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 v = f2_split(
                  f2_mul(f2(__uint_as_float(ot[j]), __uint_as_float(ot[j + 1])), al2));
              ot[j] = __float_as_uint(v.x);
              ot[j + 1] = __float_as_uint(v.y);
            }
            tmem_st32(tO + lane_off + 32 * c, ot);
          }
        }
      }
      tmem_st32(tP + lane_off, ph);
      if constexpr (kBF16) tmem_st32(tP + lane_off + 32, pl);
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready);
    }

    // ---- epilogue: O / l for this thread's row
    wait(bar_done, 0);
    tc_fence_after_sync();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    uint4* const orow = reinterpret_cast<uint4*>(a.out) + orow_off;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ot[32];
      tmem_ld32(tO + lane_off + 32 * c, ot);
      tmem_wait_ld();
      if (row_ok) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 v;
          v.x = pack2<kBF16>(__uint_as_float(ot[8 * j]) * inv, __uint_as_float(ot[8 * j + 1]) * inv);
          v.y = pack2<kBF16>(__uint_as_float(ot[8 * j + 2]) * inv, __uint_as_float(ot[8 * j + 3]) * inv);
          v.z = pack2<kBF16>(__uint_as_float(ot[8 * j + 4]) * inv, __uint_as_float(ot[8 * j + 5]) * inv);
          v.w = pack2<kBF16>(__uint_as_float(ot[8 * j + 6]) * inv, __uint_as_float(ot[8 * j + 7]) * inv);
          orow[4 * c + j] = failed ? make_uint4(0, 0, 0, 0) : v;
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kPfTmemCols);
  }
}

}  // namespace pa
