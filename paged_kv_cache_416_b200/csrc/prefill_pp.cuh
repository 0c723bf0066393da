// Paged prefill (chunked-prefill) attention, two query tiles per CTA whose
// softmax and tensor-core products alternate ("ping-pong"), sm_100a.
//
// Method as in prefill.cuh: the new query tokens of a sequence attend
// causally to its cached keys and values, gathered block by block through
// the block table ("PagedAttention", Ultralytics glossary, section
// "Sayfalama Nasil Calisir"), FlashAttention style, tiled with an online
// softmax (section "Ilgili Teknikler", Flash Attention bullet), the G query
// heads of a kv head packed into the rows of a tile (grouped-query attention
// bullet).  Both products run on tcgen05.mma with accumulators in TMEM.
//
//   CTA   = 10 warps on one (sequence, kv head, 2 x 128 query rows) unit, one
//           CTA per SM.  Tile A holds the unit's first T = 128 / G tokens,
//           tile B the next T (row r of a tile = (token r / G, head r % G),
//           TMEM lane r).  Warps 0-3 run tile A's softmax, warps 4-7 tile B's
//           (thread r of a group owns row r); warp 8 issues the MMAs (one
//           lane) and zeroes values that must not reach O; warp 9 issues the
//           TMA loads.  Every hand-over is an mbarrier.
//   TMEM  = O_A [0, D) | O_B [D, 2D) | S/P_A 64 columns | S/P_B 64 columns:
//           S_X(kt) fp32, then P_X(kt) over it (P_hi in its first 32 columns,
//           P_lo in the next 32, two 16-bit values per column)
//   per 64-key tile kt, both tiles read the same K(kt) and V(kt) stages (three
//   of each, one TMA box per (block, dim half)); the MMA warp issues
//       S_A(0) S_B(0) | PV_A(0) S_A(1) | PV_B(0) S_B(1) | PV_A(1) S_A(2) | ...
//   each PV_X(kt) = (P_hi + P_lo)(kt) V(kt) as soon as tile X's rows have
//   written P_X(kt), so the softmax of one tile runs while the tensor cores
//   work on the other.  tcgen05 operations of one thread complete in issue
//   order, so S_X(kt+1), issued right after PV_X(kt), overwrites P_X(kt) only
//   once PV_X(kt) has read it, and the commit that reports S_X(kt+1) done also
//   reports O_X(kt) done: the rows may rescale O_X before they release P_X.
//   O_X is rescaled only when a row's running max grows by more than 8 in
//   log2 units (the weights otherwise keep the stale max, below 2^8).
//
// Every shared-memory operand tile uses the 128-byte swizzle, rows of 128
// bytes, 8-row groups 1024 bytes apart.  Every wait is bounded.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode.cuh"   // tma_load_5d, prefetch_tensormap
#include "prefill.cuh"  // PrefillArgs, swz128, kPfRows, kPfKeys, kPfRescaleLog2
#include "tcgen05.cuh"

namespace pa {

constexpr int kPpRowWarps = 8;                    // 4 per query tile
constexpr int kPpThreads = (kPpRowWarps + 2) * 32;  // + MMA warp + load warp
constexpr int kPpStages = 3;                      // K and V stages each

template <int BS, int D>
struct PrefillPpCfg {
  static constexpr int kHalves = D / 64;                   // 128-byte dim halves of a row
  static constexpr int kQBytes = kPfRows * D * 2;          // one tile: [halves][128 rows][128 B]
  static constexpr int kKBytes = kPfKeys * D * 2;          // [halves][64 keys][128 B]
  static constexpr int kBlocksPerTile = kPfKeys / BS;
  static constexpr int kOffQ = 0;                          // Q_A, Q_B
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kPpStages * kKBytes;
  static constexpr int kTiles = kOffV + kPpStages * kKBytes;  // 160 KiB at D 128
  static constexpr int kHead = 512;                        // mbarriers, TMEM slot, block ids
  static constexpr int kSmemBytes = kTiles + kHead;
  static constexpr uint32_t kColO = 0;                     // O_A; O_B at D
  static constexpr uint32_t kColS = 2 * D;                 // S/P_A; S/P_B 64 further
  // TMEM columns: a power of two >= 2D + 2 * 64 (512 at D 128, 256 at D 64)
  static constexpr uint32_t kTmemCols = (2 * D + 2 * kPfKeys) <= 256 ? 256 : 512;
  static_assert(kPfKeys % BS == 0, "a key tile holds whole blocks");
  static_assert(2 * D + 2 * kPfKeys <= kTmemCols, "TMEM columns");
  static_assert(144 + 8 * kBlocksPerTile * 4 <= kHead, "block-id ring fits the header");
};

// One CTA per (unit of 2T query tokens, kv head, sequence): grid
// (ceil(max_query_len / 2T), Hkv, B); CTAs past a sequence's new tokens exit.
template <bool kBF16, int BS, int D>
__global__ void __launch_bounds__(kPpThreads, 1)
prefill_pp_kernel(const __grid_constant__ PrefillArgs a) {
  using C = PrefillPpCfg<BS, D>;
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  extern __shared__ __align__(1024) uint8_t pp_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool row_warp = warp < kPpRowWarps;
  const bool mma_warp = warp == kPpRowWarps;
  const int s = blockIdx.z, kvh = blockIdx.y;
  const int G = a.group;
  const int T = kPfRows / G;  // query tokens per tile
  const int q0 = a.query_start[s];
  const int n = a.query_start[s + 1] - q0;
  const int i0 = blockIdx.x * 2 * T;
  if (n <= 0 || i0 >= n) return;  // the whole CTA, before any TMEM use
  const int nt = min(2 * T, n - i0);
  const int X = (warp >> 2) & 1;              // a row thread's tile (A = 0, B = 1)
  const int r = (warp & 3) * 32 + lane;       // its row in the tile (TMEM lane)
  const int tok = X * T + r / G;              // its token within the unit
  const int hr = kvh * G + r % G;             // its query head
  const bool row_ok = row_warp && r / G < T && tok < nt;
  const int ctx = a.context_lens[s];
  const int64_t orow_off = (static_cast<int64_t>(q0 + i0 + tok) * a.hq + hr) * (D * 2 / 16);
  if (ctx < n || ctx > a.max_ctx || ctx > a.max_blocks * BS) {
    if (tid == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    if (row_ok)
      for (int j = 0; j < D * 2 / 16; ++j)
        reinterpret_cast<uint4*>(a.out)[orow_off + j] = make_uint4(0, 0, 0, 0);
    return;
  }
  const int qfirst = ctx - n + i0;  // position of the unit's first token
  const int qpos = qfirst + tok;    // this row's position
  const int kend = qfirst + nt;     // keys the unit's rows see: [0, kend)
  const int nkt = (kend - 1) / kPfKeys + 1;
  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks;

  // [tiles (1024-aligned) | mbarriers | TMEM slot | block ids of 8 key tiles]
  const uint32_t base_s = smem_addr(pp_smem);
  uint8_t* const base = pp_smem;
  const uint32_t head_s = base_s + C::kTiles;
  const uint32_t full_k = head_s, full_v = head_s + 24;    // + 8 * stage: TMA
  const uint32_t k_empty = head_s + 48, v_empty = head_s + 72;  // + 8 * stage: MMA commits
  const uint32_t bar_s = head_s + 96;     // + 8 * tile: S_X (and O_X before it) done
  const uint32_t p_ready = head_s + 112;  // + 8 * tile: one arrival per row warp of the tile
  const uint32_t bar_done = head_s + 128;  // the last products done
  const uint32_t tmem_slot_s = head_s + 136;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(base + C::kTiles + 136);
  // the loader's block ids of key tile kt (K issue writes, V issue reads):
  // K runs at most a few tiles ahead of V, well inside the 8 entries
  int* const s_phys = reinterpret_cast<int*>(base + C::kTiles + 144);  // [8][kBlocksPerTile]
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
  // loader lane 0: TMA loads of one K or V tile into its stage (one box per
  // block and dim half); blocks past the context or with a bad entry
  // (phys < 0) are not loaded
  auto issue_tile = [&](int kt, bool is_v, const int* phys) {
    const int st = kt % kPpStages;
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
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf)
        tma_load_5d(dst + hf * (kPfKeys * 128) + b * BS * 128, map, 0, 0, hf, kvh, phys[b], bar);
    }
  };

  const bool loader = warp == kPpRowWarps + 1;
  if (loader && lane == 0) {
    for (int i = 0; i < 2 * kPpStages; ++i) mbar_init(full_k + 8 * i, 1);       // full_k, full_v
    for (int i = 0; i < 2 * kPpStages; ++i) mbar_init(k_empty + 8 * i, 1);      // k/v_empty
    mbar_init(bar_s, 1);
    mbar_init(bar_s + 8, 1);
    mbar_init(p_ready, kPpRowWarps / 2);
    mbar_init(p_ready + 8, kPpRowWarps / 2);
    mbar_init(bar_done, 1);
    mbar_init_fence();
    prefetch_tensormap(&a.tmap_k);
    prefetch_tensormap(&a.tmap_v);
    for (int kt = 0; kt < kPpStages && kt < nkt; ++kt) {
      int phys[C::kBlocksPerTile];
#pragma unroll
      for (int b = 0; b < C::kBlocksPerTile; ++b) {
        phys[b] = tile_block(kt, b);
        s_phys[(kt & 7) * C::kBlocksPerTile + b] = phys[b];
      }
      issue_tile(kt, false, phys);
      issue_tile(kt, true, phys);
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot_s, C::kTmemCols);
    tmem_relinquish();
  }
  if (row_warp) {  // Q tiles: thread r of tile X writes its row into the dim halves
    const uint4* src = reinterpret_cast<const uint4*>(a.q) + orow_off;
    const int qoff = C::kOffQ + X * C::kQBytes;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      const uint4 v = row_ok ? src[j] : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(base + qoff + (j >> 3) * (kPfRows * 128) + swz128(r, j & 7)) = v;
    }
    fence_proxy_async_smem();
  }
  // any bad table entry among the blocks this unit reads?  (then every tile
  // takes the masked path; otherwise only the tiles that cross the diagonal
  // or the end of the context)
  int my_bad = 0;
  for (int j = tid; j * BS < kend; j += kPpThreads) {
    const int p = table[j];
    my_bad |= (p < 0 || p >= a.num_blocks);
  }
  tc_fence_before_sync();
  const bool any_bad = __syncthreads_or(my_bad) != 0;  // + Q tiles, barriers, TMEM address
  tc_fence_after_sync();
  if (any_bad && tid == 0) record_error(PA_ERR_DEVICE_BOUNDS);
  const uint32_t tmem = *tmem_slot;
  auto tO = [&](int x) { return tmem + C::kColO + static_cast<uint32_t>(x * D); };
  auto tS = [&](int x) { return tmem + C::kColS + static_cast<uint32_t>(x * kPfKeys); };
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
    auto issue_s = [&](int x, int kt) {  // S_X(kt) = Q_X K(kt)^T
      wait(full_k + 8 * (kt % kPpStages), (kt / kPpStages) & 1);
      if (failed || lane != 0) return;
      tc_fence_after_sync();
      const uint32_t k_st = sK + (kt % kPpStages) * C::kKBytes;
      const uint32_t q_t = sQ + x * C::kQBytes;
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        umma_f16(tS(x), umma_desc_k128(q_t + (k >> 2) * (kPfRows * 128) + (k & 3) * 32),
                 umma_desc_k128(k_st + (k >> 2) * (kPfKeys * 128) + (k & 3) * 32), kIdescS,
                 k > 0 ? 1u : 0u);
      umma_commit(bar_s + 8 * x);
    };
    auto issue_pv = [&](int x, int kt) {  // O_X += (P_hi + P_lo)_X(kt) V(kt)
      if (failed || lane != 0) return;
      tc_fence_after_sync();
      const uint32_t v_st = sV + (kt % kPpStages) * C::kKBytes;
      const uint32_t tP = tS(x);
#pragma unroll
      for (int k = 0; k < kPfKeys / 16; ++k)
        umma_f16_ts(tO(x), tP + 8 * k, umma_desc_mn128(v_st + k * 2048, kPfKeys * 128), kIdescO,
                    (kt > 0 || k > 0) ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < kPfKeys / 16; ++k)
        umma_f16_ts(tO(x), tP + 32 + 8 * k, umma_desc_mn128(v_st + k * 2048, kPfKeys * 128),
                    kIdescO, 1u);
    };
    issue_s(0, 0);
    issue_s(1, 0);
    if (lane == 0 && !failed) umma_commit(k_empty);
    for (int kt = 0; kt < nkt; ++kt) {
      const int st = kt % kPpStages;
      wait(p_ready, kt & 1);  // P_A(kt) in TMEM
      wait(full_v + 8 * st, (kt / kPpStages) & 1);
      // values of keys past the context or in bad blocks may hold anything
      // (0 * NaN would reach O): zero their rows of V(kt), once for both tiles
      const int bad = bad_of(kt);
      if ((kt + 1) * kPfKeys > ctx || bad) {
#pragma unroll
        for (int i = 0; i < 2 * C::kHalves; ++i) {  // (half, key) rows of the stage
          const int row = lane + 32 * i, key = row & (kPfKeys - 1), hf = row >> 6;
          if (kt * kPfKeys + key >= ctx || ((bad >> (key / BS)) & 1)) {
            uint4* dst = reinterpret_cast<uint4*>(base + C::kOffV + st * C::kKBytes +
                                                  hf * (kPfKeys * 128) + key * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      issue_pv(0, kt);
      if (kt + 1 < nkt) issue_s(0, kt + 1);
      __syncwarp();
      wait(p_ready + 8, kt & 1);  // P_B(kt) in TMEM
      issue_pv(1, kt);
      if (lane == 0 && !failed) umma_commit(v_empty + 8 * st);
      if (kt + 1 < nkt) {
        issue_s(1, kt + 1);
        if (lane == 0 && !failed) umma_commit(k_empty + 8 * ((kt + 1) % kPpStages));
      }
      __syncwarp();
    }
    if (lane == 0 && !failed) umma_commit(bar_done);
  } else if (loader) {
    // ======================= load warp (lane 0 issues) ===================
    // K(kt) waits for its stage (S_B(kt-3) done), V(kt) for its own
    // (PV_B(kt-3) done); whichever is ready goes first.  The block ids of
    // the next K tile are read ahead, while the loader waits.
    int nk = min(kPpStages, nkt), nv = min(kPpStages, nkt);  // issued above
    int nphys[C::kBlocksPerTile];
#pragma unroll
    for (int b = 0; b < C::kBlocksPerTile; ++b) nphys[b] = nk < nkt ? tile_block(nk, b) : -1;
    unsigned long long t_idle = global_timer_ns();
    while ((nk < nkt || nv < nkt) && !failed) {
      bool did = false;
      if (nv < nk && nv < nkt) {
        const int ready = __shfl_sync(
            0xffffffffu,
            lane == 0 ? (int)mbar_try_wait(v_empty + 8 * (nv % kPpStages), ((nv / kPpStages) - 1) & 1)
                      : 0,
            0);
        if (ready) {
          if (lane == 0) issue_tile(nv, true, s_phys + (nv & 7) * C::kBlocksPerTile);
          ++nv;
          did = true;
        }
      }
      if (nk < nkt) {
        const int ready = __shfl_sync(
            0xffffffffu,
            lane == 0 ? (int)mbar_try_wait(k_empty + 8 * (nk % kPpStages), ((nk / kPpStages) - 1) & 1)
                      : 0,
            0);
        if (ready) {
          if (lane == 0) {
#pragma unroll
            for (int b = 0; b < C::kBlocksPerTile; ++b)
              s_phys[(nk & 7) * C::kBlocksPerTile + b] = nphys[b];
            issue_tile(nk, false, nphys);
          }
          ++nk;
#pragma unroll
          for (int b = 0; b < C::kBlocksPerTile; ++b) nphys[b] = nk < nkt ? tile_block(nk, b) : -1;
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
    // ======================= row warps of tile X ========================
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;  // TMEM lanes
    const uint64_t sl2x2 = f2(a.sl2, a.sl2);
    const int qfirst_x = qfirst + X * T;  // the tile's first row position
    float m_run = -INFINITY;  // running max of the raw scores
    float l_run = 0.f;        // sum of weights, relative to m_run
    for (int kt = 0; kt < nkt; ++kt) {
      wait(bar_s + 8 * X, kt & 1);  // S_X(kt) done, and O_X(kt-1) before it
      tc_fence_after_sync();
      uint32_t sv[kPfKeys];
      const uint32_t tb = tS(X) + lane_off;
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        tmem_ld32(tb, lo);
        tmem_ld32(tb + 32, hi);
      }
      tmem_wait_ld();
      float x[kPfKeys];
#pragma unroll
      for (int c = 0; c < kPfKeys; ++c) x[c] = __uint_as_float(sv[c]);
      // keys past the diagonal, the context, or in a bad block get -inf;
      // tiles wholly below the tile's first row need no mask
      const bool masked = any_bad || kt * kPfKeys + kPfKeys - 1 > qfirst_x;
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
      // P = P_hi + P_lo, both in the operands' 16-bit type (P_hi alone errs
      // by up to 2^-9 of each bf16 weight, which outputs formed by
      // cancellation cannot absorb)
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
        uint64_t hf;
        if constexpr (kBF16) hf = f2(__uint_as_float(h << 16), __uint_as_float(h & 0xffff0000u));
        else hf = f2(to_float<false>(h & 0xffff), to_float<false>(h >> 16));
        const float2 d = f2_split(f2_sub(pp, hf));
        pl[c / 2] = pack2<kBF16>(d.x, d.y);
      }
      const float2 ss = f2_split(sum2);
      l_run = l_run * alpha + (ss.x + ss.y);
      // O_X(kt-1) is done (it completed before S_X(kt)) and PV_X(kt) waits
      // for these rows: rescale O_X in place when a row needs it
      if (kt > 0 && __any_sync(0xffffffffu, resc)) {
        const uint64_t al2 = f2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ot[32];
          tmem_ld32(tO(X) + lane_off + 32 * c, ot);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 v = f2_split(
                f2_mul(f2(__uint_as_float(ot[j]), __uint_as_float(ot[j + 1])), al2));
            ot[j] = __float_as_uint(v.x);
            ot[j + 1] = __float_as_uint(v.y);
          }
          tmem_st32(tO(X) + lane_off + 32 * c, ot);
        }
      }
      // P_X(kt) over S_X(kt) in its columns
      tmem_st32(tb, ph);
      tmem_st32(tb + 32, pl);
      tmem_wait_st();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_ready + 8 * X);
    }

    // ---- epilogue: O / l for this thread's row
    wait(bar_done, 0);
    tc_fence_after_sync();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    uint4* const orow = reinterpret_cast<uint4*>(a.out) + orow_off;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ot[32];
      tmem_ld32(tO(X) + lane_off + 32 * c, ot);
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
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace pa
