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
//   CTA   = 4 warps, one (sequence, kv head, 128 query rows) tile; query row
//           r = (token r / G, head r % G) lives in TMEM lane r and is owned by
//           thread r for the softmax
//   per 64-key tile (K and V by TMA, one box per (block, dim half); the next
//   tile's loads are issued as soon as this tile's K and V are consumed):
//     S[128 x 64]   = Q[128 x 128] K^T          tcgen05.mma M128 N64, K 8 x 16
//     Vt[128 x 64]  = V^T (warps transpose V in shared memory meanwhile)
//     softmax       thread r: tcgen05.ld of its S row, causal mask, online
//                   max / sum, P row -> P_hi + P_lo (two 16-bit tiles,
//                   128B-swizzled) so P keeps ~16 significant bits
//     Otile[128x128]= (P_hi + P_lo) Vt^T        tcgen05.mma M128 N128, K 2 x 4 x 16
//     O (registers) = O * alpha + Otile          tcgen05.ld of the O row
//
// Every operand tile is K-major with the 128-byte swizzle, rows of 128
// bytes, 8-row groups 1024 bytes apart.  Every wait is bounded.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode.cuh"  // tma_load_5d, prefetch_tensormap, pair helpers
#include "tcgen05.cuh"

namespace pa {

constexpr int kPfThreads = 128;   // 4 warps; thread r owns query row r (TMEM lane r)
constexpr int kPfRows = 128;      // MMA M: (token, head) rows per CTA
constexpr int kPfKeys = 64;       // keys per tile
constexpr int kPfD = 128;         // head_dim
constexpr int kPfTmemCols = 256;  // S in [0, 64), O tile in [128, 256)

template <int BS>
struct PrefillCfg {
  static constexpr int kQBytes = kPfRows * kPfD * 2;      // [2 dim halves][128 rows][128 B]
  static constexpr int kKBytes = kPfKeys * kPfD * 2;      // [2 dim halves][64 keys][128 B]
  static constexpr int kVtBytes = kPfD * kPfKeys * 2;     // [128 dims][64 keys = 128 B]
  static constexpr int kPBytes = kPfRows * kPfKeys * 2;   // [128 rows][64 keys = 128 B]
  static constexpr int kBlocksPerTile = kPfKeys / BS;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kKBytes;
  static constexpr int kOffVt = kOffV + kKBytes;
  static constexpr int kOffP = kOffVt + kVtBytes;         // P_hi, then P_lo
  static constexpr int kTiles = kOffP + 2 * kPBytes;      // 112 KiB: two CTAs per SM
  static constexpr int kHead = 256;                       // mbarriers, TMEM slot, mask
  static constexpr int kSmemBytes = kTiles + kHead;
  static_assert(kPfKeys % BS == 0, "a key tile holds whole blocks");
};

struct PrefillArgs {
  // Pools viewed as 5-D bytes (x, token, half, kv head, block) =
  // (128, bs, 2, Hkv, N); box (128, bs, 1, 1, 1): one dim half of one block.
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
template <bool kBF16, int BS>
__global__ void __launch_bounds__(kPfThreads, 2) prefill_kernel(const __grid_constant__ PrefillArgs a) {
  using C = PrefillCfg<BS>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.z, kvh = blockIdx.y;
  const int G = a.group;
  const int T = kPfRows / G;  // query tokens per CTA
  const int q0 = a.query_start[s];
  const int n = a.query_start[s + 1] - q0;
  const int i0 = blockIdx.x * T;
  if (n <= 0 || i0 >= n) return;  // the whole CTA, before any TMEM use
  const int nt = min(T, n - i0);
  const int r = tid;                          // this thread's query row
  const int tok = r / G;
  const int hr = kvh * G + r % G;             // its query head
  const bool row_ok = tok < nt;
  const int ctx = a.context_lens[s];
  uint4* const orow = reinterpret_cast<uint4*>(a.out) +
                      (static_cast<int64_t>(q0 + i0 + tok) * a.hq + hr) * (kPfD * 2 / 16);
  if (ctx < n || ctx > a.max_ctx || ctx > a.max_blocks * BS) {
    if (tid == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    if (row_ok)
      for (int j = 0; j < kPfD * 2 / 16; ++j) orow[j] = make_uint4(0, 0, 0, 0);
    return;
  }
  const int qpos = ctx - n + i0 + tok;        // this row's position in the sequence
  const int nkt = (ctx - n + i0 + nt - 1) / kPfKeys + 1;  // key tiles up to the last row
  const int32_t* table = a.block_tables + static_cast<int64_t>(s) * a.max_blocks;

  // [tiles (1024-aligned) | mbarriers: full, S done, O done | TMEM slot | bad-block mask]
  const uint32_t base_s = smem_addr(smem);
  uint8_t* const base = smem;
  const uint32_t head_s = base_s + C::kTiles;
  const uint32_t full = head_s, bar_s = head_s + 8, bar_o = head_s + 16;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(base + C::kTiles + 32);
  volatile int* bad_mask = reinterpret_cast<volatile int*>(base + C::kTiles + 64);
  const uint32_t sQ = base_s + C::kOffQ, sK = base_s + C::kOffK, sV = base_s + C::kOffV;
  const uint32_t sVt = base_s + C::kOffVt, sP = base_s + C::kOffP;
  if (base_s & 1023) {  // the swizzled tiles need a 1024-byte aligned start
    if (tid == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    return;
  }

  if (tid == 0) {
    mbar_init(full, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init_fence();
    prefetch_tensormap(&a.tmap_k);
    prefetch_tensormap(&a.tmap_v);
  }
  if (warp == 0) {
    tmem_alloc(head_s + 32, kPfTmemCols);
    tmem_relinquish();
  }

  // Q tile: thread r writes its row (256 B) into the two dim halves
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.q) +
                       (static_cast<int64_t>(q0 + i0 + tok) * a.hq + hr) * (kPfD * 2 / 16);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint4 v = row_ok ? src[j] : make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(base + C::kOffQ + (j >> 3) * (kPfRows * 128) + swz128(r, j & 7)) = v;
    }
  }
  fence_proxy_async_smem();

  // thread 0: TMA loads of key tile kt (one box per block and dim half;
  // blocks past the context, or with a bad table entry, are not loaded and
  // their keys are masked)
  auto issue_tile = [&](int kt) {
    int phys[C::kBlocksPerTile];
    int bad = 0;
    uint32_t bytes = 0;
#pragma unroll
    for (int b = 0; b < C::kBlocksPerTile; ++b) {
      const int j = kt * C::kBlocksPerTile + b;
      phys[b] = -1;
      if (j * BS < ctx) {
        const int p = table[j];
        if (p >= 0 && p < a.num_blocks) {
          phys[b] = p;
          bytes += 4u * BS * 128u;  // K and V, two halves each
        } else {
          bad |= 1 << b;
          record_error(PA_ERR_DEVICE_BOUNDS);
        }
      }
    }
    *bad_mask = bad;
    mbar_arrive_expect_tx(full, bytes);
#pragma unroll
    for (int b = 0; b < C::kBlocksPerTile; ++b) {
      if (phys[b] < 0) continue;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const uint32_t off = hf * (kPfKeys * 128) + b * BS * 128;
        tma_load_5d(sK + off, &a.tmap_k, 0, 0, hf, kvh, phys[b], full);
        tma_load_5d(sV + off, &a.tmap_v, 0, 0, hf, kvh, phys[b], full);
      }
    }
  };
  if (tid == 0) issue_tile(0);
  tc_fence_before_sync();
  __syncthreads();  // Q tile, barriers, TMEM address
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;  // the warp's TMEM lanes
  constexpr uint32_t kIdescS = umma_idesc_f16(kPfRows, kPfKeys, kBF16);
  constexpr uint32_t kIdescO = umma_idesc_f16(kPfRows, kPfD, kBF16);

  float o[kPfD];
#pragma unroll
  for (int d = 0; d < kPfD; ++d) o[d] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  bool failed = false;

  for (int kt = 0; kt < nkt; ++kt) {
    if (!failed && !mbar_wait_bounded(full, kt & 1)) {
      failed = true;
      record_error(PA_ERR_TIMEOUT);
    }
    const int bad = *bad_mask;
    // ---- S = Q K^T (one thread issues; 8 MMAs of K = 16 along head_dim)
    if (tid == 0 && !failed) {
      tc_fence_after_sync();
#pragma unroll
      for (int k = 0; k < kPfD / 16; ++k)
        umma_f16(tS, umma_desc_k128(sQ + (k >> 2) * (kPfRows * 128) + (k & 3) * 32),
                 umma_desc_k128(sK + (k >> 2) * (kPfKeys * 128) + (k & 3) * 32), kIdescS,
                 k > 0 ? 1u : 0u);
      umma_commit(bar_s);
    }
    // ---- meanwhile Vt = V^T: 8x8 tiles read with ldmatrix, stored transposed;
    // keys the tile must not use (past the context, bad block) are zeroed
    if (!failed) {
      const int dg = warp * 4 + (lane >> 3);  // 8-dim group this lane addresses
#pragma unroll
      for (int kg = 0; kg < kPfKeys / 8; ++kg) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4(sV + (dg >> 3) * (kPfKeys * 128) + swz128(kg * 8 + (lane & 7), dg & 7), r0, r1, r2,
                r3);
        const int kl = kg * 8 + (lane >> 2);  // the key this thread's fragments hold
        if (kt * kPfKeys + kl >= ctx || ((bad >> (kl / BS)) & 1)) r0 = r1 = r2 = r3 = 0;
        stsm_x4_trans(sVt + swz128(dg * 8 + (lane & 7), kg), r0, r1, r2, r3);
      }
    }
    fence_proxy_async_smem();
    // ---- online softmax of this thread's row
    if (!failed && !mbar_wait_bounded(bar_s, kt & 1)) {
      failed = true;
      record_error(PA_ERR_TIMEOUT);
    }
    tc_fence_after_sync();
    uint32_t sa[32], sb[32];
    tmem_ld32(tS + lane_off, sa);
    tmem_ld32(tS + lane_off + 32, sb);
    tmem_wait_ld();
    float x[kPfKeys];
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < kPfKeys; ++c) {
      const int key = kt * kPfKeys + c;
      const bool ok = row_ok && !failed && key <= qpos && !((bad >> (c / BS)) & 1);
      x[c] = ok ? __uint_as_float(c < 32 ? sa[c] : sb[c - 32]) * a.sl2 : -INFINITY;
      mx = fmaxf(mx, x[c]);
    }
    const float m_new = fmaxf(m_run, mx);
    const float alpha = m_new == -INFINITY ? 1.f : fast_exp2(m_run - m_new);
    // P = P_hi + P_lo, both in the operands' 16-bit type: rounding P to one
    // 16-bit value alone (8 significant bits for bf16) errs by up to 2^-9 of
    // each weight, which outputs formed by cancellation cannot absorb
    float psum = 0.f;
    uint32_t pk[kPfKeys / 2], pl[kPfKeys / 2];
#pragma unroll
    for (int c = 0; c < kPfKeys; c += 2) {
      const float p0 = x[c] == -INFINITY ? 0.f : fast_exp2(x[c] - m_new);
      const float p1 = x[c + 1] == -INFINITY ? 0.f : fast_exp2(x[c + 1] - m_new);
      psum += p0 + p1;
      const uint32_t hi = pack2<kBF16>(p0, p1);
      pk[c / 2] = hi;
      pl[c / 2] = pack2<kBF16>(p0 - to_float<kBF16>(hi & 0xffff), p1 - to_float<kBF16>(hi >> 16));
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      *reinterpret_cast<uint4*>(base + C::kOffP + swz128(r, c)) =
          make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      *reinterpret_cast<uint4*>(base + C::kOffP + C::kPBytes + swz128(r, c)) =
          make_uint4(pl[4 * c], pl[4 * c + 1], pl[4 * c + 2], pl[4 * c + 3]);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();  // P and Vt complete; S, K and V no longer read
    if (tid == 0 && !failed) {
      // ---- O tile = (P_hi + P_lo) Vt^T (2 x 4 MMAs of K = 16 along the keys)
      tc_fence_after_sync();
#pragma unroll
      for (int k = 0; k < kPfKeys / 16; ++k)
        umma_f16(tO, umma_desc_k128(sP + k * 32), umma_desc_k128(sVt + k * 32), kIdescO,
                 k > 0 ? 1u : 0u);
#pragma unroll
      for (int k = 0; k < kPfKeys / 16; ++k)
        umma_f16(tO, umma_desc_k128(sP + C::kPBytes + k * 32), umma_desc_k128(sVt + k * 32),
                 kIdescO, 1u);
      umma_commit(bar_o);
      // the next key tile's loads overlap this product and the O update
      if (kt + 1 < nkt) issue_tile(kt + 1);
    }
    if (!failed && !mbar_wait_bounded(bar_o, kt & 1)) {
      failed = true;
      record_error(PA_ERR_TIMEOUT);
    }
    tc_fence_after_sync();
#pragma unroll
    for (int c = 0; c < kPfD / 32; ++c) {
      uint32_t ot[32];
      tmem_ld32(tO + lane_off + 32 * c, ot);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) o[32 * c + j] = o[32 * c + j] * alpha + __uint_as_float(ot[j]);
    }
    tc_fence_before_sync();
    __syncthreads();  // S, the O tile, P and Vt are free again
  }

  if (row_ok) {
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
    for (int j = 0; j < kPfD / 8; ++j) {
      uint4 v;
      v.x = pack2<kBF16>(o[8 * j] * inv, o[8 * j + 1] * inv);
      v.y = pack2<kBF16>(o[8 * j + 2] * inv, o[8 * j + 3] * inv);
      v.z = pack2<kBF16>(o[8 * j + 4] * inv, o[8 * j + 5] * inv);
      v.w = pack2<kBF16>(o[8 * j + 6] * inv, o[8 * j + 7] * inv);
      orow[j] = v;
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
