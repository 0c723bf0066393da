// Shared-prefix-aware (cascade) decode attention, sm_100a.
//
// Method: sequences forked from one prompt (parallel sampling, beam search, a
// common system prompt) name the same physical blocks at the head of their
// block tables ("PagedAttention", Ultralytics glossary, section "Diziler
// Arasinda Bloklari Paylasma").  Plain decode reads those blocks once per
// sequence; here they are read once per group.
//
// Work decomposition
//   chunk = up to 16 / G members of one group that share P leading blocks
//           (or one sequence on its own, P = 0)
//   range = a run of at most R blocks that is either shared (the first P
//           blocks, attended by every member's G query heads: up to 16 rows)
//           or one member's own (its blocks from P on, attended by its G
//           heads only); the planning kernel cuts every chunk into such
//           ranges of about equal length, each with its partial slot
//   item  = (range, kv head); CTA = 4 warps, persistent, items from an atomic
//           counter; warp = every 4th block of the range through a ring of
//           stages, each K or V tile one tiled TMA copy (the decode kernel's
//           tensor maps, swizzle and layout), table entries read ahead
// A shared range runs m16n8k16 tiles whose 16 rows are the chunk's query
// heads: S = Q K^T (A = Q in registers, B = K rows), online softmax per row,
// O += P V (A = P straight from the S accumulators, B = V by ldmatrix.trans).
// An own range runs the decode kernel's form with the member's heads as the
// MMA's N = 8 columns: S^T = K Q^T, P^T by movmatrix, O^T += V^T P^T, half the
// MMAs of a 16-row tile.  When every member's own part is short (a fork,
// where each sample owns only its copied partial block), one own-group range
// takes them all, warp w walking member w's blocks, so the chunk pays one
// range start and one partial instead of one per member.  bf16 keeps P as hi + lo parts in both.
// The warps' states merge through shared memory; a chunk of one range writes
// the output, otherwise every range writes (log-sum-exp, normalised output)
// per row (-inf for rows it does not attend) and the CTA that finishes the
// chunk's last range merges them.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode.cuh"

namespace pa {

constexpr int kCascadeRows = 16;        // query rows per chunk (members x heads)
constexpr int kRangeShared = -1;        // range member field: the shared blocks
constexpr int kRangeOwnGroup = -2;      // ... every member's own blocks, one warp each
// a chunk of at most 4 members with at most 8 heads per kv head whose own
// parts are all this short runs them as one own-group range, not one range
// (four warps, a merge) per member
constexpr int kOwnGroupMaxBlocks = 8;
constexpr int kCascadeMaxRanges = 512;  // ranges per chunk (their weights sit in smem)
// work items (x Hkv) the range length aims at: ~1.5 waves of 444 persistent
// CTAs (on the shared-prefix workload 666 ran 74.9 us, 555: 75.0, 888: 74.8,
// 444: 78.0 -- too few items leave CTAs idle at the end; with one range form
// 1332 had run 87.4 against 80.1, shorter ranges paying start and merge)
constexpr int kCascadeTargetItems = 666;

struct CascadeArgs {
  CUtensorMap tmap_k;          // decode tensor maps over the pools
  CUtensorMap tmap_v;
  void* out;                   // [B, Hq, D]
  const void* q;               // [B, Hq, D]
  const int32_t* block_tables;
  const int32_t* context_lens;
  const int32_t* chunk_seqs;   // members, chunk by chunk
  const int4* chunks;          // [2 * chunks]: (member offset, members, shared blocks, first
                               // slot), (ranges, -, -, -)
  const int4* ranges;          // [slots]: (chunk, member, or -1 for shared, -2 for every
                               // member's own, first block, end block): table entries of the
                               // leader (shared) or the member(s)
  const int32_t* total;        // number of ranges
  int32_t* counter;            // work counter (zeroed by the planning kernel)
  int32_t* arrived;            // [chunks * Hkv] ranges finished
  float* lse_part;             // [slots * Hkv * 16]
  float* o_part;               // [slots * Hkv * 16 * D]
  int hq, hkv, group, max_blocks, num_blocks;
  float sl2;                   // scale * k_scale * log2(e)
  float out_scale;             // v_scale
};

// Query fragments of an e4m3 cache, whose products run in fp16: the
// values of one query row (or head) are scaled by the power of two 2^-e that
// brings their largest |q| into [2^14, 2^15) before the fp16 conversion, and
// 2^e goes back into that row's softmax scale.  Returns e (0 for a zero or
// non-finite row); `amax` is this thread's share, reduced over the 4 threads
// of its fragment row group.
__device__ __forceinline__ int q_row_exponent(float amax) {
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  return (amax > 0.f && amax < INFINITY) ? max(-126, min(126, ilogbf(amax) - 14)) : 0;
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

template <bool kQBF16>
__device__ __forceinline__ float amax4(uint2 w) {
  return fmax3(fmax3(0.f, fabsf(to_float<kQBF16>(w.x & 0xffff)), fabsf(to_float<kQBF16>(w.x >> 16))),
               fabsf(to_float<kQBF16>(w.y & 0xffff)), fabsf(to_float<kQBF16>(w.y >> 16)));
}

template <int CK, bool kQBF16, int D, int BS>
// at most 170 registers a thread (65,536 / (3 x 128)), so that three CTAs
// share an SM in every instance (the bf16 bs-32 one needed 171)
__global__ void __launch_bounds__(kDecodeThreads, 3)
cascade_kernel(const __grid_constant__ CascadeArgs a) {
  using C = DecodeCfg<CK, D, BS>;
  constexpr bool kE4M3 = CK == kCacheE4M3;
  constexpr bool kMmaBF16 = C::kMmaBF16;  // bf16 cache: bf16 products; f16 and e4m3: fp16
  constexpr bool kPBF16 = kMmaBF16;       // bf16 P is kept as hi + lo parts
  constexpr int kStages = C::kStages;
  constexpr int kNT = D / 8;  // 16-row form: output n-tiles (8 dims each)
  constexpr int kRows = kCascadeRows;
  static_assert(C::kWarpBytes >= (kRows * D + 2 * kRows) * 4, "warp ring too small for the merge");
  static_assert(kDecodeWarps * C::kWarpBytes >= (kCascadeMaxRanges + 1) * kRows * 4,
                "rings too small for the range weights");
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_item;
  __shared__ int s_flag;
  __shared__ int s_seq[kRows];  // the chunk's members
  __shared__ int s_ctx[kRows];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;   // fragment row group
  const int tig = lane & 3;  // thread in group
  const int li = lane >> 3;  // which 8x8 matrix of an ldmatrix.x4 this lane addresses

  const uint32_t smem_s = smem_addr(smem);
  const uint32_t ring_s = (smem_s + kBarrierBytes + kTileAlign - 1) & ~uint32_t(kTileAlign - 1);
  const uint32_t wbase_s = ring_s + warp * C::kWarpBytes;
  uint8_t* const ring = smem + (ring_s - smem_s);
  float* const scr = reinterpret_cast<float*>(ring + warp * C::kWarpBytes);  // merge scratch
  const uint32_t bar0 = smem_s + warp * kStages * 8;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
  }
  // launched behind cascade_plan_kernel: nothing from global memory before it is done
  grid_dependency_wait();
  if (threadIdx.x == 0) {
    prefetch_tensormap(&a.tmap_k);
    prefetch_tensormap(&a.tmap_v);
    s_item = blockIdx.x;  // CTA c starts on item c; later ones come from the counter
  }
  __syncthreads();

  const int total = *a.total * a.hkv;
  const int G = a.group;
  uint32_t n_issued = 0, n_consumed = 0;
  uint32_t skip_stage = 0;
  bool failed = false;

  for (;;) {
    const int item = s_item;
    if (item >= total) break;
    const int kvh = item % a.hkv;
    const int slot = item / a.hkv;
    const int4 rd = a.ranges[slot];
    const int chunk = rd.x, member = rd.y, b0 = rd.z, b1 = rd.w;
    const bool shared = member == kRangeShared;
    // every member's own blocks at once, warp w walking member w's
    const bool group = member == kRangeOwnGroup;
    // the 16-row form serves shared ranges, and own ranges of a member with
    // more than 8 heads per kv head; other own ranges take the 8-column form
    const bool rowform = shared || G > kMaxGroup;
    const int4 c0 = a.chunks[2 * chunk];
    const int members = c0.y, slot0 = c0.w;
    const int nranges = a.chunks[2 * chunk + 1].x;
    const int rows = members * G;
    if (threadIdx.x < members) {
      const int seq = a.chunk_seqs[c0.x + threadIdx.x];
      s_seq[threadIdx.x] = seq;
      s_ctx[threadIdx.x] = a.context_lens[seq];  // validated by the planning kernel
    }
    __syncthreads();
    // this warp's member (idle warps of an own-group range take the last
    // member's sequence and walk no block)
    const int wm = shared ? 0 : (group ? min(warp, members - 1) : member);
    const int own_seq = s_seq[wm];
    const int own_ctx = shared ? 0 : s_ctx[wm];
    const int nblk = b1 - b0;
    const int nb_w = group ? (warp < members ? max(0, (own_ctx + BS - 1) / BS - b0) : 0)
                           : (nblk > warp ? (nblk - warp + kDecodeWarps - 1) / kDecodeWarps : 0);
    const int32_t* table = a.block_tables + static_cast<int64_t>(own_seq) * a.max_blocks;
    // table index of the warp's i-th block: every 4th block of the range,
    // or, in an own-group range, every block of its member from b0 on
    auto jblk = [&](int i) { return group ? b0 + i : b0 + warp + i * kDecodeWarps; };

    // ---- table entries of the warp's blocks, 32 ahead in registers (lane l
    // holds the warp's block 32 * chunk + l)
    auto load_chunk = [&](int c) -> int {
      const int i = c * 32 + lane;
      return i < nb_w ? table[jblk(i)] : -1;
    };
    int tab_chunk = 0;
    int tab_cur = load_chunk(0);
    int tab_nxt = load_chunk(1);
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
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (ok) {
          mbar_arrive_expect_tx(bar, 2u * C::kTileBytes);
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
    // wait for the warp's next block; false when it is skipped or failed
    auto consume = [&](int& st) -> bool {
      st = n_consumed % kStages;
      const uint32_t par = (n_consumed / kStages) & 1u;
      if (!failed) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar0 + 8 * st, par));
        if (!ok) {
          failed = true;
          if (lane == 0) record_error(PA_ERR_TIMEOUT);
        }
      }
      return !failed && !((skip_stage >> st) & 1u);
    };
    auto release = [&](int i) {
      __syncwarp();
      ++n_consumed;
      if (!failed && i + kStages < nb_w) issue(i + kStages);
    };

    if (rowform) {
      // ================= 16-row tiles =====================================
      // rows: a shared range's are the chunk's (member r / G, head r % G),
      // an own range's the member's G heads
      const int nrows = shared ? rows : G;
      uint32_t qa[D / 16][4];
      float sl2r[2] = {a.sl2, a.sl2};  // softmax scale of rows g, g + 8 (log2 units)
      {
        const uint16_t* qrow[2];
        bool okr[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = g + 8 * h;
          okr[h] = r < nrows;
          const int rr = okr[h] ? r : 0;
          const int seq = s_seq[shared ? rr / G : member];
          qrow[h] = reinterpret_cast<const uint16_t*>(a.q) +
                    (static_cast<int64_t>(seq) * a.hq + kvh * G + rr % G) * D;
        }
        if constexpr (kE4M3) {
          // k-step ks takes dims 16 ks + 4 tig .. +3 (the order ldmatrix
          // gives 8-bit K rows): a0 / a1 the first pair, a2 / a3 the second
          uint2 qw[2][D / 16];
          float am[2] = {0.f, 0.f};
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              qw[h][ks] = okr[h] ? *reinterpret_cast<const uint2*>(qrow[h] + ks * 16 + 4 * tig)
                                 : make_uint2(0u, 0u);
              am[h] = fmaxf(am[h], amax4<kQBF16>(qw[h][ks]));
            }
          int e[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            e[h] = q_row_exponent(am[h]);
            sl2r[h] = a.sl2 * pow2f(e[h]);
          }
          const float dn0 = pow2f(-e[0]), dn1 = pow2f(-e[1]);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = pack_f16x2(to_float<kQBF16>(qw[0][ks].x & 0xffff) * dn0, to_float<kQBF16>(qw[0][ks].x >> 16) * dn0);
            qa[ks][1] = pack_f16x2(to_float<kQBF16>(qw[1][ks].x & 0xffff) * dn1, to_float<kQBF16>(qw[1][ks].x >> 16) * dn1);
            qa[ks][2] = pack_f16x2(to_float<kQBF16>(qw[0][ks].y & 0xffff) * dn0, to_float<kQBF16>(qw[0][ks].y >> 16) * dn0);
            qa[ks][3] = pack_f16x2(to_float<kQBF16>(qw[1][ks].y & 0xffff) * dn1, to_float<kQBF16>(qw[1][ks].y >> 16) * dn1);
          }
        } else {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const int d0 = ks * 16 + 2 * tig;
            qa[ks][0] = okr[0] ? *reinterpret_cast<const uint32_t*>(qrow[0] + d0) : 0u;
            qa[ks][1] = okr[1] ? *reinterpret_cast<const uint32_t*>(qrow[1] + d0) : 0u;
            qa[ks][2] = okr[0] ? *reinterpret_cast<const uint32_t*>(qrow[0] + d0 + 8) : 0u;
            qa[ks][3] = okr[1] ? *reinterpret_cast<const uint32_t*>(qrow[1] + d0 + 8) : 0u;
          }
        }
      }
      float acc[kNT][4];
#pragma unroll
      for (int n = 0; n < kNT; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.f;
      float m_run[2] = {-INFINITY, -INFINITY};  // rows g, g + 8 (log2 units)
      float l_run[2] = {0.f, 0.f};              // this thread's share of the row sums
      for (int i = 0; i < nb_w; ++i) {
        int st;
        if (consume(st)) {
          const uint32_t sK = wbase_s + st * C::kStageBytes;
          const uint32_t sV = sK + C::kTileBytes;
          // tokens of the block inside the range: all of a shared block; an
          // own range's last block may end early
          const int valid = shared ? BS : min(BS, own_ctx - (b0 + warp + i * kDecodeWarps) * BS);
#pragma unroll
          for (int kt = 0; kt < BS / 16; ++kt) {
            // S = Q K^T for 16 keys: two n-tiles of 8 keys, two accumulator chains
            float s[2][4], so[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) s[nt][e] = so[nt][e] = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              const int key = kt * 16 + nt * 8 + (lane & 7);
              if constexpr (kE4M3) {
                // one ldmatrix.x4 = four 16-dim chunks of 8 keys; matrix j
                // gives this thread dims 16 (c + j) + 4 tig .. +3 of key g
#pragma unroll
                for (int c = 0; c < D / 16; c += 4) {
                  uint32_t r[4];
                  ldsm_x4(sK + tile_off<C>(key, (c + li) * 16), r[0], r[1], r[2], r[3]);
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    const uint32_t k0 = e4m3x2_to_f16x2(r[j] & 0xffff);
                    const uint32_t k1 = e4m3x2_to_f16x2(r[j] >> 16);
                    if (j & 1) mma_16816<false>(so[nt], qa[c + j], k0, k1);
                    else mma_16816<false>(s[nt], qa[c + j], k0, k1);
                  }
                }
              } else {
#pragma unroll
                for (int ks = 0; ks < D / 16; ks += 2) {
                  uint32_t k0, k1, k2, k3;
                  ldsm_x4(sK + tile_off<C>(key, ((ks + (li >> 1)) * 16 + (li & 1) * 8) * 2), k0, k1,
                          k2, k3);
                  mma_16816<kMmaBF16>(s[nt], qa[ks], k0, k1);
                  mma_16816<kMmaBF16>(so[nt], qa[ks + 1], k2, k3);
                }
              }
            }
            // online softmax of rows g (elements 0, 1) and g + 8 (2, 3); keys
            // past an own range's end (only in its last block) get -inf
            const bool part = valid < BS;
            float alpha[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float x[4];
#pragma unroll
              for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c)
                  x[2 * nt + c] = (s[nt][2 * h + c] + so[nt][2 * h + c]) * sl2r[h];
              if (part) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (kt * 16 + (e >> 1) * 8 + 2 * tig + (e & 1) >= valid) x[e] = -INFINITY;
              }
              float bm = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
              bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
              bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
              const float mn = fmaxf(m_run[h], bm);
              alpha[h] = fast_exp2(m_run[h] - mn);
              m_run[h] = mn;
              float ps = 0.f;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                x[e] = fast_exp2(x[e] - mn);
                ps += x[e];
              }
              l_run[h] = l_run[h] * alpha[h] + ps;
#pragma unroll
              for (int nt = 0; nt < 2; ++nt) {
                s[nt][2 * h] = x[2 * nt];
                s[nt][2 * h + 1] = x[2 * nt + 1];
              }
            }
#pragma unroll
            for (int n = 0; n < kNT; ++n) {
              acc[n][0] *= alpha[0];
              acc[n][1] *= alpha[0];
              acc[n][2] *= alpha[1];
              acc[n][3] *= alpha[1];
            }
            // P as the A operand (the S accumulators of two n-tiles are the A
            // fragment); bf16 keeps P as hi + lo parts (one bf16 value errs by
            // up to 2^-9 of a weight), fp16 P keeps 11 bits in one part
            uint32_t pa[4], pl[4];
            pa[0] = pack2<kMmaBF16>(s[0][0], s[0][1]);
            pa[1] = pack2<kMmaBF16>(s[0][2], s[0][3]);
            pa[2] = pack2<kMmaBF16>(s[1][0], s[1][1]);
            pa[3] = pack2<kMmaBF16>(s[1][2], s[1][3]);
            if constexpr (kPBF16) {
              pl[0] = pack_bf16x2(s[0][0] - to_float<true>(pa[0] & 0xffff), s[0][1] - to_float<true>(pa[0] >> 16));
              pl[1] = pack_bf16x2(s[0][2] - to_float<true>(pa[1] & 0xffff), s[0][3] - to_float<true>(pa[1] >> 16));
              pl[2] = pack_bf16x2(s[1][0] - to_float<true>(pa[2] & 0xffff), s[1][1] - to_float<true>(pa[2] >> 16));
              pl[3] = pack_bf16x2(s[1][2] - to_float<true>(pa[3] & 0xffff), s[1][3] - to_float<true>(pa[3] >> 16));
            }
            // O += P V; values of keys past an own range's end are zeroed in the
            // fragments (they may hold anything, NaN included)
            const int tk = kt * 16 + 2 * tig;
            const uint32_t m_lo = part ? pair_mask(tk < valid, tk + 1 < valid) : 0xffffffffu;
            const uint32_t m_hi = part ? pair_mask(tk + 8 < valid, tk + 9 < valid) : 0xffffffffu;
            const int vkey = kt * 16 + (li & 1) * 8 + (lane & 7);
            if constexpr (kE4M3) {
              // matrices (keys 0-7 | 8-15) x (chunk c | c + 1); after the byte
              // permute the low half holds keys 2tig, 2tig+1 of dim 2g of the
              // chunk, the high half of dim 2g + 1: n-tile 2 chunk + parity
#pragma unroll
              for (int c = 0; c < D / 16; c += 2) {
                uint32_t r0, r1, r2, r3;
                ldsm_x4_trans(sV + tile_off<C>(vkey, (c + (li >> 1)) * 16), r0, r1, r2, r3);
                if (part) {
                  r0 &= m_lo; r1 &= m_hi; r2 &= m_lo; r3 &= m_hi;
                }
                const uint32_t p0 = __byte_perm(r0, 0, 0x3120), p1 = __byte_perm(r1, 0, 0x3120);
                const uint32_t p2 = __byte_perm(r2, 0, 0x3120), p3 = __byte_perm(r3, 0, 0x3120);
                mma_16816<false>(acc[2 * c], pa, e4m3x2_to_f16x2(p0 & 0xffff), e4m3x2_to_f16x2(p1 & 0xffff));
                mma_16816<false>(acc[2 * c + 1], pa, e4m3x2_to_f16x2(p0 >> 16), e4m3x2_to_f16x2(p1 >> 16));
                mma_16816<false>(acc[2 * c + 2], pa, e4m3x2_to_f16x2(p2 & 0xffff), e4m3x2_to_f16x2(p3 & 0xffff));
                mma_16816<false>(acc[2 * c + 3], pa, e4m3x2_to_f16x2(p2 >> 16), e4m3x2_to_f16x2(p3 >> 16));
              }
            } else {
#pragma unroll
              for (int n2 = 0; n2 < D / 16; ++n2) {
                uint32_t v0, v1, v2, v3;
                ldsm_x4_trans(sV + tile_off<C>(vkey, (n2 * 16 + (li >> 1) * 8) * 2), v0, v1, v2, v3);
                if (part) {
                  v0 &= m_lo; v1 &= m_hi; v2 &= m_lo; v3 &= m_hi;
                }
                mma_16816<kMmaBF16>(acc[2 * n2], pa, v0, v1);
                mma_16816<kMmaBF16>(acc[2 * n2 + 1], pa, v2, v3);
                if constexpr (kPBF16) {
                  mma_16816<kMmaBF16>(acc[2 * n2], pl, v0, v1);
                  mma_16816<kMmaBF16>(acc[2 * n2 + 1], pl, v2, v3);
                }
              }
            }
          }
        }
        release(i);
      }
      // the warp's state into its scratch: O [16][D], max [16], sum [16]
      float lsum[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float v = l_run[h];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        lsum[h] = v;
      }
#pragma unroll
      for (int n = 0; n < kNT; ++n) {
        if constexpr (kE4M3) {  // n-tile n: chunk n / 2, dims of parity n % 2
          const int d = 16 * (n >> 1) + 4 * tig + (n & 1);
          scr[g * D + d] = acc[n][0];
          scr[g * D + d + 2] = acc[n][1];
          scr[(g + 8) * D + d] = acc[n][2];
          scr[(g + 8) * D + d + 2] = acc[n][3];
        } else {
          const int d = n * 8 + 2 * tig;
          *reinterpret_cast<float2*>(scr + g * D + d) = make_float2(acc[n][0], acc[n][1]);
          *reinterpret_cast<float2*>(scr + (g + 8) * D + d) = make_float2(acc[n][2], acc[n][3]);
        }
      }
      if (tig == 0) {
        scr[kRows * D + g] = m_run[0];
        scr[kRows * D + g + 8] = m_run[1];
        scr[kRows * D + kRows + g] = lsum[0];
        scr[kRows * D + kRows + g + 8] = lsum[1];
      }
    } else {
      // ================= own range: the member's heads as N = 8 ==========
      // (the decode kernel's form: S^T = K Q^T, P^T by movmatrix, O^T += V^T P^T)
      constexpr int kDT = D / 16;
      uint32_t qf[kDT][2];
      float sl2c[2] = {a.sl2, a.sl2};  // softmax scale of heads 2tig, 2tig + 1
      {
        const bool hv = g < G;
        const uint16_t* qrow = reinterpret_cast<const uint16_t*>(a.q) +
                               (static_cast<int64_t>(own_seq) * a.hq + kvh * G + (hv ? g : 0)) * D;
        if constexpr (kE4M3) {
          uint2 qw[kDT];
          float am = 0.f;
#pragma unroll
          for (int ks = 0; ks < kDT; ++ks) {
            qw[ks] = hv ? *reinterpret_cast<const uint2*>(qrow + ks * 16 + 4 * tig) : make_uint2(0u, 0u);
            am = fmaxf(am, amax4<kQBF16>(qw[ks]));
          }
          const int e = q_row_exponent(am);
          const float dn = pow2f(-e);
#pragma unroll
          for (int ks = 0; ks < kDT; ++ks) {
            qf[ks][0] = pack_f16x2(to_float<kQBF16>(qw[ks].x & 0xffff) * dn, to_float<kQBF16>(qw[ks].x >> 16) * dn);
            qf[ks][1] = pack_f16x2(to_float<kQBF16>(qw[ks].y & 0xffff) * dn, to_float<kQBF16>(qw[ks].y >> 16) * dn);
          }
          sl2c[0] = a.sl2 * pow2f(__shfl_sync(0xffffffffu, e, 8 * tig));
          sl2c[1] = a.sl2 * pow2f(__shfl_sync(0xffffffffu, e, 8 * tig + 4));
        } else {
#pragma unroll
          for (int ks = 0; ks < kDT; ++ks) {
            qf[ks][0] = hv ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 2 * tig) : 0u;
            qf[ks][1] = hv ? *reinterpret_cast<const uint32_t*>(qrow + ks * 16 + 8 + 2 * tig) : 0u;
          }
        }
      }
      float acc[kDT][4];
#pragma unroll
      for (int dt = 0; dt < kDT; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[dt][e] = 0.f;
      float m_run[2] = {-INFINITY, -INFINITY};  // heads 2tig, 2tig + 1 (log2 units)
      float l_run[2] = {0.f, 0.f};              // this thread's share of the sums
      for (int i = 0; i < nb_w; ++i) {
        int st;
        if (consume(st)) {
          const uint32_t sK = wbase_s + st * C::kStageBytes;
          const uint32_t sV = sK + C::kTileBytes;
          const int j = jblk(i);                            // the block's table entry
          const int valid = min(BS, own_ctx - j * BS);      // its tokens inside the context
          // S^T = K Q^T (rows: tokens, cols: the member's heads), four chains
          float s[BS / 16][4];
#pragma unroll
          for (int mt = 0; mt < BS / 16; ++mt) {
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
            float s2[4] = {0.f, 0.f, 0.f, 0.f}, s3[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (kE4M3) {
              const int tok = mt * 16 + (lane & 7) + (li & 1) * 8;
#pragma unroll
              for (int cp = 0; cp < kDT / 2; ++cp) {
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
              for (int ks = 0; ks < kDT; ++ks) {
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
              const int tok = mt * 16 + g + (e >> 1) * 8;
              const float x = ((s0[e] + s1[e]) + (s2[e] + s3[e])) * sl2c[e & 1];
              s[mt][e] = tok < valid ? x : -INFINITY;
            }
          }
          // online softmax per head column (every block has a valid token)
          float alpha[2];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float bm = -INFINITY;
#pragma unroll
            for (int mt = 0; mt < BS / 16; ++mt) bm = fmaxf(bm, fmaxf(s[mt][c], s[mt][2 + c]));
            bm = shfl_xor_max(bm);
            const float mn = fmaxf(m_run[c], bm);
            alpha[c] = fast_exp2(m_run[c] - mn);
            m_run[c] = mn;
            float ps = 0.f;
#pragma unroll
            for (int mt = 0; mt < BS / 16; ++mt) {
              s[mt][c] = fast_exp2(s[mt][c] - mn);
              s[mt][2 + c] = fast_exp2(s[mt][2 + c] - mn);
              ps += s[mt][c] + s[mt][2 + c];
            }
            l_run[c] = l_run[c] * alpha[c] + ps;
          }
#pragma unroll
          for (int dt = 0; dt < kDT; ++dt) {
            acc[dt][0] *= alpha[0];
            acc[dt][1] *= alpha[1];
            acc[dt][2] *= alpha[0];
            acc[dt][3] *= alpha[1];
          }
          // P^T as the B operand (8x8 (token, head) tiles transposed in
          // registers); bf16 keeps hi + lo parts
          uint32_t pb[BS / 16][2], pl[BS / 16][2];
#pragma unroll
          for (int mt = 0; mt < BS / 16; ++mt) {
            const uint32_t h0 = pack2<kMmaBF16>(s[mt][0], s[mt][1]);
            const uint32_t h1 = pack2<kMmaBF16>(s[mt][2], s[mt][3]);
            pb[mt][0] = movmatrix_trans(h0);
            pb[mt][1] = movmatrix_trans(h1);
            if constexpr (kPBF16) {
              pl[mt][0] = movmatrix_trans(pack_bf16x2(s[mt][0] - to_float<true>(h0 & 0xffff),
                                                      s[mt][1] - to_float<true>(h0 >> 16)));
              pl[mt][1] = movmatrix_trans(pack_bf16x2(s[mt][2] - to_float<true>(h1 & 0xffff),
                                                      s[mt][3] - to_float<true>(h1 >> 16)));
            }
          }
          // O^T += V^T P^T; in the member's last block the value rows past its
          // length are zeroed in the fragments (they may hold anything)
          const bool part = valid < BS;
#pragma unroll
          for (int mt = 0; mt < BS / 16; ++mt) {
            uint32_t m_lo = 0xffffffffu, m_hi = 0xffffffffu;  // tokens 2tig(+1), 2tig+8(+9)
            if (part) {
              const int tk = mt * 16 + 2 * tig;
              m_lo = pair_mask(tk < valid, tk + 1 < valid);
              m_hi = pair_mask(tk + 8 < valid, tk + 9 < valid);
            }
            if constexpr (kE4M3) {
              const int tok = mt * 16 + (lane & 7) + (li & 1) * 8;
#pragma unroll
              for (int cp = 0; cp < kDT / 2; ++cp) {
                uint32_t r0, r1, r2, r3;
                ldsm_x4_trans(sV + tile_off<C>(tok, (2 * cp + (li >> 1)) * 16), r0, r1, r2, r3);
                if (part) {
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
              for (int dt = 0; dt < kDT; ++dt) {
                uint32_t af[4];
                ldsm_x4_trans(sV + tile_off<C>(tok, (dt * 16 + (li & 1) * 8) * 2), af[0], af[1],
                              af[2], af[3]);
                if (part) {
                  af[0] &= m_lo; af[1] &= m_lo; af[2] &= m_hi; af[3] &= m_hi;
                }
                mma_16816<kMmaBF16>(acc[dt], af, pb[mt][0], pb[mt][1]);
                if constexpr (kPBF16) mma_16816<kMmaBF16>(acc[dt], af, pl[mt][0], pl[mt][1]);
              }
            }
          }
        }
        release(i);
      }
      // the warp's state into its scratch: O [8][D] (head-major), max [8], sum [8]
      const float lsum0 = shfl_xor_sum(l_run[0]);
      const float lsum1 = shfl_xor_sum(l_run[1]);
#pragma unroll
      for (int dt = 0; dt < kDT; ++dt) {
        // C fragment rows: 16-bit path dims 16dt + g (+8); 8-bit path 16dt + 2g (+1)
        const int dlo = kE4M3 ? dt * 16 + 2 * g : dt * 16 + g;
        const int dhi = kE4M3 ? dlo + 1 : dlo + 8;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int h = 2 * tig + c;
          scr[h * D + dlo] = acc[dt][c];
          scr[h * D + dhi] = acc[dt][2 + c];
        }
      }
      if (g == 0) {
        scr[8 * D + 2 * tig] = m_run[0];
        scr[8 * D + 2 * tig + 1] = m_run[1];
        scr[8 * D + 8 + 2 * tig] = lsum0;
        scr[8 * D + 8 + 2 * tig + 1] = lsum1;
      }
    }
    __syncthreads();
    {
      // combine the 4 warps; the 16-row form covers rows 0..nrow-1 of its
      // tile (scratch: O [16][D], max at 16 D, sums at 16 D + 16), the
      // 8-column form the member's G rows (scratch: O [8][D], max at 8 D,
      // sums at 8 D + 8); in an own-group range row r is member r / G's
      // head r % G, held by warp r / G alone
      const int nrow = (shared || group) ? rows : G;
      const int mrow = rowform ? kRows : 8;
      constexpr int kVec = 8;
      const int units = nrow * (D / kVec);
      for (int u = threadIdx.x; u < units; u += kDecodeThreads) {
        const int rl = u / (D / kVec);
        const int d0 = (u % (D / kVec)) * kVec;
        const int hl = group ? rl % G : rl;  // the row in the warps' scratch
        float mw[kDecodeWarps];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
          const float* sw = reinterpret_cast<const float*>(ring + w * C::kWarpBytes);
          mw[w] = (!group || w == rl / G) ? sw[mrow * D + hl] : -INFINITY;
          M = fmaxf(M, mw[w]);
        }
        float o[kVec];
#pragma unroll
        for (int v = 0; v < kVec; ++v) o[v] = 0.f;
        float L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kDecodeWarps; ++w) {
            if (group && w != rl / G) continue;
            const float* sw = reinterpret_cast<const float*>(ring + w * C::kWarpBytes);
            const float f = fast_exp2(mw[w] - M);
            L += f * sw[mrow * D + mrow + hl];
            const float4 x0 = *reinterpret_cast<const float4*>(sw + hl * D + d0);
            const float4 x1 = *reinterpret_cast<const float4*>(sw + hl * D + d0 + 4);
            o[0] += f * x0.x; o[1] += f * x0.y; o[2] += f * x0.z; o[3] += f * x0.w;
            o[4] += f * x1.x; o[5] += f * x1.y; o[6] += f * x1.z; o[7] += f * x1.w;
          }
          const float inv = a.out_scale / L;
#pragma unroll
          for (int v = 0; v < kVec; ++v) o[v] *= inv;
        }
        const int r = (shared || group) ? rl : member * G + rl;  // the chunk's row
        if (nranges == 1) {
          const int64_t qh = static_cast<int64_t>(s_seq[r / G]) * a.hq + kvh * G + r % G;
          uint4 pk;
          pk.x = pack2<kQBF16>(o[0], o[1]);
          pk.y = pack2<kQBF16>(o[2], o[3]);
          pk.z = pack2<kQBF16>(o[4], o[5]);
          pk.w = pack2<kQBF16>(o[6], o[7]);
          *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.out) + qh * D + d0) = pk;
        } else {
          const int64_t pi = (static_cast<int64_t>(slot) * a.hkv + kvh) * kRows + r;
          float* op = a.o_part + pi * D + d0;
          *reinterpret_cast<float4*>(op) = make_float4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<float4*>(op + 4) = make_float4(o[4], o[5], o[6], o[7]);
          if (d0 == 0) a.lse_part[pi] = (M == -INFINITY) ? -INFINITY : M + log2f(L);
        }
      }
      // the rows an own range does not attend carry no weight
      if (!shared && !group && nranges > 1)
        for (int r = threadIdx.x; r < rows; r += kDecodeThreads)
          if (r / G != member)
            a.lse_part[(static_cast<int64_t>(slot) * a.hkv + kvh) * kRows + r] = -INFINITY;
    }
    if (nranges > 1) {
      // the CTA that finishes the chunk's last range merges every range:
      // out = sum_i w_i o_i / sum_i w_i, w_i = 2^(lse_i - max lse); partials
      // are published with a fence before the arrival count, read through L2;
      // a range with no weight for a row (-inf) is skipped (its vector for
      // that row was not written)
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        const int prev = atomicAdd(&a.arrived[chunk * a.hkv + kvh], 1);
        s_flag = (prev == nranges - 1) ? 1 : 0;
      }
      __syncthreads();
      if (s_flag) {
        __threadfence();
        float* w_s = reinterpret_cast<float*>(ring);   // [nranges][16] weights
        float* wsum_s = w_s + nranges * kRows;         // [16]
        const int64_t base = (static_cast<int64_t>(slot0) * a.hkv + kvh) * kRows;
        const int64_t rstride = static_cast<int64_t>(a.hkv) * kRows;  // between slots
        for (int k2 = threadIdx.x; k2 < nranges * rows; k2 += kDecodeThreads) {
          const int i = k2 / rows, r = k2 % rows;
          w_s[i * kRows + r] = __ldcg(a.lse_part + base + i * rstride + r);
        }
        __syncthreads();
        for (int r = warp; r < rows; r += kDecodeWarps) {
          float M = -INFINITY;
          for (int i = lane; i < nranges; i += 32) M = fmaxf(M, w_s[i * kRows + r]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
          float W = 0.f;
          for (int i = lane; i < nranges; i += 32) {
            const float w = (M == -INFINITY) ? 0.f : fast_exp2(w_s[i * kRows + r] - M);
            w_s[i * kRows + r] = w;
            W += w;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
          if (lane == 0) wsum_s[r] = W;
        }
        __syncthreads();
        // one unit = 16 dims of one row; four ranges per pass, their loads
        // issued together (a weightless range loads nothing)
        constexpr int kVec = 16;
        const int units = rows * (D / kVec);
        for (int u = threadIdx.x; u < units; u += kDecodeThreads) {
          const int r = u / (D / kVec);
          const int d0 = (u % (D / kVec)) * kVec;
          float o[kVec];
#pragma unroll
          for (int v = 0; v < kVec; ++v) o[v] = 0.f;
          const float* op = a.o_part + (base + r) * D + d0;
          for (int i0 = 0; i0 < nranges; i0 += 4) {
            float w[4];
            float4 x[4][kVec / 4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              w[k] = i0 + k < nranges ? w_s[(i0 + k) * kRows + r] : 0.f;
#pragma unroll
              for (int q4 = 0; q4 < kVec / 4; ++q4)
                x[k][q4] = w[k] > 0.f ? __ldcg(reinterpret_cast<const float4*>(
                                            op + (i0 + k) * rstride * D + 4 * q4))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
              for (int q4 = 0; q4 < kVec / 4; ++q4) {
                o[4 * q4] += w[k] * x[k][q4].x;
                o[4 * q4 + 1] += w[k] * x[k][q4].y;
                o[4 * q4 + 2] += w[k] * x[k][q4].z;
                o[4 * q4 + 3] += w[k] * x[k][q4].w;
              }
          }
          const float W = wsum_s[r];
          const float inv = W > 0.f ? 1.f / W : 0.f;
          const int64_t qh = static_cast<int64_t>(s_seq[r / G]) * a.hq + kvh * G + r % G;
          uint4 pk0, pk1;
          pk0.x = pack2<kQBF16>(o[0] * inv, o[1] * inv);
          pk0.y = pack2<kQBF16>(o[2] * inv, o[3] * inv);
          pk0.z = pack2<kQBF16>(o[4] * inv, o[5] * inv);
          pk0.w = pack2<kQBF16>(o[6] * inv, o[7] * inv);
          pk1.x = pack2<kQBF16>(o[8] * inv, o[9] * inv);
          pk1.y = pack2<kQBF16>(o[10] * inv, o[11] * inv);
          pk1.z = pack2<kQBF16>(o[12] * inv, o[13] * inv);
          pk1.w = pack2<kQBF16>(o[14] * inv, o[15] * inv);
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.out) + qh * D + d0);
          dst[0] = pk0;
          dst[1] = pk1;
        }
      }
    }
    if (threadIdx.x == 0) s_item = static_cast<int>(gridDim.x) + atomicAdd(a.counter, 1);
    __syncthreads();           // scratch (= stage memory) and s_seq free again ...
    fence_proxy_async_smem();  // ... before the next item's tile loads
  }

  if (failed) {  // drain copies still in flight after a timeout (bounded again)
    while (n_consumed < n_issued) {
      const int st = n_consumed % kStages;
      mbar_wait_bounded(bar0 + 8 * st, (n_consumed / kStages) & 1u);
      ++n_consumed;
    }
  }
}

// ------------------------------------------------------------- planning
// One CTA of 1024 threads, once per call:
//  1. members are counted; a sequence listed twice, or outside [0, B),
//     invalidates every group holding it (those decode unshared; reported);
//  2. one warp per group: the shared blocks P = the longest run of leading
//     table entries equal in every member's row, cut so that every member
//     keeps at least one token of its own (P * bs <= len - 1).  Groups of
//     one member, or with a length outside [1, max_ctx], share nothing.  A
//     group with P > 0 becomes chunks of up to 16 / G members;
//  3. every other sequence is a chunk of its own (P = 0); a length outside
//     [0, min(max_ctx, max_blocks * bs)] counts as 0 and is reported;
//  4. the range length R = the largest of r_floor, T * Hkv /
//     kCascadeTargetItems (T = all chunks' blocks, shared ones once) and
//     what keeps a chunk under kCascadeMaxRanges ranges;
//  5. each chunk's shared blocks are cut into ceil(P / R) equal ranges and
//     each member's own blocks into max(1, ceil(n / R)) (an empty range
//     still writes a zero output), every range with its partial slot; in a
//     chunk of up to 4 members and 8 heads per kv head whose own parts are
//     all at most kOwnGroupMaxBlocks (and R) blocks, one own-group range
//     covers every member's own blocks instead; the work list holds one
//     (chunk, member / -1 / -2, first block, end block) per slot, and the
//     arrival counters and the work counter are zeroed.
// Chunk and slot numbers come from atomics (their order varies), but every
// output depends only on its chunk's ranges, merged in range order: results
// are the same from call to call.
__global__ void __launch_bounds__(1024) cascade_plan_kernel(
    const int32_t* __restrict__ ctx_lens, const int32_t* __restrict__ block_tables,
    const int32_t* __restrict__ group_start, const int32_t* __restrict__ group_seqs,
    int num_groups, int B, int max_ctx, int max_blocks, int bs, int group, int hkv, int r_floor,
    int32_t* seen, int32_t* chunk_seqs, int4* chunks, int4* ranges, int32_t* total,
    int32_t* counter, int32_t* arrived) {
  __shared__ int n_chunks, n_used, tv_sum, v_max, n_slots;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_launch_dependents();  // the cascade grid may set up while the plan runs
  if (tid == 0) {
    n_chunks = n_used = tv_sum = v_max = n_slots = 0;
    *counter = 0;
  }
  for (int s = tid; s < B; s += 1024) seen[s] = 0;
  __syncthreads();
  const int n_members = num_groups > 0 ? group_start[num_groups] : 0;
  for (int i = tid; i < n_members; i += 1024) {
    const int m = group_seqs[i];
    if (m >= 0 && m < B) atomicAdd(&seen[m], 1);
  }
  __syncthreads();
  const int per_chunk = max(1, kCascadeRows / group);
  for (int gi = warp; gi < num_groups; gi += 32) {
    const int m0 = group_start[gi], m1 = group_start[gi + 1];
    const int k = m1 - m0;
    const bool listed = k >= 2 && m0 >= 0 && m1 <= n_members;  // a well-formed range
    int limit = 1 << 30;
    int bad = 0;
    for (int i = m0 + lane; listed && i < m1; i += 32) {
      const int m = group_seqs[i];
      if (m < 0 || m >= B || seen[m] != 1) {
        bad = 1;
        continue;
      }
      const int c = ctx_lens[m];
      if (c < 1 || c > max_ctx || c > max_blocks * bs) bad = 1;
      else limit = min(limit, (c - 1) / bs);
    }
    const bool any_bad = __any_sync(0xffffffffu, bad);
    if (lane == 0 && k >= 2 && (!listed || any_bad)) record_error(PA_ERR_RANGE);
    if (!listed || any_bad) continue;
    limit = __reduce_min_sync(0xffffffffu, limit);
    // first table index below limit where some member differs from the first
    const int32_t* lead = block_tables + static_cast<int64_t>(group_seqs[m0]) * max_blocks;
    int first_diff = limit;
    for (int j = lane; j < limit; j += 32) {
      const int e = lead[j];
      bool same = true;
      for (int i = m0 + 1; i < m1; ++i)
        same &= block_tables[static_cast<int64_t>(group_seqs[i]) * max_blocks + j] == e;
      if (!same) {
        first_diff = j;
        break;
      }
    }
    const int P = __reduce_min_sync(0xffffffffu, first_diff);
    if (P <= 0) continue;
    const int nch = (k + per_chunk - 1) / per_chunk;
    int cbase = 0, mbase = 0;
    if (lane == 0) {
      cbase = atomicAdd(&n_chunks, nch);
      mbase = atomicAdd(&n_used, k);
    }
    cbase = __shfl_sync(0xffffffffu, cbase, 0);
    mbase = __shfl_sync(0xffffffffu, mbase, 0);
    for (int i = lane; i < k; i += 32) {
      const int m = group_seqs[m0 + i];
      chunk_seqs[mbase + i] = m;
      seen[m] = -1;  // claimed
    }
    for (int c = lane; c < nch; c += 32)
      chunks[2 * (cbase + c)] = make_int4(mbase + c * per_chunk, min(per_chunk, k - c * per_chunk), P, 0);
  }
  __syncthreads();
  for (int s = tid; s < B; s += 1024) {
    if (seen[s] == -1) continue;
    const int c = atomicAdd(&n_chunks, 1);
    const int m = atomicAdd(&n_used, 1);
    chunk_seqs[m] = s;
    chunks[2 * c] = make_int4(m, 1, 0, 0);
  }
  __syncthreads();
  const int nc = n_chunks;
  auto own_blocks = [&](int seq, int P) {  // a member's blocks from P on (0 if invalid)
    int len = ctx_lens[seq];
    if (len < 0 || len > max_ctx || len > max_blocks * bs) len = 0;  // only unshared ones
    return max(0, (len + bs - 1) / bs - P);
  };
  for (int c = tid; c < nc; c += 1024) {
    const int4 d = chunks[2 * c];
    int V = d.z;
    for (int i = 0; i < d.y; ++i) {
      const int seq = chunk_seqs[d.x + i];
      const int len = ctx_lens[seq];
      if (d.z == 0 && (len < 0 || len > max_ctx || len > max_blocks * bs))
        record_error(PA_ERR_DEVICE_BOUNDS);
      V += own_blocks(seq, d.z);
    }
    atomicAdd(&tv_sum, V);
    atomicMax(&v_max, V);
  }
  __syncthreads();
  const int R = max(max(r_floor, 1),
                    max(static_cast<int>((static_cast<int64_t>(tv_sum) * hkv + kCascadeTargetItems - 1) /
                                         kCascadeTargetItems),
                        (v_max + (kCascadeMaxRanges - kCascadeRows - 1) - 1) /
                            (kCascadeMaxRanges - kCascadeRows - 1)));
  for (int c = tid; c < nc; c += 1024) {
    const int4 d = chunks[2 * c];
    const int P = d.z;
    const int nsh = P > 0 ? (P + R - 1) / R : 0;
    // short own parts of a shared chunk: one own-group range
    int own_max = 0;
    for (int i = 0; i < d.y; ++i) own_max = max(own_max, own_blocks(chunk_seqs[d.x + i], P));
    const bool own_group = P > 0 && d.y <= kDecodeWarps && group <= kMaxGroup &&
                           own_max <= min(kOwnGroupMaxBlocks, R);
    int nr = nsh;
    if (own_group) nr += 1;
    else
      for (int i = 0; i < d.y; ++i) nr += max(1, (own_blocks(chunk_seqs[d.x + i], P) + R - 1) / R);
    const int slot0 = atomicAdd(&n_slots, nr);
    chunks[2 * c] = make_int4(d.x, d.y, P, slot0);
    chunks[2 * c + 1] = make_int4(nr, 0, 0, 0);
    int sl = slot0;
    if (nsh > 0) {
      const int len = (P + nsh - 1) / nsh;  // equal shared ranges
      for (int k = 0; k < nsh; ++k)
        ranges[sl++] = make_int4(c, kRangeShared, k * len, min(P, (k + 1) * len));
    }
    if (own_group) {
      ranges[sl++] = make_int4(c, kRangeOwnGroup, P, P + own_max);
    } else {
      for (int i = 0; i < d.y; ++i) {
        const int n = own_blocks(chunk_seqs[d.x + i], P);
        const int no = max(1, (n + R - 1) / R);
        const int len = n > 0 ? (n + no - 1) / no : 0;  // equal own ranges
        for (int k = 0; k < no; ++k)
          ranges[sl++] = make_int4(c, i, P + min(n, k * len), P + min(n, (k + 1) * len));
      }
    }
    for (int h = 0; h < hkv; ++h) arrived[c * hkv + h] = 0;
  }
  __syncthreads();
  if (tid == 0) *total = n_slots;
}

}  // namespace pa
