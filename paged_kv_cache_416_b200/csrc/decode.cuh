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
//   item  = (sequence, context range of split_tokens tokens, kv head)
//   CTA   = 4 warps; a persistent grid pulls items from an atomic counter
//   warp  = takes every 4th block of the item's range; each warp owns a ring
//           of kStages shared-memory stages, one stage = the K and V rows of
//           one block for one kv head, filled by 1-D bulk asynchronous copies
//           (one per token row, completion counted on an mbarrier)
// Per block and warp, with the packed heads as the MMA's N = 8 columns:
//   S^T[t, g] = K[t, :] . Q[g, :]        m16n8k16, A = K rows (ldmatrix)
//   online softmax over t per column g   (exp2, running max and sum)
//   O^T[d, g] += V^T[d, t] P^T[t, g]     A = V (ldmatrix.trans), B = P^T
//                                         (S^T fragment transposed in
//                                         registers with movmatrix)
// The warps' partial (max, sum, O) are merged through shared memory at the
// end of an item; a split item writes (log-sum-exp, O / sum) to the
// workspace and merge_kernel combines the ranges of a sequence.
#pragma once

#include "common.cuh"

namespace pa {

enum CacheKind : int { kCacheF16 = 0, kCacheBF16 = 1, kCacheE4M3 = 2 };

constexpr int kDecodeWarps = 4;
constexpr int kDecodeThreads = kDecodeWarps * 32;
constexpr int kMaxGroup = 8;          // packed query heads per kv head (MMA N)
constexpr int kBarrierBytes = 256;    // mbarrier area at the start of smem

template <int CK, int D, int BS>
struct DecodeCfg {
  static constexpr int kElem = (CK == kCacheE4M3) ? 1 : 2;
  static constexpr int kRowBytes = D * kElem;          // one token row of one head
  static constexpr int kRowStride = kRowBytes + 16;    // padded: ldmatrix rows hit distinct banks
  static constexpr int kStageBytes = 2 * BS * kRowStride;  // K rows then V rows
  static constexpr int kBudget = 110 * 1024;           // per CTA: two CTAs fit one SM
  static constexpr int kStagesRaw = kBudget / (kDecodeWarps * kStageBytes);
  static constexpr int kStages = kStagesRaw < 1 ? 1 : (kStagesRaw > 6 ? 6 : kStagesRaw);
  static constexpr int kWarpBytes = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarrierBytes + kDecodeWarps * kWarpBytes;
  static constexpr int kTokTiles = BS / 16;
  static constexpr int kDimTiles = D / 16;
  static constexpr bool kMmaBF16 = (CK == kCacheBF16);
  // merge scratch of one warp: O[8][D] fp32, then max[8], sum[8]
  static constexpr int kScratchBytes = (kMaxGroup * D + 2 * kMaxGroup) * 4;
  static_assert(kWarpBytes >= kScratchBytes, "warp ring too small for the merge scratch");
  static_assert(kDecodeWarps * kStages <= kBarrierBytes / 8, "too many mbarriers");
  static_assert(kRowBytes % 16 == 0, "bulk copies move 16-byte multiples");
};

struct DecodeArgs {
  void* out;
  const void* q;
  const uint8_t* k_pool;
  const uint8_t* v_pool;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int32_t* counter;        // workspace: work-queue counter (zeroed by plan_kernel)
  const int32_t* total;    // workspace: number of items (written by plan_kernel)
  const int32_t* seq_off;  // workspace: [B + 1] first range index of each sequence
  float* lse_part;         // workspace: [ranges * Hq]
  float* o_part;           // workspace: [ranges * Hq * D]
  int num_seqs, hq, hkv, group, max_blocks, num_blocks, max_ctx, split_tokens;
  float sl2;               // scale * k_scale * log2(e)
  float out_scale;         // v_scale
};

// ---------------------------------------------------------------- planning
// One CTA: validates context lengths, counts each sequence's ranges
// (max(1, ceil(len / split_tokens))), writes their exclusive prefix sum,
// the item total (ranges * Hkv) and zeroes the work counter.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ ctx_lens, int B,
                                                    int max_ctx, int max_blocks, int bs, int S,
                                                    int hkv, int32_t* counter, int32_t* total,
                                                    int32_t* seq_off) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry = 0;
    *counter = 0;
  }
  __syncthreads();
  for (int base = 0; base < B; base += 1024) {
    const int s = base + tid;
    int n = 0;
    if (s < B) {
      int c = ctx_lens[s];
      if (c < 0 || c > max_ctx || c > max_blocks * bs) {
        record_error(PA_ERR_DEVICE_BOUNDS);
        c = 0;
      }
      n = c > 0 ? (c + S - 1) / S : 1;
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
}

// ------------------------------------------------------------ main kernel
template <int CK, bool kQBF16, int D, int BS>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const DecodeArgs a) {
  using C = DecodeCfg<CK, D, BS>;
  constexpr bool kMmaBF16 = C::kMmaBF16;
  constexpr int kStages = C::kStages;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_item;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;    // fragment row group
  const int tig = lane & 3;   // thread in group

  uint8_t* const wbase = smem + kBarrierBytes + warp * C::kWarpBytes;
  const uint32_t wbase_s = smem_addr(wbase);
  const uint32_t bar0 = smem_addr(smem) + warp * kStages * 8;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
  }
  __syncthreads();

  const int total = *a.total;
  const bool split_mode = a.split_tokens < a.max_ctx;
  uint32_t n_issued = 0, n_consumed = 0;  // warp-uniform ring counters
  bool failed = false;                    // a wait timed out: stop issuing / computing

  for (;;) {
    if (threadIdx.x == 0) s_item = atomicAdd(a.counter, 1);
    __syncthreads();
    const int item = s_item;
    if (item >= total) break;

    // ---- item -> (sequence, range, kv head)
    const int kvh = item % a.hkv;
    const int r = item / a.hkv;
    int seq, split, nsplit;
    if (split_mode) {
      int lo = 0, hi = a.num_seqs;  // largest seq with seq_off[seq] <= r
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (a.seq_off[mid] <= r) lo = mid; else hi = mid;
      }
      seq = lo;
      split = r - a.seq_off[seq];
      nsplit = a.seq_off[seq + 1] - a.seq_off[seq];
    } else {
      seq = r;
      split = 0;
      nsplit = 1;
    }
    int ctx = a.context_lens[seq];
    if (ctx < 0 || ctx > a.max_ctx || ctx > a.max_blocks * BS) ctx = 0;  // recorded by plan_kernel
    const int t0 = split * a.split_tokens;
    const int t1 = min(ctx, t0 + a.split_tokens);
    const int jb0 = t0 / BS;
    const int nblk = t1 > t0 ? (t1 + BS - 1) / BS - jb0 : 0;
    const int nb_w = nblk > warp ? (nblk - warp + kDecodeWarps - 1) / kDecodeWarps : 0;
    const int32_t* table = a.block_tables + static_cast<int64_t>(seq) * a.max_blocks;
    const int h0 = kvh * a.group;

    // ---- issue the loads of the warp's i-th block of this item
    auto issue = [&](int i) {
      const int j = jb0 + warp + i * kDecodeWarps;
      const int st = n_issued % kStages;
      const uint32_t bar = bar0 + 8 * st;
      const uint32_t sK = wbase_s + st * C::kStageBytes;
      uint8_t* const gK = wbase + st * C::kStageBytes;
      const int phys = table[j];
      const bool ok = phys >= 0 && phys < a.num_blocks;
      if (!ok && lane == 0) record_error(PA_ERR_DEVICE_BOUNDS);
      const int nv = ok ? min(BS, t1 - j * BS) : 0;  // valid token rows
      fence_proxy_async_smem();  // earlier generic reads/writes of this stage first
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(bar, 2u * nv * C::kRowBytes);
      __syncwarp();
      const int64_t row0 = (static_cast<int64_t>(ok ? phys : 0) * BS * a.hkv + kvh);
#pragma unroll
      for (int rr = lane; rr < 2 * BS; rr += 32) {
        const bool isv = rr >= BS;
        const int tok = isv ? rr - BS : rr;
        const uint32_t dst = sK + rr * C::kRowStride;
        if (tok < nv) {
          const uint8_t* src = (isv ? a.v_pool : a.k_pool) +
                               (row0 + static_cast<int64_t>(tok) * a.hkv) * C::kRowBytes;
          bulk_copy_g2s(dst, src, C::kRowBytes, bar);
        } else {  // rows past the sequence: zeros, so masked tokens add 0 * 0
          uint4* z = reinterpret_cast<uint4*>(gK + rr * C::kRowStride);
#pragma unroll
          for (int c = 0; c < C::kRowBytes / 16; ++c) z[c] = make_uint4(0, 0, 0, 0);
        }
      }
      __syncwarp();
      ++n_issued;
    };

    // ---- query fragments (B operand of S^T = K Q^T): rows = dims, cols = heads
    uint32_t qf[C::kDimTiles][2];
    {
      const bool hv = g < a.group;
      const uint16_t* qrow = reinterpret_cast<const uint16_t*>(a.q) +
                             (static_cast<int64_t>(seq) * a.hq + h0 + (hv ? g : 0)) * D;
#pragma unroll
      for (int ks = 0; ks < C::kDimTiles; ++ks) {
        if constexpr (CK == kCacheE4M3) {
          // dims 16ks + 4tig .. +3 (the order ldmatrix gives 8-bit K rows)
          const uint2 w = *reinterpret_cast<const uint2*>(qrow + ks * 16 + 4 * tig);
          const float f0 = to_float<kQBF16>(w.x & 0xffff), f1 = to_float<kQBF16>(w.x >> 16);
          const float f2 = to_float<kQBF16>(w.y & 0xffff), f3 = to_float<kQBF16>(w.y >> 16);
          qf[ks][0] = hv ? pack_f16x2(f0, f1) : 0u;
          qf[ks][1] = hv ? pack_f16x2(f2, f3) : 0u;
        } else {
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

    if (!failed) {
      const int pro = min(kStages, nb_w);
      for (int i = 0; i < pro; ++i) issue(i);
    }

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
      if (!failed) {
        const int j = jb0 + warp + i * kDecodeWarps;
        const int tbase = j * BS;
        const uint32_t sK = wbase_s + st * C::kStageBytes;
        const uint32_t sV = sK + BS * C::kRowStride;

        // ---- S^T = K Q^T  (rows: tokens, cols: packed heads)
        float s[C::kTokTiles][4];
#pragma unroll
        for (int mt = 0; mt < C::kTokTiles; ++mt) {
          float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
          if constexpr (CK == kCacheE4M3) {
            const int li = lane >> 3;
            const int tok = mt * 16 + (lane & 7) + (li & 1) * 8;
#pragma unroll
            for (int cp = 0; cp < C::kDimTiles / 2; ++cp) {
              uint32_t r0, r1, r2, r3;
              ldsm_x4(sK + tok * C::kRowStride + (2 * cp + (li >> 1)) * 16, r0, r1, r2, r3);
              const uint32_t a0[4] = {e4m3x2_to_f16x2(r0 & 0xffff), e4m3x2_to_f16x2(r1 & 0xffff),
                                      e4m3x2_to_f16x2(r0 >> 16), e4m3x2_to_f16x2(r1 >> 16)};
              const uint32_t a1[4] = {e4m3x2_to_f16x2(r2 & 0xffff), e4m3x2_to_f16x2(r3 & 0xffff),
                                      e4m3x2_to_f16x2(r2 >> 16), e4m3x2_to_f16x2(r3 >> 16)};
              mma_16816<false>(s0, a0, qf[2 * cp][0], qf[2 * cp][1]);
              mma_16816<false>(s1, a1, qf[2 * cp + 1][0], qf[2 * cp + 1][1]);
            }
          } else {
            const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const uint32_t base = sK + row * C::kRowStride + (lane >> 4) * 16;
#pragma unroll
            for (int ks = 0; ks < C::kDimTiles; ++ks) {
              uint32_t af[4];
              ldsm_x4(base + ks * 32, af[0], af[1], af[2], af[3]);
              if (ks & 1) mma_16816<kMmaBF16>(s1, af, qf[ks][0], qf[ks][1]);
              else mma_16816<kMmaBF16>(s0, af, qf[ks][0], qf[ks][1]);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = tbase + mt * 16 + g + (e >> 1) * 8;
            const float x = (s0[e] + s1[e]) * a.sl2;
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
        uint32_t pb[C::kTokTiles][2];
        constexpr bool kPBF16 = (CK == kCacheBF16);
#pragma unroll
        for (int mt = 0; mt < C::kTokTiles; ++mt) {
          pb[mt][0] = movmatrix_trans(pack2<kPBF16>(s[mt][0], s[mt][1]));
          pb[mt][1] = movmatrix_trans(pack2<kPBF16>(s[mt][2], s[mt][3]));
        }

        // ---- O^T += V^T P^T  (rows: dims, cols: packed heads)
        if constexpr (CK == kCacheE4M3) {
          const int li = lane >> 3;
#pragma unroll
          for (int mt = 0; mt < C::kTokTiles; ++mt) {
            const int tok = mt * 16 + (lane & 7) + (li & 1) * 8;
#pragma unroll
            for (int cp = 0; cp < C::kDimTiles / 2; ++cp) {
              uint32_t r0, r1, r2, r3;
              ldsm_x4_trans(sV + tok * C::kRowStride + (2 * cp + (li >> 1)) * 16, r0, r1, r2, r3);
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
          }
        } else {
          const int li = lane >> 3;
#pragma unroll
          for (int mt = 0; mt < C::kTokTiles; ++mt) {
            const int tok = mt * 16 + (lane & 7) + (li >> 1) * 8;
            const uint32_t base = sV + tok * C::kRowStride + (li & 1) * 16;
#pragma unroll
            for (int dt = 0; dt < C::kDimTiles; ++dt) {
              uint32_t af[4];
              ldsm_x4_trans(base + dt * 32, af[0], af[1], af[2], af[3]);
              mma_16816<kMmaBF16>(acc[dt], af, pb[mt][0], pb[mt][1]);
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
      const int units = a.group * (D / kVec);
      for (int u = threadIdx.x; u < units; u += kDecodeThreads) {
        const int h = u / (D / kVec);
        const int d0 = (u % (D / kVec)) * kVec;
        float mw[kDecodeWarps];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
          const float* scr = reinterpret_cast<const float*>(smem + kBarrierBytes + w * C::kWarpBytes);
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
            const float* scr = reinterpret_cast<const float*>(smem + kBarrierBytes + w * C::kWarpBytes);
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
    __syncthreads();  // scratch (= stage memory) is free again
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

// ------------------------------------------------------------ merge kernel
// out[s, h, :] = sum_i w_i o_i / sum_i w_i with w_i = 2^(lse_i - max lse) over
// the ranges i of sequence s; sequences with one range were written by the
// main kernel directly.
template <bool kOutBF16>
__global__ void __launch_bounds__(128) merge_kernel(void* __restrict__ out,
                                                    const float* __restrict__ lse_part,
                                                    const float* __restrict__ o_part,
                                                    const int32_t* __restrict__ seq_off, int hq,
                                                    int D) {
  const int seq = blockIdx.y;
  const int base = seq_off[seq];
  const int n = seq_off[seq + 1] - base;
  if (n <= 1) return;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int per_head = D / 4;
  const int h = e / per_head;
  if (h >= hq) return;
  const int d0 = (e % per_head) * 4;
  float M = -INFINITY;
  for (int i = 0; i < n; ++i) M = fmaxf(M, lse_part[static_cast<int64_t>(base + i) * hq + h]);
  float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f, W = 0.f;
  if (M != -INFINITY) {
    for (int i = 0; i < n; ++i) {
      const int64_t pi = static_cast<int64_t>(base + i) * hq + h;
      const float w = fast_exp2(lse_part[pi] - M);
      const float4 x = *reinterpret_cast<const float4*>(o_part + pi * D + d0);
      W += w;
      o0 += w * x.x; o1 += w * x.y; o2 += w * x.z; o3 += w * x.w;
    }
    const float inv = 1.f / W;
    o0 *= inv; o1 *= inv; o2 *= inv; o3 *= inv;
  }
  uint2 pk;
  pk.x = static_cast<uint32_t>(from_float<kOutBF16>(o0)) | (static_cast<uint32_t>(from_float<kOutBF16>(o1)) << 16);
  pk.y = static_cast<uint32_t>(from_float<kOutBF16>(o2)) | (static_cast<uint32_t>(from_float<kOutBF16>(o3)) << 16);
  *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(out) + (static_cast<int64_t>(seq) * hq + h) * D + d0) = pk;
}

}  // namespace pa
