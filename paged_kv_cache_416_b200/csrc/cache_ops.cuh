// Cache maintenance kernels: the slot-mapping scatter of new keys/values,
// the copy-on-write block copy, the block swap between the device pool and
// host memory, and the chained block hashes used for prefix caching.
//
// Both are pure data movement in 16-byte vectors (HBM-bound, and at decode
// sizes launch-bound).  "PagedAttention" (Ultralytics glossary): token `pos`
// of a request is stored at key_pool[block_table[pos // bs], pos % bs]
// (section "Sayfalama Nasil Calisir", PyTorch sketch); a block that other
// sequences still use is copied before it is written (section "Diziler
// Arasinda Bloklari Paylasma").
#pragma once

#include "common.cuh"

namespace pa {

// One thread moves one 16-byte vector of one (token, kv head) row of K or V.
// 16-bit cache: the words are copied unchanged.  kFP8: the thread reads 8
// 16-bit inputs (16 bytes) and stores 8 e4m3 codes (8 bytes), each
// e4m3_rne_satfinite(fp32(x) / scale) with an IEEE fp32 division.
template <bool kFP8, bool kInBF16>
__global__ void __launch_bounds__(256) write_kv_kernel(
    const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const int64_t* __restrict__ slots, int num_tokens, uint8_t* __restrict__ k_pool,
    uint8_t* __restrict__ v_pool, int64_t num_slots, int hkv, int D, float k_scale,
    float v_scale) {
  const int vec_per_row = D / 8;  // 8 input elements per vector
  const int64_t per_tensor = static_cast<int64_t>(num_tokens) * hkv * vec_per_row;
  const int64_t total = 2 * per_tensor;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool isv = i >= per_tensor;
    const int64_t e = isv ? i - per_tensor : i;
    const int c = static_cast<int>(e % vec_per_row);
    const int64_t th = e / vec_per_row;  // token * hkv + head
    const int h = static_cast<int>(th % hkv);
    const int64_t t = th / hkv;
    const int64_t slot = slots[t];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      record_error(PA_ERR_DEVICE_BOUNDS);
      continue;
    }
    const uint4 x = *reinterpret_cast<const uint4*>((isv ? v : k) + th * D + c * 8);
    const int64_t dst_elem = (slot * hkv + h) * D + c * 8;
    uint8_t* pool = isv ? v_pool : k_pool;
    if constexpr (!kFP8) {
      *reinterpret_cast<uint4*>(pool + dst_elem * 2) = x;
    } else {
      const float s = isv ? v_scale : k_scale;
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
      uint32_t outw[2];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const float f0 = __fdiv_rn(to_float<kInBF16>(w[2 * p] & 0xffff), s);
        const float f1 = __fdiv_rn(to_float<kInBF16>(w[2 * p] >> 16), s);
        const float f2 = __fdiv_rn(to_float<kInBF16>(w[2 * p + 1] & 0xffff), s);
        const float f3 = __fdiv_rn(to_float<kInBF16>(w[2 * p + 1] >> 16), s);
        outw[p] = static_cast<uint32_t>(f32x2_to_e4m3x2(f0, f1)) |
                  (static_cast<uint32_t>(f32x2_to_e4m3x2(f2, f3)) << 16);
      }
      *reinterpret_cast<uint2*>(pool + dst_elem) = make_uint2(outw[0], outw[1]);
    }
  }
}

// Grid (x: pair, y: CTAs per pair).  Each pair copies block_bytes of K and of
// V from src to dst in 16-byte vectors.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint8_t* __restrict__ k_pool,
                                                          uint8_t* __restrict__ v_pool,
                                                          const int64_t* __restrict__ pairs,
                                                          int64_t num_blocks,
                                                          int64_t block_bytes) {
  const int64_t p = blockIdx.x;
  const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
    if (blockIdx.y == 0 && threadIdx.x == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    return;
  }
  const int64_t nvec = block_bytes / 16;
  const uint4* ks = reinterpret_cast<const uint4*>(k_pool + src * block_bytes);
  const uint4* vs = reinterpret_cast<const uint4*>(v_pool + src * block_bytes);
  uint4* kd = reinterpret_cast<uint4*>(k_pool + dst * block_bytes);
  uint4* vd = reinterpret_cast<uint4*>(v_pool + dst * block_bytes);
  for (int64_t i = blockIdx.y * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.y) * blockDim.x) {
    const uint4 a = ks[i];
    const uint4 b = vs[i];
    kd[i] = a;
    vd[i] = b;
  }
}

// Block swap between two pools of the same block shape, either of which may
// be host memory mapped into the device's address space (pinned, unified
// addressing): for each pair p, dst[pairs[p][1]] = src[pairs[p][0]] for K and
// V.  Grid (x: pair, y: CTAs per pair); each thread keeps 4 independent
// 16-byte loads in flight per tensor, since host memory sits behind the
// high-latency host link.
__global__ void __launch_bounds__(256) swap_blocks_kernel(
    const uint8_t* __restrict__ src_k, const uint8_t* __restrict__ src_v,
    uint8_t* __restrict__ dst_k, uint8_t* __restrict__ dst_v, const int64_t* __restrict__ pairs,
    int64_t src_blocks, int64_t dst_blocks, int64_t block_bytes) {
  const int64_t p = blockIdx.x;
  const int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
  if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
    if (blockIdx.y == 0 && threadIdx.x == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    return;
  }
  const int64_t nvec = block_bytes / 16;
  const uint4* ks = reinterpret_cast<const uint4*>(src_k + src * block_bytes);
  const uint4* vs = reinterpret_cast<const uint4*>(src_v + src * block_bytes);
  uint4* kd = reinterpret_cast<uint4*>(dst_k + dst * block_bytes);
  uint4* vd = reinterpret_cast<uint4*>(dst_v + dst * block_bytes);
  const int64_t stride = static_cast<int64_t>(gridDim.y) * blockDim.x;
  constexpr int kUnroll = 4;
  for (int64_t i0 = blockIdx.y * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < nvec;
       i0 += kUnroll * stride) {
    uint4 a[kUnroll], b[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < nvec) {
        a[u] = ks[i];
        b[u] = vs[i];
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < nvec) {
        kd[i] = a[u];
        vd[i] = b[u];
      }
    }
  }
}

// ------------------------------------------------------------ block hashes
// 64-bit FNV-1a (Fowler / Noll / Vo): per byte, xor then multiply by the
// prime, mod 2^64, from the offset basis.
constexpr unsigned long long kFnvOffset = 0xcbf29ce484222325ull;
constexpr uint32_t kFnvPrimeLow = 0x1b3u;  // the prime is 2^40 + 0x1b3

// One FNV-1a byte step on the hash's 32-bit halves (lo, hi): with
// l = lo ^ byte, (l + hi 2^32)(2^40 + 0x1b3) mod 2^64 has low word
// low32(l 0x1b3) and high word high32(l 0x1b3) + hi 0x1b3 + (l << 8), all
// mod 2^32 (hi 2^72 vanishes mod 2^64).  One wide multiply on the low word's
// path instead of a full 64 x 64-bit product.
__device__ __forceinline__ void fnv1a_byte(uint32_t& lo, uint32_t& hi, uint32_t byte) {
  const uint32_t l = lo ^ byte;
  const unsigned long long p = static_cast<unsigned long long>(l) * kFnvPrimeLow;
  lo = static_cast<uint32_t>(p);
  hi = static_cast<uint32_t>(p >> 32) + hi * kFnvPrimeLow + (l << 8);
}

// FNV-1a over the 4 little-endian bytes of w
__device__ __forceinline__ void fnv1a_u32(uint32_t& lo, uint32_t& hi, uint32_t w) {
#pragma unroll
  for (int i = 0; i < 4; ++i) fnv1a_byte(lo, hi, (w >> (8 * i)) & 0xffu);
}

constexpr int kHashChunk = 256;  // blocks hashed per pass (one per thread)

// One CTA per sequence, over its full blocks in chunks of 256.  Phase 1 (all
// threads): inner_j = FNV-1a over the 4 little-endian bytes of each of block
// j's token ids, into shared memory.  Phase 2 (one thread, in order): hash_j
// = FNV-1a over hash_{j-1} then inner_j (8 little-endian bytes each),
// hash_{-1} = 0.  Entries of blocks that are not full are 0.
__global__ void __launch_bounds__(kHashChunk) hash_blocks_kernel(
    const int32_t* __restrict__ tokens, int64_t token_stride, const int32_t* __restrict__ num_tokens,
    int bs, unsigned long long* __restrict__ hashes, int max_blocks) {
  __shared__ uint32_t s_lo[kHashChunk], s_hi[kHashChunk];
  const int s = blockIdx.x;
  int n = num_tokens[s];
  if (n < 0 || n > token_stride) {
    if (threadIdx.x == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    n = n < 0 ? 0 : static_cast<int>(token_stride);
  }
  int full = n / bs;
  if (full > max_blocks) {
    if (threadIdx.x == 0) record_error(PA_ERR_DEVICE_BOUNDS);
    full = max_blocks;
  }
  const int32_t* row = tokens + static_cast<int64_t>(s) * token_stride;
  unsigned long long* out = hashes + static_cast<int64_t>(s) * max_blocks;
  for (int j = full + static_cast<int>(threadIdx.x); j < max_blocks; j += blockDim.x) out[j] = 0;
  constexpr uint32_t kOffLo = static_cast<uint32_t>(kFnvOffset);
  constexpr uint32_t kOffHi = static_cast<uint32_t>(kFnvOffset >> 32);
  uint32_t plo = 0, phi = 0;  // the parent hash (thread 0)
  for (int j0 = 0; j0 < full; j0 += kHashChunk) {  // the same trip count in every thread
    const int j = j0 + static_cast<int>(threadIdx.x);
    if (j < full) {
      uint32_t lo = kOffLo, hi = kOffHi;
      for (int t = 0; t < bs; ++t) fnv1a_u32(lo, hi, static_cast<uint32_t>(row[static_cast<int64_t>(j) * bs + t]));
      s_lo[threadIdx.x] = lo;
      s_hi[threadIdx.x] = hi;
    }
    __syncthreads();  // the chunk's inner hashes are visible to thread 0
    if (threadIdx.x == 0) {
      const int m = min(kHashChunk, full - j0);
      for (int i = 0; i < m; ++i) {
        const uint32_t ilo = s_lo[i], ihi = s_hi[i];
        uint32_t lo = kOffLo, hi = kOffHi;
        fnv1a_u32(lo, hi, plo);
        fnv1a_u32(lo, hi, phi);
        fnv1a_u32(lo, hi, ilo);
        fnv1a_u32(lo, hi, ihi);
        plo = lo;
        phi = hi;
        out[j0 + i] = (static_cast<unsigned long long>(hi) << 32) | lo;
      }
    }
    __syncthreads();  // the chunk's slots are free again
  }
}

}  // namespace pa
