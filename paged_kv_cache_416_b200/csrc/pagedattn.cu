// Host side of libpagedattn.so: argument validation, kernel selection,
// workspace layout and the C entry points declared in include/pagedattn.h.
#include <cuda.h>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "cache_ops.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "cascade.cuh"

namespace {

thread_local char g_msg[1024] = "";

pa_status fail(pa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

pa_status ok() {
  g_msg[0] = '\0';
  return PA_OK;
}

pa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;

int current_device(int* dev) {
  const cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess || *dev < 0 || *dev >= kMaxDevices) return -1;
  return 0;
}

// SM count of the current device (cached per device; host threads that make
// their first call at once may both query it and store the same value).
int device_sms(int dev) {
  static std::atomic<int> cache[kMaxDevices] = {};
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 1;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// Resident CTAs per SM of a persistent kernel on device `dev`, cached per
// (kernel, device) in `occ`.  The first call on a device raises the kernel's
// dynamic shared-memory limit; concurrent first calls repeat that idempotent
// step and store the same value.
template <typename Kern>
pa_status resident_ctas(std::atomic<int>* occ, int dev, Kern kern, int threads, int smem_bytes,
                        const char* what, int* out) {
  int n = occ[dev].load(std::memory_order_acquire);
  if (n == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem_bytes);
    if (e != cudaSuccess) return cuda_fail(e, what);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem_bytes);
    if (e != cudaSuccess) return cuda_fail(e, what);
    n = n > 0 ? n : 1;
    occ[dev].store(n, std::memory_order_release);
  }
  *out = n;
  return PA_OK;
}

int elem_bytes(pa_dtype t) { return t == PA_FP8_E4M3 ? 1 : 2; }

bool valid_dtype(int t) { return t == PA_F16 || t == PA_BF16 || t == PA_FP8_E4M3; }

bool cache_shape_ok(int32_t num_blocks, int32_t bs, int32_t hkv, int32_t d) {
  return num_blocks > 0 && (bs == 16 || bs == 32) && hkv > 0 && (d == 64 || d == 128);
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }

// ------------------------------------------------------------- split rule
// Persistent CTAs the split rule plans for (two per SM of a 148-SM B200);
// fixed so that the split, and so the rounding of every result, depends on
// the call's arguments only and not on the device it runs on.
constexpr int64_t kPlanCtas = 296;
// query heads per kv head pa_decode accepts: column groups of kMaxGroup heads,
// each its own work item over the kv head's blocks
constexpr int kMaxQHeadsPerKv = 64;
int32_t col_groups(int32_t hq, int32_t hkv) {
  return hkv > 0 ? std::max<int32_t>(1, static_cast<int32_t>(cdiv(hq / hkv, pa::kMaxGroup))) : 1;
}
// SMs the device-side lengthening of the automatic split plans for (a
// B200's 148), fixed for the same reason as kPlanCtas; with the instance's
// resident CTAs per SM it sets the work items the planning kernel aims at:
// 15/16 of the persistent grid.  On the FP8 long-tail batch (128 sequences,
// 177,982 tokens, 32/8 heads, e4m3) the best range lengths were 2,560 tokens
// at bs 16 (592 CTAs: 74.1 us, against 76.5 at 2,048 and 75.6 at 3,072) and
// 3,584 at bs 32 (444 CTAs: 70.2 us, against 74.5 at 2,048), i.e. about 0.93
// of the grid's CTAs in (range, kv head) items.
constexpr int64_t kPlanSms = 148;
constexpr int64_t kMinSplit = 256;        // shortest range worth its partial
constexpr int64_t kLongContext = 4096;    // above this, cap ranges ...
constexpr int64_t kLongSplit = 1024;      // ... at this many tokens

int32_t choose_split(int32_t B, int32_t hkv, int32_t bs, int32_t max_ctx, int32_t user) {
  // at most kMaxRanges ranges per sequence, whatever was asked for
  const int64_t floor_s = std::max<int64_t>(bs, cdiv(max_ctx, pa::kMaxRanges));
  if (user > 0) return static_cast<int32_t>(round_up(std::max<int64_t>(user, floor_s), bs));
  if (max_ctx <= 0) return bs;
  const int64_t units = static_cast<int64_t>(B) * hkv;
  // enough ranges for two waves of persistent CTAs ...
  int64_t s = cdiv(units * max_ctx, 2 * kPlanCtas);
  s = std::max<int64_t>(kMinSplit, std::min<int64_t>(max_ctx, s));
  // ... and no single range much longer than the typical one when lengths
  // can spread far (long contexts): the longest sequence is cut up
  if (max_ctx > kLongContext) s = std::min<int64_t>(s, kLongSplit);
  return static_cast<int32_t>(round_up(std::max(s, floor_s), bs));
}

// Workspace of one decode call: work counter and item total, per-sequence
// range offsets [B + 1], the work order [ranges] of int4, and when contexts
// are split, arrival counters [B * Hkv], fp32 lse [ranges * Hq] and fp32
// partial outputs [ranges * Hq * D].
struct WsLayout {
  size_t counter = 0, total = 4, split = 8, seq_off = 256, order = 0, arrived = 0, lse = 0, o = 0,
         bytes = 0;
  bool is_split = false;  // contexts may be cut into ranges (partials allocated)
  int64_t ranges = 0;     // upper bound on (sequence, range) pairs
};

WsLayout ws_layout(int32_t B, int32_t hq, int32_t hkv, int32_t D, int32_t max_ctx, int32_t S) {
  WsLayout w;
  w.is_split = S < max_ctx;
  w.ranges = w.is_split ? static_cast<int64_t>(B) * cdiv(max_ctx, S) : B;
  w.order = w.seq_off + static_cast<size_t>(round_up(static_cast<int64_t>(B + 1) * 4, 256));
  w.arrived = w.order + static_cast<size_t>(round_up(w.ranges * 16, 256));
  if (!w.is_split) {
    w.lse = w.o = w.arrived;
    w.bytes = w.arrived;
    return w;
  }
  w.lse = w.arrived + static_cast<size_t>(round_up(static_cast<int64_t>(B) * hkv * 4, 256));
  w.o = w.lse + static_cast<size_t>(round_up(w.ranges * hq * 4, 256));
  w.bytes = w.o + static_cast<size_t>(w.ranges * hq * D * 4);
  return w;
}

// Shared-prefix (cascade) decode workspace: work counter and range count,
// then seen [B], chunk members [B], chunk descriptors [2B] int4, the ranges
// [slots] int4, arrival counters [B * Hkv], and the partials: fp32 lse
// [slots * Hkv * 16] and fp32 outputs [slots * Hkv * 16 * D].  Slots are
// bounded through the shortest range r_floor: a chunk takes at most
// P / R + 1 shared ranges and n_i / R + 1 per member, so all chunks together
// at most B * max_blocks / r_floor + 2 B.
struct CascadeWs {
  size_t counter = 0, total = 4, seen = 256, chunk_seqs = 0, chunks = 0, ranges = 0, arrived = 0,
         lse = 0, o = 0, bytes = 0;
  int32_t r_floor = 1;
  int64_t slots = 0;
};

CascadeWs cascade_ws_layout(int32_t B, int32_t hkv, int32_t D, int32_t bs, int32_t max_ctx,
                            int32_t split_tokens) {
  CascadeWs w;
  const int64_t max_nb = std::max<int64_t>(1, cdiv(max_ctx, bs));
  const int64_t auto_floor = cdiv(static_cast<int64_t>(B) * max_nb * hkv, 4 * pa::kCascadeTargetItems);
  const int64_t user_floor = split_tokens > 0 ? cdiv(split_tokens, bs) : 1;
  w.r_floor = static_cast<int32_t>(std::max<int64_t>(std::max<int64_t>(4, auto_floor), user_floor));
  w.slots = cdiv(static_cast<int64_t>(B) * max_nb, w.r_floor) + 2 * static_cast<int64_t>(B);
  const size_t arr = static_cast<size_t>(round_up(static_cast<int64_t>(B) * 4, 256));
  w.chunk_seqs = w.seen + arr;
  w.chunks = w.chunk_seqs + arr;
  w.ranges = w.chunks + static_cast<size_t>(round_up(static_cast<int64_t>(B) * 32, 256));
  w.arrived = w.ranges + static_cast<size_t>(round_up(w.slots * 16, 256));
  w.lse = w.arrived + static_cast<size_t>(round_up(static_cast<int64_t>(B) * hkv * 4, 256));
  w.o = w.lse + static_cast<size_t>(round_up(w.slots * hkv * pa::kCascadeRows * 4, 256));
  w.bytes = w.o + static_cast<size_t>(w.slots * hkv * pa::kCascadeRows * D * 4);
  return w;
}

// --------------------------------------------------------- tensor maps
// cuTensorMapEncodeTiled is a driver entry point; it is fetched through the
// runtime so the library needs no link-time dependency on libcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && p != nullptr) {
      f = reinterpret_cast<EncodeTiledFn>(p);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

// Tensor map over a pool [N, bs, Hkv, D] viewed as 5-D bytes
// (x, token, half, kv head, block) = (R, bs, D*e/R, Hkv, N) with R = min(128,
// D*e) bytes per swizzle row; one box = the bs token rows of one kv head of
// one block, landing in shared memory as [half][token][R] with the R-byte
// swizzle (128B or 64B).  Must match DecodeCfg / tile_off in decode.cuh.
// With one_half the box is a single dim half (the prefill kernel places the
// halves of consecutive blocks of K in separate K-major tiles).
pa_status encode_pool_map(CUtensorMap* map, const void* pool, int32_t num_blocks, int32_t bs,
                          int32_t hkv, int32_t head_dim, int32_t elem, bool one_half = false) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (fn == nullptr) return fail(PA_ERR_CUDA, "pa_decode: cuTensorMapEncodeTiled unavailable");
  const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * elem;
  const cuuint64_t R = row >= 128 ? 128 : 64;
  const cuuint64_t halves = row / R;
  const cuuint64_t dims[5] = {R, static_cast<cuuint64_t>(bs), halves, static_cast<cuuint64_t>(hkv),
                              static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t strides[4] = {hkv * row, R, row, static_cast<cuuint64_t>(bs) * hkv * row};
  const cuuint32_t box[5] = {static_cast<cuuint32_t>(R), static_cast<cuuint32_t>(bs),
                             static_cast<cuuint32_t>(one_half ? 1 : halves), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(pool), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        R == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(PA_ERR_CUDA, "pa_decode: cuTensorMapEncodeTiled failed (%d) for the pool", (int)r);
  return PA_OK;
}

// ------------------------------------------------------ decode dispatch
// Launch a persistent attention kernel behind its planning kernel with
// programmatic stream serialization: its CTAs are scheduled, initialise their
// barriers and prefetch the tensor maps while the plan finishes, then wait in
// grid_dependency_wait for the plan's writes.
template <typename Args>
cudaError_t launch_behind_plan(void (*kern)(Args), unsigned grid, int threads, int smem_bytes,
                               cudaStream_t stream, const Args& args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args);
}

// Resident CTAs per SM of one decode kernel instance (cached per device).
template <int CK, bool kQBF16, int D, int BS>
pa_status decode_occupancy(int dev, int* per_sm) {
  using C = pa::DecodeCfg<CK, D, BS>;
  static std::atomic<int> occ[kMaxDevices] = {};
  return resident_ctas(occ, dev, pa::decode_kernel<CK, kQBF16, D, BS>, pa::kDecodeThreads,
                       C::kSmemBytes, "pa_decode: kernel set-up", per_sm);
}

template <int CK, bool kQBF16, int D, int BS>
pa_status launch_decode_main(const pa::DecodeArgs& args, int64_t items_upper, int dev,
                             cudaStream_t stream) {
  using C = pa::DecodeCfg<CK, D, BS>;
  auto kern = pa::decode_kernel<CK, kQBF16, D, BS>;
  int per_sm = 0;
  const pa_status os = decode_occupancy<CK, kQBF16, D, BS>(dev, &per_sm);
  if (os != PA_OK) return os;
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(items_upper, static_cast<int64_t>(device_sms(dev)) * per_sm));
  const cudaError_t e = launch_behind_plan(kern, static_cast<unsigned>(grid), pa::kDecodeThreads,
                                           C::kSmemBytes, stream, args);
  if (e != cudaSuccess) return cuda_fail(e, "pa_decode launch");
  return PA_OK;
}

template <int CK, bool kQBF16>
pa_status occupancy_shape(int D, int BS, int dev, int* per_sm) {
  if (D == 128 && BS == 16) return decode_occupancy<CK, kQBF16, 128, 16>(dev, per_sm);
  if (D == 128 && BS == 32) return decode_occupancy<CK, kQBF16, 128, 32>(dev, per_sm);
  if (D == 64 && BS == 16) return decode_occupancy<CK, kQBF16, 64, 16>(dev, per_sm);
  if (D == 64 && BS == 32) return decode_occupancy<CK, kQBF16, 64, 32>(dev, per_sm);
  return fail(PA_ERR_SHAPE, "head_dim %d / block_size %d not supported", D, BS);
}

template <int CK, bool kQBF16>
pa_status dispatch_shape(const pa::DecodeArgs& a, int D, int BS, int64_t items, int dev,
                         cudaStream_t st) {
  if (D == 128 && BS == 16) return launch_decode_main<CK, kQBF16, 128, 16>(a, items, dev, st);
  if (D == 128 && BS == 32) return launch_decode_main<CK, kQBF16, 128, 32>(a, items, dev, st);
  if (D == 64 && BS == 16) return launch_decode_main<CK, kQBF16, 64, 16>(a, items, dev, st);
  if (D == 64 && BS == 32) return launch_decode_main<CK, kQBF16, 64, 32>(a, items, dev, st);
  return fail(PA_ERR_SHAPE, "head_dim %d / block_size %d not supported", D, BS);
}

template <int CK, bool kQBF16, int D, int BS>
pa_status launch_cascade(const pa::CascadeArgs& args, int64_t items_upper, int dev,
                         cudaStream_t stream) {
  using C = pa::DecodeCfg<CK, D, BS>;
  auto kern = pa::cascade_kernel<CK, kQBF16, D, BS>;
  static std::atomic<int> occ[kMaxDevices] = {};
  int per_sm = 0;
  const pa_status os = resident_ctas(occ, dev, kern, pa::kDecodeThreads, C::kSmemBytes,
                                     "pa_decode_shared_prefix: kernel set-up", &per_sm);
  if (os != PA_OK) return os;
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(items_upper, static_cast<int64_t>(device_sms(dev)) * per_sm));
  const cudaError_t e = launch_behind_plan(kern, static_cast<unsigned>(grid), pa::kDecodeThreads,
                                           C::kSmemBytes, stream, args);
  if (e != cudaSuccess) return cuda_fail(e, "pa_decode_shared_prefix launch");
  return PA_OK;
}

template <int CK, bool kQBF16>
pa_status dispatch_cascade(const pa::CascadeArgs& a, int D, int BS, int64_t items, int dev,
                           cudaStream_t st) {
  if (D == 128 && BS == 16) return launch_cascade<CK, kQBF16, 128, 16>(a, items, dev, st);
  if (D == 128 && BS == 32) return launch_cascade<CK, kQBF16, 128, 32>(a, items, dev, st);
  if (D == 64 && BS == 16) return launch_cascade<CK, kQBF16, 64, 16>(a, items, dev, st);
  if (D == 64 && BS == 32) return launch_cascade<CK, kQBF16, 64, 32>(a, items, dev, st);
  return fail(PA_ERR_SHAPE, "head_dim %d / block_size %d not supported", D, BS);
}

// Copy n indices to the host (debug checks only).
template <typename T>
pa_status fetch(std::vector<T>& h, const T* d, size_t n, cudaStream_t st, const char* what) {
  h.resize(n);
  if (n == 0) return PA_OK;
  cudaError_t e = cudaMemcpyAsync(h.data(), d, n * sizeof(T), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return PA_OK;
}

}  // namespace

extern "C" {

const char* pa_last_error(void) { return g_msg; }

pa_status pa_write_kv(const void* k, const void* v, pa_dtype in_dtype,
                      const int64_t* slot_mapping, int32_t num_tokens, void* k_pool,
                      void* v_pool, pa_dtype cache_dtype, int32_t num_blocks,
                      int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                      float k_scale, float v_scale, pa_stream_t stream) {
  if (!valid_dtype(in_dtype) || !valid_dtype(cache_dtype))
    return fail(PA_ERR_DTYPE, "pa_write_kv: unknown dtype");
  if (in_dtype == PA_FP8_E4M3)
    return fail(PA_ERR_DTYPE, "pa_write_kv: inputs must be f16 or bf16");
  if (cache_dtype != PA_FP8_E4M3 && cache_dtype != in_dtype)
    return fail(PA_ERR_DTYPE, "pa_write_kv: a 16-bit cache must have the input dtype");
  if (num_tokens < 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
    return fail(PA_ERR_SHAPE, "pa_write_kv: unsupported sizes (tokens %d, blocks %d, bs %d, "
                "heads %d, dim %d)", num_tokens, num_blocks, block_size, num_kv_heads, head_dim);
  if (cache_dtype == PA_FP8_E4M3 &&
      !(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return fail(PA_ERR_SHAPE, "pa_write_kv: e4m3 scales must be finite and positive");
  if (num_tokens == 0) return ok();
  if (!k || !v || !slot_mapping || !k_pool || !v_pool)
    return fail(PA_ERR_NULL, "pa_write_kv: null pointer");
  int dev;
  if (current_device(&dev)) return fail(PA_ERR_CUDA, "pa_write_kv: no current device");
  const int64_t total = 2LL * num_tokens * num_kv_heads * (head_dim / 8);
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(cdiv(total, 256), static_cast<int64_t>(device_sms(dev)) * 8));
  const int64_t num_slots = static_cast<int64_t>(num_blocks) * block_size;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const auto* kk = static_cast<const uint16_t*>(k);
  const auto* vv = static_cast<const uint16_t*>(v);
  auto* kp = static_cast<uint8_t*>(k_pool);
  auto* vp = static_cast<uint8_t*>(v_pool);
  const unsigned g = static_cast<unsigned>(grid);
  if (cache_dtype != PA_FP8_E4M3)
    pa::write_kv_kernel<false, false><<<g, 256, 0, st>>>(kk, vv, slot_mapping, num_tokens, kp, vp,
                                                         num_slots, num_kv_heads, head_dim, 1.f, 1.f);
  else if (in_dtype == PA_BF16)
    pa::write_kv_kernel<true, true><<<g, 256, 0, st>>>(kk, vv, slot_mapping, num_tokens, kp, vp,
                                                       num_slots, num_kv_heads, head_dim, k_scale, v_scale);
  else
    pa::write_kv_kernel<true, false><<<g, 256, 0, st>>>(kk, vv, slot_mapping, num_tokens, kp, vp,
                                                        num_slots, num_kv_heads, head_dim, k_scale, v_scale);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pa_write_kv launch");
  return ok();
}

pa_status pa_copy_blocks(void* k_pool, void* v_pool, pa_dtype cache_dtype, int32_t num_blocks,
                         int32_t block_size, int32_t num_kv_heads, int32_t head_dim,
                         const int64_t* src_dst_pairs, int32_t num_pairs, pa_stream_t stream) {
  if (!valid_dtype(cache_dtype)) return fail(PA_ERR_DTYPE, "pa_copy_blocks: unknown dtype");
  if (num_pairs < 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
    return fail(PA_ERR_SHAPE, "pa_copy_blocks: unsupported sizes");
  if (num_pairs == 0) return ok();
  if (!k_pool || !v_pool || !src_dst_pairs) return fail(PA_ERR_NULL, "pa_copy_blocks: null pointer");
  const int64_t block_bytes =
      static_cast<int64_t>(block_size) * num_kv_heads * head_dim * elem_bytes(cache_dtype);
  const int64_t nvec = block_bytes / 16;
  const unsigned per_pair = static_cast<unsigned>(std::min<int64_t>(8, cdiv(nvec, 256)));
  dim3 grid(static_cast<unsigned>(num_pairs), per_pair);
  pa::copy_blocks_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint8_t*>(k_pool), static_cast<uint8_t*>(v_pool), src_dst_pairs, num_blocks,
      block_bytes);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pa_copy_blocks launch");
  return ok();
}

pa_status pa_swap_blocks(const void* src_k, const void* src_v, int32_t src_blocks, void* dst_k,
                         void* dst_v, int32_t dst_blocks, pa_dtype cache_dtype, int32_t block_size,
                         int32_t num_kv_heads, int32_t head_dim, const int64_t* src_dst_pairs,
                         int32_t num_pairs, pa_stream_t stream) {
  if (!valid_dtype(cache_dtype)) return fail(PA_ERR_DTYPE, "pa_swap_blocks: unknown dtype");
  if (num_pairs < 0 || !cache_shape_ok(src_blocks, block_size, num_kv_heads, head_dim) ||
      dst_blocks <= 0)
    return fail(PA_ERR_SHAPE, "pa_swap_blocks: unsupported sizes");
  if (num_pairs == 0) return ok();
  if (!src_k || !src_v || !dst_k || !dst_v || !src_dst_pairs)
    return fail(PA_ERR_NULL, "pa_swap_blocks: null pointer");
  const void* ptrs[5] = {src_k, src_v, dst_k, dst_v, src_dst_pairs};
  for (const void* p : ptrs) {  // every buffer must be reachable from the device
    cudaPointerAttributes at;
    const cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return fail(PA_ERR_MEMORY, "pa_swap_blocks: a buffer is not known to CUDA");
    }
    const bool reachable = at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged ||
                           (at.type == cudaMemoryTypeHost && at.devicePointer == p);
    if (!reachable)
      return fail(PA_ERR_MEMORY, "pa_swap_blocks: a buffer is pageable or not mapped for the device");
  }
  const int64_t block_bytes =
      static_cast<int64_t>(block_size) * num_kv_heads * head_dim * elem_bytes(cache_dtype);
  const int64_t nvec = block_bytes / 16;
  const unsigned per_pair = static_cast<unsigned>(std::min<int64_t>(8, cdiv(nvec, 256 * 4)));
  dim3 grid(static_cast<unsigned>(num_pairs), std::max(1u, per_pair));
  pa::swap_blocks_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(src_k), static_cast<const uint8_t*>(src_v),
      static_cast<uint8_t*>(dst_k), static_cast<uint8_t*>(dst_v), src_dst_pairs, src_blocks,
      dst_blocks, block_bytes);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pa_swap_blocks launch");
  return ok();
}

pa_status pa_hash_blocks(const int32_t* token_ids, int64_t token_stride,
                         const int32_t* num_tokens, int32_t num_seqs, int32_t block_size,
                         uint64_t* block_hashes, int32_t max_blocks, pa_stream_t stream) {
  if (num_seqs < 0 || block_size <= 0 || max_blocks <= 0 || token_stride <= 0)
    return fail(PA_ERR_SHAPE, "pa_hash_blocks: bad sizes");
  if (num_seqs == 0) return ok();
  if (!token_ids || !num_tokens || !block_hashes) return fail(PA_ERR_NULL, "pa_hash_blocks: null pointer");
  pa::hash_blocks_kernel<<<static_cast<unsigned>(num_seqs), pa::kHashChunk, 0,
                           reinterpret_cast<cudaStream_t>(stream)>>>(
      token_ids, token_stride, num_tokens, block_size,
      reinterpret_cast<unsigned long long*>(block_hashes), max_blocks);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pa_hash_blocks launch");
  return ok();
}

int32_t pa_decode_split_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t block_size,
                               int32_t max_context_len, int32_t split_tokens) {
  if (num_seqs < 0 || num_kv_heads <= 0 || (block_size != 16 && block_size != 32) ||
      max_context_len < 0 || split_tokens < 0)
    return 0;
  return choose_split(num_seqs, num_kv_heads, block_size, max_context_len, split_tokens);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t block_size, int32_t max_context_len,
                                int32_t split_tokens) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || (head_dim != 64 && head_dim != 128) ||
      (block_size != 16 && block_size != 32) || max_context_len < 0 || split_tokens < 0)
    return 0;
  const int32_t S = choose_split(num_seqs, num_kv_heads, block_size, max_context_len, split_tokens);
  return ws_layout(num_seqs, num_q_heads, num_kv_heads * col_groups(num_q_heads, num_kv_heads),
                   head_dim, max_context_len, S).bytes;
}

pa_status pa_decode(void* out, const void* q, pa_dtype q_dtype, const void* k_pool,
                    const void* v_pool, pa_dtype cache_dtype, const int32_t* block_tables,
                    int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, int32_t num_seqs, int32_t num_q_heads,
                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                    int32_t num_blocks, float scale, float k_scale, float v_scale,
                    int32_t split_tokens, void* workspace, size_t workspace_bytes,
                    pa_stream_t stream) {
  if (!valid_dtype(q_dtype) || !valid_dtype(cache_dtype))
    return fail(PA_ERR_DTYPE, "pa_decode: unknown dtype");
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (q_dtype == PA_FP8_E4M3 || (!fp8 && q_dtype != cache_dtype))
    return fail(PA_ERR_DTYPE, "pa_decode: q must be f16/bf16 and match a 16-bit cache");
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || max_context_len < 0 || split_tokens < 0 ||
      !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
    return fail(PA_ERR_SHAPE, "pa_decode: unsupported sizes (seqs %d, max_blocks %d, max_ctx %d, "
                "blocks %d, bs %d, kv heads %d, dim %d)", num_seqs, max_blocks_per_seq,
                max_context_len, num_blocks, block_size, num_kv_heads, head_dim);
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return fail(PA_ERR_SHAPE, "pa_decode: max_context_len %d exceeds max_blocks_per_seq * bs",
                max_context_len);
  if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      num_q_heads / num_kv_heads > kMaxQHeadsPerKv)
    return fail(PA_ERR_HEADS, "pa_decode: num_q_heads %d must be a multiple of num_kv_heads %d "
                "with at most %d query heads per kv head", num_q_heads, num_kv_heads,
                kMaxQHeadsPerKv);
  if (!std::isfinite(scale) || (fp8 && !(std::isfinite(k_scale) && k_scale > 0.f &&
                                         std::isfinite(v_scale) && v_scale > 0.f)))
    return fail(PA_ERR_SHAPE, "pa_decode: scales must be finite (and positive for e4m3)");
  if (num_seqs == 0) return ok();
  if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens)
    return fail(PA_ERR_NULL, "pa_decode: null pointer");
  const int32_t S = choose_split(num_seqs, num_kv_heads, block_size, max_context_len, split_tokens);
  const int32_t ncg = col_groups(num_q_heads, num_kv_heads);
  const WsLayout w = ws_layout(num_seqs, num_q_heads, num_kv_heads * ncg, head_dim,
                               max_context_len, S);
  if (!workspace || workspace_bytes < w.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(PA_ERR_WORKSPACE, "pa_decode: workspace needs %zu bytes, 256-byte aligned (got %zu)",
                w.bytes, workspace_bytes);
  int dev;
  if (current_device(&dev)) return fail(PA_ERR_CUDA, "pa_decode: no current device");
  auto st = reinterpret_cast<cudaStream_t>(stream);
  auto* ws = static_cast<uint8_t*>(workspace);

  if ((reinterpret_cast<uintptr_t>(k_pool) | reinterpret_cast<uintptr_t>(v_pool)) & 15)
    return fail(PA_ERR_SHAPE, "pa_decode: the pools must be 16-byte aligned");
  pa::DecodeArgs a;
  pa_status ms = encode_pool_map(&a.tmap_k, k_pool, num_blocks, block_size, num_kv_heads,
                                 head_dim, elem_bytes(cache_dtype));
  if (ms == PA_OK)
    ms = encode_pool_map(&a.tmap_v, v_pool, num_blocks, block_size, num_kv_heads, head_dim,
                         elem_bytes(cache_dtype));
  if (ms != PA_OK) return ms;
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.counter = reinterpret_cast<int32_t*>(ws + w.counter);
  a.total = reinterpret_cast<const int32_t*>(ws + w.total);
  a.seq_off = reinterpret_cast<const int32_t*>(ws + w.seq_off);
  a.order = reinterpret_cast<const int4*>(ws + w.order);
  a.arrived = reinterpret_cast<int32_t*>(ws + w.arrived);
  a.lse_part = reinterpret_cast<float*>(ws + w.lse);
  a.o_part = reinterpret_cast<float*>(ws + w.o);
  a.num_seqs = num_seqs;
  a.hq = num_q_heads;
  a.hkv = num_kv_heads;
  a.group = num_q_heads / num_kv_heads;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.max_ctx = max_context_len;
  a.sl2 = scale * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
  a.out_scale = fp8 ? v_scale : 1.f;
  a.ncg = ncg;
  const bool qbf = q_dtype == PA_BF16;

  int per_sm = 0;  // resident CTAs of this instance (cached per device)
  {
    pa_status os;
    if (cache_dtype == PA_F16)
      os = occupancy_shape<pa::kCacheF16, false>(head_dim, block_size, dev, &per_sm);
    else if (cache_dtype == PA_BF16)
      os = occupancy_shape<pa::kCacheBF16, true>(head_dim, block_size, dev, &per_sm);
    else if (qbf)
      os = occupancy_shape<pa::kCacheE4M3, true>(head_dim, block_size, dev, &per_sm);
    else
      os = occupancy_shape<pa::kCacheE4M3, false>(head_dim, block_size, dev, &per_sm);
    if (os != PA_OK) return os;
  }
  const int64_t items_upper = w.ranges * num_kv_heads * ncg;
  // unsplit contexts and no more items than resident CTAs: no planning
  // kernel (CTA c forms item c itself; there is no queue to order)
  const bool direct = !w.is_split && items_upper <= static_cast<int64_t>(device_sms(dev)) * per_sm;
  a.direct = direct ? 1 : 0;
  a.split_len = w.is_split ? S : std::max(S, max_context_len);
  a.split_out = reinterpret_cast<int32_t*>(ws + w.split);
  // the automatic split may be lengthened on the device from the actual
  // lengths (never shortened: the workspace holds the ranges of S), aiming
  // at 15/16 of a kPlanSms-SM persistent grid of this instance in items
  int adapt_items = 0;
  if (split_tokens == 0 && w.is_split)
    adapt_items = static_cast<int>(std::max<int64_t>(1, kPlanSms * per_sm * 15 / 16));
  if (!direct) {
    pa::plan_kernel<<<1, 1024, 0, st>>>(context_lens, num_seqs, max_context_len, max_blocks_per_seq,
                                        block_size, w.is_split ? S : std::max(S, max_context_len),
                                        adapt_items, num_kv_heads * ncg,
                                        reinterpret_cast<int32_t*>(ws + w.counter),
                                        reinterpret_cast<int32_t*>(ws + w.total),
                                        reinterpret_cast<int32_t*>(ws + w.split),
                                        reinterpret_cast<int32_t*>(ws + w.seq_off),
                                        reinterpret_cast<int4*>(ws + w.order),
                                        w.is_split ? reinterpret_cast<int32_t*>(ws + w.arrived) : nullptr);
  }
  pa_status s;
  if (cache_dtype == PA_F16)
    s = dispatch_shape<pa::kCacheF16, false>(a, head_dim, block_size, items_upper, dev, st);
  else if (cache_dtype == PA_BF16)
    s = dispatch_shape<pa::kCacheBF16, true>(a, head_dim, block_size, items_upper, dev, st);
  else if (qbf)
    s = dispatch_shape<pa::kCacheE4M3, true>(a, head_dim, block_size, items_upper, dev, st);
  else
    s = dispatch_shape<pa::kCacheE4M3, false>(a, head_dim, block_size, items_upper, dev, st);
  if (s != PA_OK) return s;
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pa_decode launch");
  return ok();
}

size_t pa_decode_shared_prefix_workspace_size(int32_t num_seqs, int32_t num_q_heads,
                                              int32_t num_kv_heads, int32_t head_dim,
                                              int32_t block_size, int32_t max_context_len,
                                              int32_t split_tokens) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || (head_dim != 64 && head_dim != 128) ||
      (block_size != 16 && block_size != 32) || max_context_len < 0 || split_tokens < 0)
    return 0;
  return cascade_ws_layout(num_seqs, num_kv_heads, head_dim, block_size, max_context_len,
                           split_tokens).bytes;
}

pa_status pa_decode_shared_prefix(void* out, const void* q, pa_dtype q_dtype, const void* k_pool,
                                  const void* v_pool, pa_dtype cache_dtype,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t max_context_len,
                                  const int32_t* group_start, const int32_t* group_seqs,
                                  int32_t num_groups, int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t num_blocks, float scale, float k_scale, float v_scale,
                                  int32_t split_tokens, void* workspace, size_t workspace_bytes,
                                  pa_stream_t stream) {
  if (!valid_dtype(q_dtype) || !valid_dtype(cache_dtype))
    return fail(PA_ERR_DTYPE, "pa_decode_shared_prefix: unknown dtype");
  const bool fp8 = cache_dtype == PA_FP8_E4M3;
  if (q_dtype == PA_FP8_E4M3 || (!fp8 && q_dtype != cache_dtype))
    return fail(PA_ERR_DTYPE, "pa_decode_shared_prefix: q must be f16/bf16 and match a 16-bit cache");
  if (num_seqs < 0 || num_groups < 0 || max_blocks_per_seq <= 0 || max_context_len < 0 ||
      split_tokens < 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim))
    return fail(PA_ERR_SHAPE, "pa_decode_shared_prefix: unsupported sizes (seqs %d, groups %d, "
                "max_blocks %d, max_ctx %d, blocks %d, bs %d, kv heads %d, dim %d)", num_seqs,
                num_groups, max_blocks_per_seq, max_context_len, num_blocks, block_size,
                num_kv_heads, head_dim);
  if (static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return fail(PA_ERR_SHAPE, "pa_decode_shared_prefix: max_context_len %d exceeds "
                "max_blocks_per_seq * bs", max_context_len);
  if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      num_q_heads / num_kv_heads > pa::kCascadeRows)
    return fail(PA_ERR_HEADS, "pa_decode_shared_prefix: num_q_heads %d must be a multiple of "
                "num_kv_heads %d with at most %d query heads per kv head", num_q_heads,
                num_kv_heads, pa::kCascadeRows);
  if (!std::isfinite(scale) || (fp8 && !(std::isfinite(k_scale) && k_scale > 0.f &&
                                         std::isfinite(v_scale) && v_scale > 0.f)))
    return fail(PA_ERR_SHAPE, "pa_decode_shared_prefix: scales must be finite (and positive for e4m3)");
  if (num_seqs == 0) return ok();
  if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens ||
      (num_groups > 0 && (!group_start || !group_seqs)))
    return fail(PA_ERR_NULL, "pa_decode_shared_prefix: null pointer");
  const CascadeWs w = cascade_ws_layout(num_seqs, num_kv_heads, head_dim, block_size,
                                        max_context_len, split_tokens);
  if (!workspace || workspace_bytes < w.bytes || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(PA_ERR_WORKSPACE, "pa_decode_shared_prefix: workspace needs %zu bytes, 256-byte "
                "aligned (got %zu)", w.bytes, workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(k_pool) | reinterpret_cast<uintptr_t>(v_pool)) & 15)
    return fail(PA_ERR_SHAPE, "pa_decode_shared_prefix: the pools must be 16-byte aligned");
  int dev;
  if (current_device(&dev)) return fail(PA_ERR_CUDA, "pa_decode_shared_prefix: no current device");
  auto st = reinterpret_cast<cudaStream_t>(stream);
  auto* ws = static_cast<uint8_t*>(workspace);

  pa::CascadeArgs a;
  pa_status ms = encode_pool_map(&a.tmap_k, k_pool, num_blocks, block_size, num_kv_heads,
                                 head_dim, elem_bytes(cache_dtype));
  if (ms == PA_OK)
    ms = encode_pool_map(&a.tmap_v, v_pool, num_blocks, block_size, num_kv_heads, head_dim,
                         elem_bytes(cache_dtype));
  if (ms != PA_OK) return ms;
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.chunk_seqs = reinterpret_cast<const int32_t*>(ws + w.chunk_seqs);
  a.chunks = reinterpret_cast<const int4*>(ws + w.chunks);
  a.ranges = reinterpret_cast<const int4*>(ws + w.ranges);
  a.total = reinterpret_cast<const int32_t*>(ws + w.total);
  a.counter = reinterpret_cast<int32_t*>(ws + w.counter);
  a.arrived = reinterpret_cast<int32_t*>(ws + w.arrived);
  a.lse_part = reinterpret_cast<float*>(ws + w.lse);
  a.o_part = reinterpret_cast<float*>(ws + w.o);
  a.hq = num_q_heads;
  a.hkv = num_kv_heads;
  a.group = num_q_heads / num_kv_heads;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.sl2 = scale * (fp8 ? k_scale : 1.f) * 1.4426950408889634f;
  a.out_scale = fp8 ? v_scale : 1.f;

  pa::cascade_plan_kernel<<<1, 1024, 0, st>>>(
      context_lens, block_tables, group_start, group_seqs, num_groups, num_seqs, max_context_len,
      max_blocks_per_seq, block_size, a.group, num_kv_heads, w.r_floor,
      reinterpret_cast<int32_t*>(ws + w.seen), reinterpret_cast<int32_t*>(ws + w.chunk_seqs),
      reinterpret_cast<int4*>(ws + w.chunks), reinterpret_cast<int4*>(ws + w.ranges),
      reinterpret_cast<int32_t*>(ws + w.total), a.counter, a.arrived);
  const int64_t items_upper = w.slots * num_kv_heads;
  pa_status s;
  if (cache_dtype == PA_F16)
    s = dispatch_cascade<pa::kCacheF16, false>(a, head_dim, block_size, items_upper, dev, st);
  else if (cache_dtype == PA_BF16)
    s = dispatch_cascade<pa::kCacheBF16, true>(a, head_dim, block_size, items_upper, dev, st);
  else if (q_dtype == PA_BF16)
    s = dispatch_cascade<pa::kCacheE4M3, true>(a, head_dim, block_size, items_upper, dev, st);
  else
    s = dispatch_cascade<pa::kCacheE4M3, false>(a, head_dim, block_size, items_upper, dev, st);
  if (s != PA_OK) return s;
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pa_decode_shared_prefix launch");
  return ok();
}

pa_status pa_prefill(void* out, const void* q, pa_dtype q_dtype, const void* k_pool,
                     const void* v_pool, pa_dtype cache_dtype, const int32_t* block_tables,
                     int32_t max_blocks_per_seq, const int32_t* context_lens,
                     const int32_t* query_start, int32_t num_seqs, int32_t max_query_len,
                     int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                     int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
                     pa_stream_t stream) {
  if (!valid_dtype(q_dtype) || !valid_dtype(cache_dtype) || q_dtype == PA_FP8_E4M3 ||
      cache_dtype != q_dtype)
    return fail(PA_ERR_DTYPE, "pa_prefill: q and the cache must share a 16-bit dtype");
  if ((head_dim != 64 && head_dim != pa::kPfMaxD) || num_seqs < 0 || max_query_len < 0 || max_context_len < 0 ||
      max_blocks_per_seq <= 0 || !cache_shape_ok(num_blocks, block_size, num_kv_heads, head_dim) ||
      static_cast<int64_t>(max_context_len) > static_cast<int64_t>(max_blocks_per_seq) * block_size)
    return fail(PA_ERR_SHAPE, "pa_prefill: unsupported sizes (head_dim must be 64 or %d)",
                pa::kPfMaxD);
  // a CTA takes T = floor(128 / G) new tokens (T * G rows of its 128; the
  // rest are padding rows that are never loaded or written)
  if (num_q_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
      num_q_heads / num_kv_heads > pa::kPfRows)
    return fail(PA_ERR_HEADS, "pa_prefill: num_q_heads must be a multiple of num_kv_heads with "
                "at most %d query heads per kv head", pa::kPfRows);
  if (!std::isfinite(scale)) return fail(PA_ERR_SHAPE, "pa_prefill: scale must be finite");
  if (num_seqs == 0 || max_query_len == 0) return ok();
  if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens || !query_start)
    return fail(PA_ERR_NULL, "pa_prefill: null pointer");
  if ((reinterpret_cast<uintptr_t>(k_pool) | reinterpret_cast<uintptr_t>(v_pool) |
       reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(PA_ERR_SHAPE, "pa_prefill: pools, q and out must be 16-byte aligned");
  int dev;
  if (current_device(&dev)) return fail(PA_ERR_CUDA, "pa_prefill: no current device");
  pa::PrefillArgs a;
  pa_status ms = encode_pool_map(&a.tmap_k, k_pool, num_blocks, block_size, num_kv_heads,
                                 head_dim, 2, true);
  if (ms == PA_OK)
    ms = encode_pool_map(&a.tmap_v, v_pool, num_blocks, block_size, num_kv_heads, head_dim, 2);
  if (ms != PA_OK) return ms;
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_start = query_start;
  a.hq = num_q_heads;
  a.hkv = num_kv_heads;
  a.group = num_q_heads / num_kv_heads;
  a.max_blocks = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.max_ctx = max_context_len;
  a.sl2 = scale * 1.4426950408889634f;
  const int T = pa::kPfRows / a.group;
  dim3 grid(static_cast<unsigned>(cdiv(max_query_len, T)), static_cast<unsigned>(num_kv_heads),
            static_cast<unsigned>(num_seqs));
  if (grid.y > 65535 || grid.z > 65535)
    return fail(PA_ERR_SHAPE, "pa_prefill: too many kv heads or sequences for one launch");
  auto st = reinterpret_cast<cudaStream_t>(stream);
  auto launch = [&](auto kern, int smem_bytes) -> pa_status {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill)");
    kern<<<grid, pa::kPfThreads, smem_bytes, st>>>(a);
    return PA_OK;
  };
  pa_status ls;
  const bool bf = q_dtype == PA_BF16;
#define PA_PF_LAUNCH(BS_, D_)                                                              \
  (bf ? launch(pa::prefill_kernel<true, BS_, D_>, pa::PrefillCfg<BS_, D_>::kSmemBytes)     \
      : launch(pa::prefill_kernel<false, BS_, D_>, pa::PrefillCfg<BS_, D_>::kSmemBytes))
  if (head_dim == 64)
    ls = block_size == 16 ? PA_PF_LAUNCH(16, 64) : PA_PF_LAUNCH(32, 64);
  else
    ls = block_size == 16 ? PA_PF_LAUNCH(16, 128) : PA_PF_LAUNCH(32, 128);
#undef PA_PF_LAUNCH
  if (ls != PA_OK) return ls;
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pa_prefill launch");
  return ok();
}

pa_status pa_sync_status(pa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pa_sync_status: stream");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, pa::g_device_error, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "pa_sync_status: read error word");
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(pa::g_device_error, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "pa_sync_status: clear error word");
    if (v == PA_ERR_TIMEOUT)
      return fail(PA_ERR_TIMEOUT, "a kernel gave up waiting for an asynchronous copy");
    return fail(static_cast<pa_status>(v), "a kernel met an out-of-range index and skipped it");
  }
  return ok();
}

// ------------------------------------------------------------- debug checks
pa_status pa_validate_slot_mapping(const int64_t* slot_mapping, int32_t num_tokens,
                                   int32_t num_blocks, int32_t block_size, pa_stream_t stream) {
  if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0)
    return fail(PA_ERR_SHAPE, "pa_validate_slot_mapping: bad sizes");
  if (num_tokens > 0 && !slot_mapping) return fail(PA_ERR_NULL, "pa_validate_slot_mapping: null");
  std::vector<int64_t> h;
  pa_status s = fetch(h, slot_mapping, num_tokens, reinterpret_cast<cudaStream_t>(stream),
                      "pa_validate_slot_mapping");
  if (s != PA_OK) return s;
  const int64_t n = static_cast<int64_t>(num_blocks) * block_size;
  std::vector<uint8_t> seen(static_cast<size_t>(n), 0);
  for (int32_t t = 0; t < num_tokens; ++t) {
    if (h[t] < 0) continue;
    if (h[t] >= n) return fail(PA_ERR_RANGE, "slot_mapping[%d] = %lld is outside the pool", t, (long long)h[t]);
    if (seen[h[t]]++) return fail(PA_ERR_ALIAS, "slot %lld is written twice", (long long)h[t]);
  }
  return ok();
}

pa_status pa_validate_copy_pairs(const int64_t* src_dst_pairs, int32_t num_pairs,
                                 int32_t num_blocks, pa_stream_t stream) {
  if (num_pairs < 0 || num_blocks <= 0) return fail(PA_ERR_SHAPE, "pa_validate_copy_pairs: bad sizes");
  if (num_pairs > 0 && !src_dst_pairs) return fail(PA_ERR_NULL, "pa_validate_copy_pairs: null");
  std::vector<int64_t> h;
  pa_status s = fetch(h, src_dst_pairs, 2 * static_cast<size_t>(num_pairs),
                      reinterpret_cast<cudaStream_t>(stream), "pa_validate_copy_pairs");
  if (s != PA_OK) return s;
  std::vector<uint8_t> role(static_cast<size_t>(num_blocks), 0);  // 1 src, 2 dst
  for (int32_t p = 0; p < num_pairs; ++p)
    for (int k = 0; k < 2; ++k)
      if (h[2 * p + k] < 0 || h[2 * p + k] >= num_blocks)
        return fail(PA_ERR_RANGE, "pair %d holds block id %lld outside the pool", p,
                    (long long)h[2 * p + k]);
  for (int32_t p = 0; p < num_pairs; ++p) role[h[2 * p]] |= 1;
  for (int32_t p = 0; p < num_pairs; ++p) {
    const int64_t d = h[2 * p + 1];
    if (role[d] & 2) return fail(PA_ERR_ALIAS, "block %lld is a destination twice", (long long)d);
    if (role[d] & 1) return fail(PA_ERR_ALIAS, "block %lld is both a source and a destination", (long long)d);
    role[d] |= 2;
  }
  return ok();
}

pa_status pa_validate_block_tables(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* context_lens, int32_t num_seqs,
                                   int32_t max_context_len, int32_t block_size, int32_t num_blocks,
                                   pa_stream_t stream) {
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(PA_ERR_SHAPE, "pa_validate_block_tables: bad sizes");
  if (num_seqs > 0 && (!block_tables || !context_lens))
    return fail(PA_ERR_NULL, "pa_validate_block_tables: null");
  auto st = reinterpret_cast<cudaStream_t>(stream);
  std::vector<int32_t> t, c;
  pa_status s = fetch(c, context_lens, num_seqs, st, "pa_validate_block_tables");
  if (s == PA_OK)
    s = fetch(t, block_tables, static_cast<size_t>(num_seqs) * max_blocks_per_seq, st,
              "pa_validate_block_tables");
  if (s != PA_OK) return s;
  for (int32_t i = 0; i < num_seqs; ++i) {
    if (c[i] < 0 || c[i] > max_context_len)
      return fail(PA_ERR_RANGE, "context_lens[%d] = %d outside [0, %d]", i, c[i], max_context_len);
    const int64_t nb = cdiv(c[i], block_size);
    if (nb > max_blocks_per_seq)
      return fail(PA_ERR_RANGE, "sequence %d needs %lld blocks, table holds %d", i, (long long)nb,
                  max_blocks_per_seq);
    for (int64_t j = 0; j < nb; ++j) {
      const int32_t b = t[static_cast<size_t>(i) * max_blocks_per_seq + j];
      if (b < 0 || b >= num_blocks)
        return fail(PA_ERR_RANGE, "block_tables[%d][%lld] = %d outside the pool", i, (long long)j, b);
    }
  }
  return ok();
}

}  // extern "C"

// ------------------------------------------------- decode without a workspace
// Scratch for pa_decode_noalloc: reserved in device memory when the library
// is loaded (on every GPU that loads it, until the process exits).  Host code
// must not use this name as a device address: it is a host-side stand-in;
// the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[PA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of g_noalloc_scratch, looked up once per device and CUDA
// context: the array lives in the library's module of each context, so a
// new context on the same device (after cudaDeviceReset, or a caller's own
// non-primary context) gets its own address.  Contexts are told apart by
// the driver's unique context id, which is never reused within a process.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current context (0 if none).
unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_ctx == nullptr || get_id == nullptr || get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

struct NoallocSlot {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
std::mutex g_noalloc_mu;
NoallocSlot g_noalloc_slot[kMaxDevices];

pa_status noalloc_scratch(int dev, void** ptr) {
  // cudaGetDevice made the device's primary context current if the thread
  // had none, so the id below is the context the launches will use
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  if (slot.ptr == nullptr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return cuda_fail(e, "pa_decode_noalloc: cudaGetSymbolAddress of the built-in scratch");
    slot.ctx_id = id;
    slot.ptr = p;
  }
  *ptr = slot.ptr;
  return PA_OK;
}
}  // namespace

extern "C" pa_status pa_decode_noalloc(
    void* out, const void* q, pa_dtype q_dtype, const void* k_pool, const void* v_pool,
    pa_dtype cache_dtype, const int32_t* block_tables, int32_t max_blocks_per_seq,
    const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
    float k_scale, float v_scale, int32_t split_tokens, pa_stream_t stream) {
  const size_t need = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                               block_size, max_context_len, split_tokens);
  if (need > PA_DECODE_NOALLOC_SCRATCH_BYTES)
    return fail(PA_ERR_WORKSPACE,
                "pa_decode_noalloc: these sizes need %zu bytes of scratch but the built-in scratch "
                "holds %u; pass a larger split_tokens or call pa_decode with your own workspace",
                need, PA_DECODE_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  if (num_seqs > 0 && need > 0) {  // invalid sizes fall through to pa_decode's checks
    int dev;
    if (current_device(&dev)) return fail(PA_ERR_CUDA, "pa_decode_noalloc: no current device");
    const pa_status s = noalloc_scratch(dev, &scratch);
    if (s != PA_OK) return s;
  }
  return pa_decode(out, q, q_dtype, k_pool, v_pool, cache_dtype, block_tables,
                   max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_q_heads,
                   num_kv_heads, head_dim, block_size, num_blocks, scale, k_scale, v_scale,
                   split_tokens, scratch, PA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}
