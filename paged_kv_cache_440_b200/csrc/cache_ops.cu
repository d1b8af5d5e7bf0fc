// Append (reshape_and_cache), per-token-head quantization and copy-on-write
// block copy.
//
// * Append: a decode step computes only the new token's K and V and puts them
//   at the end of its sequence's cache [KV Cache 原理与 PagedAttention, §一;
//   bjdmk.com.cn/news/6246348, §2.1]; in a paged cache that end is row
//   slot % block_size of physical block slot / block_size.
// * Quantize: symmetric absmax per (token, head) row, fp32 scale
//   [bjdmk.com.cn/news/6246348, §5.2]; INT8 or FP8-E5M2 codes
//   [KV Cache 原理与 PagedAttention, §四]. INT8_KCHAN caches code keys with
//   the layer's fixed per-channel scales (per-channel granularity, §5.2 of
//   the same page) and values per row as INT8.
// * Block copy: the copy half of copy-on-write [bjdmk.com.cn/news/6246348,
//   §3.2]: whole blocks, every layer, K, V and scales.
//
// All three are pure data movement at a few hundred KB per decode step; a
// warp handles one token's rows (or a CTA one block region) with 16-byte
// vector accesses, its loads in flight together before its stores.
#include <algorithm>
#include <cstring>
#include <vector>

#include "device.cuh"
#include "internal.h"

namespace pagedkv {
namespace {

using namespace dev;

// Small CTAs: measured faster than 8 or 16 warps for a 4096-token append
// (more CTAs in flight per SM as they retire).
constexpr int kWarpsPerCta = 4;

// ---------------------------------------------------------------- 16-bit copy

// Up to this many 16-byte chunks per lane are loaded before any is stored, so
// a warp has all of them in flight at once (one memory round trip per batch).
constexpr int kBatch = 8;

// One warp per token: the K and V rows of all its kv heads (2 * kv_heads *
// row_chunks 16-byte chunks), spread over the lanes.
__global__ void __launch_bounds__(kWarpsPerCta * 32)
append16_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                const int64_t *__restrict__ slots, int num_tokens, int kv_heads,
                int block_size, int row_chunks, int64_t num_slots, uint4 *__restrict__ kc,
                uint4 *__restrict__ vc, int *status) {
  launch_dependents();
  grid_dependency_wait();
  const int t = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= num_tokens) return;
  const int per_kv = kv_heads * row_chunks;  // chunks of one token's K (or V)
  const int n = 2 * per_kv;
  const int64_t slot = slots[t];
  int64_t blk = 0;
  int row = 0;
  for (int i0 = 0; i0 < n; i0 += kBatch * 32) {
    uint4 x[kBatch];
    // the rows do not depend on the slot: their loads go out with its load
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * 32 + lane;
      if (i < n) {
        const int j = i < per_kv ? i : i - per_kv;  // head * row_chunks + chunk
        x[u] = (i < per_kv ? k_new : v_new)[static_cast<int64_t>(t) * per_kv + j];
      }
    }
    if (i0 == 0) {
      if (slot < 0) return;
      if (slot >= num_slots) {
        if (lane == 0) atomicOr(status, kErrSlot);
        return;
      }
      blk = slot / block_size;
      row = static_cast<int>(slot - blk * block_size);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * 32 + lane;
      if (i < n) {
        const int j = i < per_kv ? i : i - per_kv;
        const int h = j / row_chunks, c = j - h * row_chunks;
        (i < per_kv ? kc : vc)[((blk * kv_heads + h) * block_size + row) * row_chunks + c] = x[u];
      }
    }
  }
}

// ---------------------------------------------------------------- quantize

// One warp per (token, kv head): quantize the K row and the V row, store the
// codes and scales at the slot. The rows are loaded together with the slot
// (they do not depend on it), so the warp waits on memory once.
template <int D, int IN_T, int OUT_T>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
append_quant_kernel(const uint16_t *__restrict__ k_new, const uint16_t *__restrict__ v_new,
                    const int64_t *__restrict__ slots, int num_tokens, int kv_heads,
                    int block_size, int64_t num_slots, uint8_t *__restrict__ kc,
                    uint8_t *__restrict__ vc, float *__restrict__ ks, float *__restrict__ vs,
                    int *status) {
  launch_dependents();
  grid_dependency_wait();
  const int warp = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (warp >= num_tokens * kv_heads) return;
  const int t = warp / kv_heads;
  const int h = warp - t * kv_heads;
  const int64_t src_row = static_cast<int64_t>(t) * kv_heads + h;
  float xk[D / 32], xv[D / 32];
  const int64_t slot = slots[t];
  load_row<D, IN_T>(k_new + src_row * D, lane, xk);
  load_row<D, IN_T>(v_new + src_row * D, lane, xv);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (lane == 0 && h == 0) atomicOr(status, kErrSlot);
    return;
  }
  const int64_t blk = slot / block_size;
  const int row = static_cast<int>(slot - blk * block_size);
  const int64_t dst_row = (blk * kv_heads + h) * block_size + row;
  // INT8_KCHAN: ks holds the layer's [kv_heads][D] channel scales
  constexpr int VQ = OUT_T == KV_INT8_KCHAN ? KV_INT8 : OUT_T;  // value coding
  constexpr int kRow = OUT_T == KV_INT4 ? D / 2 : D;  // bytes per row
  float scale;
  if constexpr (OUT_T == KV_INT8_KCHAN) {
    store_codes<D, KV_INT8>(kc + dst_row * kRow, lane, quantize_row_chan<D>(xk, ks + h * D, lane));
  } else {
    const uint32_t packed = quantize_row<D, OUT_T>(xk, &scale);
    store_codes<D, OUT_T>(kc + dst_row * kRow, lane, packed);
    if (OUT_T != KV_FP8_E5M2_CAST && lane == 0) ks[dst_row] = scale;
  }
  const uint32_t vpacked = quantize_row<D, VQ>(xv, &scale);
  store_codes<D, VQ>(vc + dst_row * kRow, lane, vpacked);
  if (VQ != KV_FP8_E5M2_CAST && lane == 0) vs[dst_row] = scale;
}

// Standalone: one warp per contiguous row.
template <int D, int IN_T, int OUT_T>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
quantize_kernel(const uint16_t *__restrict__ x_in, int64_t rows, uint8_t *__restrict__ codes,
                float *__restrict__ scales) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float x[D / 32];
  float scale;
  load_row<D, IN_T>(x_in + row * D, lane, x);
  uint32_t packed = quantize_row<D, OUT_T>(x, &scale);
  store_codes<D, OUT_T>(codes + row * (OUT_T == KV_INT4 ? D / 2 : D), lane, packed);
  if (lane == 0) scales[row] = scale;
}

// ---------------------------------------------------------------- block copy

constexpr int kMaxPairsPerLaunch = 1024;

struct CopyPairs {
  int32_t src[kMaxPairsPerLaunch];
  int32_t dst[kMaxPairsPerLaunch];
};

// grid (pair, layer, region): region 0 = K, 1 = V, 2 = K scale, 3 = V scale
// (no K-scale rows when the keys use channel scales: region 2 is then V's).
__global__ void __launch_bounds__(256)
block_copy_kernel(const __grid_constant__ CopyPairs pairs, char *__restrict__ base,
                  uint64_t layer_stride, uint64_t kv_stride, uint64_t ksc_stride,
                  uint32_t kv_block_bytes, uint32_t sc_block_bytes, int k_scale_rows) {
  const int i = blockIdx.x;
  const uint64_t layer = blockIdx.y;
  const int region = (blockIdx.z == 2 && !k_scale_rows) ? 3 : blockIdx.z;
  char *lb = base + layer * layer_stride;
  char *rb;
  uint32_t bytes;
  switch (region) {
    case 0: rb = lb; bytes = kv_block_bytes; break;
    case 1: rb = lb + kv_stride; bytes = kv_block_bytes; break;
    case 2: rb = lb + 2 * kv_stride; bytes = sc_block_bytes; break;
    default: rb = lb + 2 * kv_stride + ksc_stride; bytes = sc_block_bytes; break;
  }
  const uint4 *src = reinterpret_cast<const uint4 *>(rb + (uint64_t)pairs.src[i] * bytes);
  uint4 *dst = reinterpret_cast<uint4 *>(rb + (uint64_t)pairs.dst[i] * bytes);
  const uint32_t n = bytes / 16;
  // every load of a batch before its stores: one round trip per batch
  for (uint32_t j0 = threadIdx.x; j0 < n; j0 += kBatch * blockDim.x) {
    uint4 x[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (j0 + u * blockDim.x < n) x[u] = src[j0 + u * blockDim.x];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (j0 + u * blockDim.x < n) dst[j0 + u * blockDim.x] = x[u];
  }
}

template <int D, int IN_T, int OUT_T>
cudaError_t launch_quantize(const void *x, int64_t rows, void *codes, float *scales,
                            cudaStream_t st) {
  const int64_t grid = (rows + kWarpsPerCta - 1) / kWarpsPerCta;
  quantize_kernel<D, IN_T, OUT_T><<<(unsigned)grid, kWarpsPerCta * 32, 0, st>>>(
      static_cast<const uint16_t *>(x), rows, static_cast<uint8_t *>(codes), scales);
  return cudaGetLastError();
}

template <int D, int IN_T, int OUT_T>
cudaError_t launch_append_quant(kv_pool *p, int layer, const void *k, const void *v,
                                const int64_t *slots, int T, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(T) * p->d.num_kv_heads;
  const int64_t grid = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  cudaError_t e = launch_pdl(
      append_quant_kernel<D, IN_T, OUT_T>, dim3((unsigned)grid), dim3(kWarpsPerCta * 32), 0, st,
      static_cast<const uint16_t *>(k), static_cast<const uint16_t *>(v), slots, T,
      p->d.num_kv_heads, p->d.block_size, (int64_t)p->d.num_blocks * p->d.block_size,
      reinterpret_cast<uint8_t *>(layer_k(p, layer)), reinterpret_cast<uint8_t *>(layer_v(p, layer)),
      layer_ks(p, layer), layer_vs(p, layer), status_word(p));
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int IN_T, int OUT_T>
cudaError_t dispatch_append_quant_d(kv_pool *p, int layer, const void *k, const void *v,
                                    const int64_t *slots, int T, cudaStream_t st) {
  return p->d.head_dim == 128 ? launch_append_quant<128, IN_T, OUT_T>(p, layer, k, v, slots, T, st)
                              : launch_append_quant<64, IN_T, OUT_T>(p, layer, k, v, slots, T, st);
}

template <int IN_T, int OUT_T>
cudaError_t dispatch_quantize_d(int D, const void *x, int64_t rows, void *codes, float *scales,
                                cudaStream_t st) {
  return D == 128 ? launch_quantize<128, IN_T, OUT_T>(x, rows, codes, scales, st)
                  : launch_quantize<64, IN_T, OUT_T>(x, rows, codes, scales, st);
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace pagedkv

using namespace pagedkv;

extern "C" {

kv_status kv_append(kv_pool *pool, int32_t layer, const void *k_new, const void *v_new,
                    int32_t in_dtype, const int64_t *slot_mapping, int32_t num_tokens,
                    kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (layer < 0 || layer >= pool->d.num_layers)
    return fail(KV_ERR_INVALID, "layer %d out of range", layer);
  if (num_tokens < 0) return fail(KV_ERR_INVALID, "negative num_tokens");
  if (num_tokens == 0) return ok();
  if (!k_new || !v_new || !slot_mapping) return fail(KV_ERR_INVALID, "null input pointer");
  if (!aligned16(k_new) || !aligned16(v_new) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7))
    return fail(KV_ERR_INVALID, "k_new / v_new must be 16-byte aligned, slot_mapping 8-byte");
  if (in_dtype != KV_BF16 && in_dtype != KV_FP16)
    return fail(KV_ERR_UNSUPPORTED, "in_dtype must be KV_BF16 or KV_FP16");
  cudaStream_t st = (cudaStream_t)stream;
  const int cd = pool->d.cache_dtype;
  cudaError_t e;
  if (!is_quant(cd)) {
    if (in_dtype != cd)
      return fail(KV_ERR_UNSUPPORTED, "a 16-bit cache takes rows of its own dtype");
    const int64_t grid = (static_cast<int64_t>(num_tokens) + kWarpsPerCta - 1) / kWarpsPerCta;
    e = launch_pdl(append16_kernel, dim3((unsigned)grid), dim3(kWarpsPerCta * 32), 0, st,
                   static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new),
                   slot_mapping, num_tokens, pool->d.num_kv_heads, pool->d.block_size,
                   pool->row_bytes / 16, (int64_t)pool->d.num_blocks * pool->d.block_size,
                   reinterpret_cast<uint4 *>(layer_k(pool, layer)),
                   reinterpret_cast<uint4 *>(layer_v(pool, layer)), status_word(pool));
    if (e == cudaSuccess) e = cudaGetLastError();
  } else if (cd == KV_INT8) {
    e = in_dtype == KV_BF16
            ? dispatch_append_quant_d<KV_BF16, KV_INT8>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st)
            : dispatch_append_quant_d<KV_FP16, KV_INT8>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st);
  } else if (cd == KV_INT4) {
    e = in_dtype == KV_BF16
            ? launch_append_quant<128, KV_BF16, KV_INT4>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st)
            : launch_append_quant<128, KV_FP16, KV_INT4>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st);
  } else if (cd == KV_INT8_KCHAN) {
    e = in_dtype == KV_BF16
            ? dispatch_append_quant_d<KV_BF16, KV_INT8_KCHAN>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st)
            : dispatch_append_quant_d<KV_FP16, KV_INT8_KCHAN>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st);
  } else if (cd == KV_FP8_E5M2) {
    e = in_dtype == KV_BF16
            ? dispatch_append_quant_d<KV_BF16, KV_FP8_E5M2>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st)
            : dispatch_append_quant_d<KV_FP16, KV_FP8_E5M2>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st);
  } else {  // scale-less cast
    e = in_dtype == KV_BF16
            ? dispatch_append_quant_d<KV_BF16, KV_FP8_E5M2_CAST>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st)
            : dispatch_append_quant_d<KV_FP16, KV_FP8_E5M2_CAST>(pool, layer, k_new, v_new, slot_mapping, num_tokens, st);
  }
  kv_status s = cuda_check(e, "kv_append launch");
  return s == KV_OK ? ok() : s;
}

kv_status kv_quantize(const void *x, int32_t in_dtype, int64_t rows, int32_t head_dim,
                      int32_t out_dtype, void *codes, float *scales, kv_stream_t stream) {
  if (rows < 0) return fail(KV_ERR_INVALID, "negative rows");
  if (head_dim != 64 && head_dim != 128)
    return fail(KV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (in_dtype != KV_BF16 && in_dtype != KV_FP16)
    return fail(KV_ERR_UNSUPPORTED, "in_dtype must be KV_BF16 or KV_FP16");
  if (out_dtype != KV_INT8 && out_dtype != KV_FP8_E5M2 && out_dtype != KV_INT4)
    return fail(KV_ERR_UNSUPPORTED, "out_dtype must be KV_INT8, KV_FP8_E5M2 or KV_INT4");
  if (out_dtype == KV_INT4 && head_dim != 128)
    return fail(KV_ERR_UNSUPPORTED, "KV_INT4 rows need head_dim 128");
  if (rows == 0) return ok();
  if (!x || !codes || !scales) return fail(KV_ERR_INVALID, "null pointer");
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(codes) & 3) ||
      (reinterpret_cast<uintptr_t>(scales) & 3))
    return fail(KV_ERR_INVALID, "x must be 16-byte aligned, codes and scales 4-byte");
  if ((rows + kWarpsPerCta - 1) / kWarpsPerCta > 0x7FFFFFFF)
    return fail(KV_ERR_INVALID, "too many rows");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (out_dtype == KV_INT8)
    e = in_dtype == KV_BF16 ? dispatch_quantize_d<KV_BF16, KV_INT8>(head_dim, x, rows, codes, scales, st)
                            : dispatch_quantize_d<KV_FP16, KV_INT8>(head_dim, x, rows, codes, scales, st);
  else if (out_dtype == KV_INT4)
    e = in_dtype == KV_BF16 ? launch_quantize<128, KV_BF16, KV_INT4>(x, rows, codes, scales, st)
                            : launch_quantize<128, KV_FP16, KV_INT4>(x, rows, codes, scales, st);
  else
    e = in_dtype == KV_BF16 ? dispatch_quantize_d<KV_BF16, KV_FP8_E5M2>(head_dim, x, rows, codes, scales, st)
                            : dispatch_quantize_d<KV_FP16, KV_FP8_E5M2>(head_dim, x, rows, codes, scales, st);
  kv_status s = cuda_check(e, "kv_quantize launch");
  return s == KV_OK ? ok() : s;
}

kv_status kv_block_copy(kv_pool *pool, const int32_t *host_pairs, int32_t n_pairs,
                        kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (n_pairs < 0) return fail(KV_ERR_INVALID, "negative n_pairs");
  if (n_pairs == 0) return ok();
  if (!host_pairs) return fail(KV_ERR_INVALID, "null host_pairs");
  const int32_t nb = pool->d.num_blocks;
  std::vector<uint8_t> role(nb, 0);  // 1 = src, 2 = dst
  for (int32_t i = 0; i < n_pairs; ++i) {
    const int32_t s = host_pairs[2 * i], d = host_pairs[2 * i + 1];
    if (s < 0 || s >= nb || d < 0 || d >= nb)
      return fail(KV_ERR_INVALID, "pair %d (%d -> %d) has an id outside [0, %d)", i, s, d, nb);
    if (s == d) return fail(KV_ERR_INVALID, "pair %d copies block %d onto itself", i, s);
    role[s] |= 1;
  }
  for (int32_t i = 0; i < n_pairs; ++i) {
    const int32_t d = host_pairs[2 * i + 1];
    if (role[d] & 2) return fail(KV_ERR_INVALID, "block %d is the destination of two pairs", d);
    if (role[d] & 1) return fail(KV_ERR_INVALID, "block %d is both a source and a destination", d);
    role[d] |= 2;
  }
  const kv_pool_desc &dd = pool->d;
  const uint32_t kv_block = (uint32_t)dd.num_kv_heads * dd.block_size * pool->row_bytes;
  const uint32_t sc_block = (uint32_t)dd.num_kv_heads * dd.block_size * sizeof(float);
  const int regions = !has_scales(dd.cache_dtype) ? 2 : k_chan_scales(dd.cache_dtype) ? 3 : 4;
  cudaStream_t st = (cudaStream_t)stream;
  for (int32_t base = 0; base < n_pairs; base += kMaxPairsPerLaunch) {
    const int32_t n = std::min<int32_t>(kMaxPairsPerLaunch, n_pairs - base);
    CopyPairs cp;
    for (int32_t i = 0; i < n; ++i) {
      cp.src[i] = host_pairs[2 * (base + i)];
      cp.dst[i] = host_pairs[2 * (base + i) + 1];
    }
    dim3 grid(n, dd.num_layers, regions);
    block_copy_kernel<<<grid, 256, 0, st>>>(cp, pool->base, pool->lay.layer_stride,
                                            pool->lay.kv_stride, pool->lay.ksc_stride, kv_block,
                                            sc_block, k_chan_scales(dd.cache_dtype) ? 0 : 1);
    kv_status s = cuda_check(cudaGetLastError(), "kv_block_copy launch");
    if (s != KV_OK) return s;
  }
  return ok();
}

}  // extern "C"
