// Pool layout, host block allocator with reference counts, status word,
// error reporting and tensor-map creation.
//
// A pool is a set of fixed-size physical blocks carved out of one caller-owned
// device buffer; sequences take blocks on demand and give them back, and
// blocks shared by several sequences carry a reference count so that a write
// can copy them first [KV Cache 原理与 PagedAttention, §三 "工作方式" 1-3;
// bjdmk.com.cn/news/6246348, §3.1-§3.2].
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <unordered_map>

#include "internal.h"

namespace pagedkv {

static thread_local std::string g_last_error;

kv_status fail(kv_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

kv_status ok() {
  g_last_error.clear();
  return KV_OK;
}

kv_status cuda_check(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return KV_OK;
  return fail(KV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool compute_layout(const kv_pool_desc &d, Layout *out, std::string *why,
                    kv_status *code) {
  *code = KV_ERR_INVALID;
  if (d.num_layers <= 0 || d.num_blocks <= 0 || d.num_kv_heads <= 0 ||
      d.block_size <= 0 || d.head_dim <= 0) {
    *why = "num_layers, num_blocks, block_size, num_kv_heads, head_dim must be > 0";
    return false;
  }
  if (d.num_layers > 4096 || d.num_kv_heads > 1024) {
    *why = "num_layers must be <= 4096 and num_kv_heads <= 1024";
    return false;
  }
  *code = KV_ERR_UNSUPPORTED;
  if (d.block_size != 16 && d.block_size != 32) {
    *why = "block_size must be 16 or 32";
    return false;
  }
  if (d.head_dim != 64 && d.head_dim != 128) {
    *why = "head_dim must be 64 or 128";
    return false;
  }
  if (d.cache_dtype < KV_BF16 || d.cache_dtype > KV_INT8_KCHAN) {
    *why = "cache_dtype must be KV_BF16, KV_FP16, KV_FP8_E5M2, KV_INT8, KV_FP8_E5M2_CAST, KV_INT4 "
           "or KV_INT8_KCHAN";
    return false;
  }
  if (d.cache_dtype == KV_INT4 && d.head_dim != 128) {
    *why = "KV_INT4 caches need head_dim 128";
    return false;
  }
  const uint64_t rows = (uint64_t)d.num_blocks * d.num_kv_heads * d.block_size;
  if (rows >= (1ull << 31)) {  // TMA row coordinates are signed 32-bit
    *code = KV_ERR_INVALID;
    *why = "num_blocks * num_kv_heads * block_size must be < 2^31";
    return false;
  }
  Layout L;
  L.kv_bytes = rows * row_bytes_of(d.cache_dtype, d.head_dim);
  L.kv_stride = round_up(L.kv_bytes, 256);
  L.sc_bytes = has_scales(d.cache_dtype) ? rows * sizeof(float) : 0;
  L.sc_stride = round_up(L.sc_bytes, 256);
  // K scales: per-token rows like V, or the layer's [heads][head_dim] channel scales
  L.ksc_stride = k_chan_scales(d.cache_dtype)
                     ? round_up((uint64_t)d.num_kv_heads * d.head_dim * sizeof(float), 256)
                     : L.sc_stride;
  L.layer_stride = 2 * L.kv_stride + L.ksc_stride + L.sc_stride;
  L.status_off = L.layer_stride * (uint64_t)d.num_layers;
  L.total = L.status_off + 256;
  *out = L;
  *code = KV_OK;
  return true;
}

// --------------------------------------------------------------------------
// Tensor maps: one 2-D map per K / V region, rows = (block, head, token),
// columns = head_dim elements. The box is one 128-byte (or 64-byte) column
// slab of box_rows consecutive rows: the block_size rows of each of a group of
// heads of one block, which are contiguous in the pool. Boxes land in shared
// memory with the hardware swizzle so that the 8-row fragment loads the
// attention kernel issues are bank-conflict free.
// --------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn(std::string *why) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  static std::string err;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p,
                                                     12000, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) {
      err = std::string("cannot resolve cuTensorMapEncodeTiled: ") +
            cudaGetErrorString(e);
      (void)cudaGetLastError();
      return;
    }
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  if (!fn) *why = err;
  return fn;
}

static bool encode_region(const kv_pool *p, void *base, int box_rows, CUtensorMap *map,
                          std::string *why) {
  auto fn = encode_fn(why);
  if (!fn) return false;
  const kv_pool_desc &d = p->d;
  CUtensorMapDataType dt;
  switch (d.cache_dtype) {
    case KV_BF16: dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; break;
    case KV_FP16: dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT16; break;
    default: dt = CU_TENSOR_MAP_DATA_TYPE_UINT8; break;
  }
  const int elt = p->elt;
  const int row_bytes = p->row_bytes;
  const int slab_bytes = row_bytes >= 128 ? 128 : row_bytes;  // 128 or 64
  cuuint64_t gdim[2] = {(cuuint64_t)(row_bytes / elt),
                        (cuuint64_t)d.num_blocks * d.num_kv_heads * d.block_size};
  cuuint64_t gstride[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(slab_bytes / elt), (cuuint32_t)box_rows};
  cuuint32_t estride[2] = {1, 1};
  CUtensorMapSwizzle swz =
      slab_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = fn(map, dt, 2, base, gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[96];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    *why = buf;
    return false;
  }
  return true;
}

// 3-D view of a 16-bit region with 256-byte rows: (64 elements, row, slab),
// strides (row: 256 bytes, slab: 128 bytes); a (64, box_rows, 2) box lands in
// shared memory as [slab][row][128 bytes], 128-byte swizzled.
static bool encode_region_slabs(const kv_pool *p, void *base, int box_rows, CUtensorMap *map) {
  std::string why;
  auto fn = encode_fn(&why);
  if (!fn) return false;
  const kv_pool_desc &d = p->d;
  if ((d.cache_dtype != KV_BF16 && d.cache_dtype != KV_FP16) || p->row_bytes != 256) return false;
  const CUtensorMapDataType dt =
      d.cache_dtype == KV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  cuuint64_t gdim[3] = {64, (cuuint64_t)d.num_blocks * d.num_kv_heads * d.block_size, 2};
  cuuint64_t gstride[2] = {256, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 2};
  cuuint32_t estride[3] = {1, 1, 1};
  return fn(map, dt, 3, base, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4-D view of a 16-bit region with 256-byte rows: (64 elements, row within an
// 8-row group, slab, 8-row group), strides (256, 128, 2048 bytes); a (64, 8, 2,
// box_rows / 8) box lands in shared memory as [group][slab][8 rows][128 bytes],
// 128-byte swizzled: every 1024-byte swizzle atom is 8 rows of one slab.
static bool encode_region_groups(const kv_pool *p, void *base, int box_rows, CUtensorMap *map) {
  std::string why;
  auto fn = encode_fn(&why);
  if (!fn) return false;
  const kv_pool_desc &d = p->d;
  if ((d.cache_dtype != KV_BF16 && d.cache_dtype != KV_FP16) || p->row_bytes != 256 ||
      box_rows % 8 != 0)
    return false;
  const CUtensorMapDataType dt =
      d.cache_dtype == KV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t rows = (cuuint64_t)d.num_blocks * d.num_kv_heads * d.block_size;
  cuuint64_t gdim[4] = {64, 8, 2, rows / 8};
  cuuint64_t gstride[3] = {256, 128, 2048};
  cuuint32_t box[4] = {64, 8, 2, (cuuint32_t)(box_rows / 8)};
  cuuint32_t estride[4] = {1, 1, 1, 1};
  return fn(map, dt, 4, base, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool layer_maps(kv_pool *p, int layer, int box_rows, LayerMaps *out, kv_status *code) {
  std::lock_guard<std::mutex> g(p->map_mu);
  std::vector<LayerMaps> &v = p->maps[layer];
  for (const LayerMaps &m : v) {
    if (m.box_rows == box_rows) {
      *out = m;
      *code = KV_OK;
      return true;
    }
  }
  LayerMaps m;
  std::string why;
  if (!encode_region(p, layer_k(p, layer), box_rows, &m.k, &why) ||
      !encode_region(p, layer_v(p, layer), box_rows, &m.v, &why)) {
    *code = fail(KV_ERR_CUDA, "tensor map for layer %d: %s", layer, why.c_str());
    return false;
  }
  m.v_blk_ok = encode_region_slabs(p, layer_v(p, layer), box_rows, &m.v_blk);
  m.k_grp_ok = encode_region_groups(p, layer_k(p, layer), box_rows, &m.k_grp);
  m.box_rows = box_rows;
  v.push_back(m);
  *out = m;
  *code = KV_OK;
  return true;
}

}  // namespace pagedkv

using namespace pagedkv;

extern "C" {

const char *kv_last_error(void) { return g_last_error.c_str(); }

const char *kv_version(void) { return "pagedkv 0.2 (sm_100a)"; }

kv_status kv_pool_required_bytes(const kv_pool_desc *desc, uint64_t *bytes) {
  if (!desc || !bytes) return fail(KV_ERR_INVALID, "null argument");
  Layout L;
  std::string why;
  kv_status code;
  if (!compute_layout(*desc, &L, &why, &code)) return fail(code, "%s", why.c_str());
  *bytes = L.total;
  return ok();
}

kv_status kv_pool_create(const kv_pool_desc *desc, void *device_base, uint64_t bytes,
                         kv_pool **out) {
  if (!desc || !out) return fail(KV_ERR_INVALID, "null argument");
  *out = nullptr;
  Layout L;
  std::string why;
  kv_status code;
  if (!compute_layout(*desc, &L, &why, &code)) return fail(code, "%s", why.c_str());
  if (!device_base) return fail(KV_ERR_INVALID, "device_base is null");
  if (((uintptr_t)device_base & 255) != 0)
    return fail(KV_ERR_INVALID, "device_base must be 256-byte aligned");
  if (bytes < L.total)
    return fail(KV_ERR_INVALID, "buffer of %llu bytes < required %llu",
                (unsigned long long)bytes, (unsigned long long)L.total);
  kv_pool *p = new kv_pool();
  p->d = *desc;
  p->base = static_cast<char *>(device_base);
  p->bytes = bytes;
  p->lay = L;
  p->elt = elem_bytes(desc->cache_dtype);
  p->row_bytes = row_bytes_of(desc->cache_dtype, desc->head_dim);
  p->ref.assign(desc->num_blocks, 0);
  p->free_stack.resize(desc->num_blocks);
  for (int32_t i = 0; i < desc->num_blocks; ++i)
    p->free_stack[i] = desc->num_blocks - 1 - i;  // block 0 is handed out first
  p->maps.resize(desc->num_layers);
  *out = p;
  return ok();
}

kv_status kv_pool_destroy(kv_pool *pool) {
  delete pool;
  return ok();
}

kv_status kv_pool_layer_ptrs(const kv_pool *pool, int32_t layer, void **k, void **v,
                             float **k_scale, float **v_scale) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (layer < 0 || layer >= pool->d.num_layers)
    return fail(KV_ERR_INVALID, "layer %d out of range", layer);
  if (k) *k = layer_k(pool, layer);
  if (v) *v = layer_v(pool, layer);
  if (k_scale) *k_scale = layer_ks(pool, layer);
  if (v_scale) *v_scale = layer_vs(pool, layer);
  return ok();
}

kv_status kv_pool_status_ptr(const kv_pool *pool, int32_t **status) {
  if (!pool || !status) return fail(KV_ERR_INVALID, "null argument");
  *status = status_word(pool);
  return ok();
}

kv_status kv_pool_status_clear(kv_pool *pool, kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  kv_status s = cuda_check(
      cudaMemsetAsync(status_word(pool), 0, sizeof(int32_t), (cudaStream_t)stream),
      "status clear");
  return s == KV_OK ? ok() : s;
}

kv_status kv_pool_status(kv_pool *pool, kv_stream_t stream, int32_t *host_bits) {
  if (!pool || !host_bits) return fail(KV_ERR_INVALID, "null argument");
  int32_t v = 0;
  kv_status s = cuda_check(cudaMemcpyAsync(&v, status_word(pool), sizeof(int32_t),
                                           cudaMemcpyDeviceToHost, (cudaStream_t)stream),
                           "status read");
  if (s != KV_OK) return s;
  s = cuda_check(cudaStreamSynchronize((cudaStream_t)stream), "status read sync");
  if (s != KV_OK) return s;
  *host_bits = v;
  return ok();
}

// ---------------------------------------------------------------- allocator

kv_status kv_alloc_blocks(kv_pool *pool, int32_t n, int32_t *out_ids) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (n < 0) return fail(KV_ERR_INVALID, "negative block count");
  if (n > 0 && !out_ids) return fail(KV_ERR_INVALID, "null out_ids");
  std::lock_guard<std::mutex> g(pool->mu);
  if ((size_t)n > pool->free_stack.size())
    return fail(KV_ERR_OOM, "asked for %d blocks, %zu free", n, pool->free_stack.size());
  for (int32_t i = 0; i < n; ++i) {
    int32_t id = pool->free_stack.back();
    pool->free_stack.pop_back();
    pool->ref[id] = 1;
    out_ids[i] = id;
  }
  return ok();
}

// Checks that every id is allocated often enough to take `per_id` references
// away (a list may name one block several times).
static kv_status check_allocated(kv_pool *pool, int32_t n, const int32_t *ids,
                                 bool dropping) {
  std::unordered_map<int32_t, int32_t> count;
  for (int32_t i = 0; i < n; ++i) {
    int32_t id = ids[i];
    if (id < 0 || id >= pool->d.num_blocks)
      return fail(KV_ERR_INVALID, "block id %d out of range [0, %d)", id,
                  pool->d.num_blocks);
    if (pool->ref[id] == 0) return fail(KV_ERR_INVALID, "block %d is not allocated", id);
    if (dropping && ++count[id] > pool->ref[id])
      return fail(KV_ERR_INVALID, "block %d freed more times than referenced", id);
  }
  return KV_OK;
}

kv_status kv_free_blocks(kv_pool *pool, int32_t n, const int32_t *ids) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (n < 0) return fail(KV_ERR_INVALID, "negative block count");
  if (n > 0 && !ids) return fail(KV_ERR_INVALID, "null ids");
  std::lock_guard<std::mutex> g(pool->mu);
  kv_status s = check_allocated(pool, n, ids, true);
  if (s != KV_OK) return s;
  for (int32_t i = 0; i < n; ++i) {
    int32_t id = ids[i];
    if (pool->ref[id] == 2) pool->shared--;
    if (--pool->ref[id] == 0) pool->free_stack.push_back(id);
  }
  return ok();
}

kv_status kv_share_blocks(kv_pool *pool, int32_t n, const int32_t *ids) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (n < 0) return fail(KV_ERR_INVALID, "negative block count");
  if (n > 0 && !ids) return fail(KV_ERR_INVALID, "null ids");
  std::lock_guard<std::mutex> g(pool->mu);
  kv_status s = check_allocated(pool, n, ids, false);
  if (s != KV_OK) return s;
  for (int32_t i = 0; i < n; ++i) {
    int32_t id = ids[i];
    if (++pool->ref[id] == 2) pool->shared++;
  }
  return ok();
}

kv_status kv_cow_prepare(kv_pool *pool, int32_t block, int32_t *new_block) {
  if (!pool || !new_block) return fail(KV_ERR_INVALID, "null argument");
  std::lock_guard<std::mutex> g(pool->mu);
  kv_status s = check_allocated(pool, 1, &block, false);
  if (s != KV_OK) return s;
  if (pool->ref[block] == 1) {
    *new_block = block;
    return ok();
  }
  if (pool->free_stack.empty()) return fail(KV_ERR_OOM, "no free block for copy-on-write");
  int32_t id = pool->free_stack.back();
  pool->free_stack.pop_back();
  pool->ref[id] = 1;
  if (pool->ref[block] == 2) pool->shared--;
  pool->ref[block]--;
  *new_block = id;
  return ok();
}

kv_status kv_block_refcount(const kv_pool *pool, int32_t block, int32_t *ref) {
  if (!pool || !ref) return fail(KV_ERR_INVALID, "null argument");
  if (block < 0 || block >= pool->d.num_blocks)
    return fail(KV_ERR_INVALID, "block id %d out of range", block);
  std::lock_guard<std::mutex> g(const_cast<kv_pool *>(pool)->mu);
  *ref = pool->ref[block];
  return ok();
}

kv_status kv_pool_stats(const kv_pool *pool, int32_t *used, int32_t *free_,
                        int32_t *shared) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  std::lock_guard<std::mutex> g(const_cast<kv_pool *>(pool)->mu);
  int32_t f = (int32_t)pool->free_stack.size();
  if (used) *used = pool->d.num_blocks - f;
  if (free_) *free_ = f;
  if (shared) *shared = pool->shared;
  return ok();
}

}  // extern "C"
