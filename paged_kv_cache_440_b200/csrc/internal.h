// Host-side internals shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "pagedkv.h"

namespace pagedkv {

// Device status word bit set when a bounded wait in a kernel gives up.
constexpr int32_t kDevErrTimeout = 8;

// Element size of the tensor maps (INT4 rows are addressed as bytes).
inline int elem_bytes(int dtype) {
  return (dtype == KV_BF16 || dtype == KV_FP16) ? 2 : 1;
}
// Bytes of one (token, head) row of head_dim values.
inline int row_bytes_of(int dtype, int head_dim) {
  return dtype == KV_INT4 ? head_dim / 2 : head_dim * elem_bytes(dtype);
}
// 1-byte codes (read through the code paths of the kernels)
inline bool is_quant(int dtype) {
  return dtype == KV_INT8 || dtype == KV_FP8_E5M2 || dtype == KV_FP8_E5M2_CAST ||
         dtype == KV_INT4 || dtype == KV_INT8_KCHAN;
}
// codes with fp32 scales (scale regions in the pool): per-token-head rows for
// V, and for K too unless the keys use channel scales
inline bool has_scales(int dtype) {
  return dtype == KV_INT8 || dtype == KV_FP8_E5M2 || dtype == KV_INT4 || dtype == KV_INT8_KCHAN;
}
// keys with one fixed scale per (kv head, channel) of the layer
inline bool k_chan_scales(int dtype) { return dtype == KV_INT8_KCHAN; }
inline uint64_t round_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

// Byte offsets of one layer's regions inside the pool buffer.
struct Layout {
  uint64_t kv_bytes;      // one K (or V) region
  uint64_t kv_stride;     // kv_bytes rounded to 256
  uint64_t sc_bytes;      // the V-scale region (0 for 16-bit caches)
  uint64_t sc_stride;
  uint64_t ksc_stride;    // the K-scale region (per-token rows, or channel scales)
  uint64_t layer_stride;  // K + V (+ K scale + V scale), each 256-aligned
  uint64_t status_off;    // 256-byte status region after the last layer
  uint64_t total;
};

// Tensor maps of one layer's K and V regions (built on first use; encoding
// needs the CUDA driver, which a GPU-less host may not have).
struct LayerMaps {
  CUtensorMap k;
  CUtensorMap v;
  // V as [row][slab of 128 bytes] with the slab as the outer coordinate: one
  // box brings a block-head's rows of every slab, landing slab-major (16-bit
  // caches with 256-byte rows only; v_blk_ok is false where the driver
  // declined the encoding)
  CUtensorMap v_blk;
  bool v_blk_ok = false;
  // K as (64 elements, 8 rows, slab, 8-row group): one box brings a
  // block-head's rows of both slabs, landing as [8-row group][slab][8 rows][128
  // bytes], so that the 8-row groups of consecutive blocks sit 2048 bytes
  // apart (same conditions as v_blk)
  CUtensorMap k_grp;
  bool k_grp_ok = false;
  int box_rows = 0;  // rows per box the maps were encoded for (0 = none yet)
};

}  // namespace pagedkv

struct kv_pool {
  kv_pool_desc d;
  char *base = nullptr;
  uint64_t bytes = 0;
  pagedkv::Layout lay;
  int elt = 2;
  int row_bytes = 0;  // bytes of one (token, head) row

  std::mutex mu;                    // guards the allocator state
  std::vector<int32_t> ref;         // refcount per block
  std::vector<int32_t> free_stack;  // free ids; the top is handed out next
  int32_t shared = 0;               // blocks with refcount >= 2

  std::mutex map_mu;                // guards the tensor-map cache
  std::vector<std::vector<pagedkv::LayerMaps>> maps;  // per layer, one per box height
};

namespace pagedkv {

kv_status fail(kv_status s, const char *fmt, ...);
kv_status ok();
kv_status cuda_check(cudaError_t e, const char *what);

bool compute_layout(const kv_pool_desc &d, Layout *out, std::string *why,
                    kv_status *code);

inline char *layer_k(const kv_pool *p, int layer) {
  return p->base + (uint64_t)layer * p->lay.layer_stride;
}
inline char *layer_v(const kv_pool *p, int layer) {
  return layer_k(p, layer) + p->lay.kv_stride;
}
inline float *layer_ks(const kv_pool *p, int layer) {
  return p->lay.sc_bytes ? (float *)(layer_v(p, layer) + p->lay.kv_stride) : nullptr;
}
inline float *layer_vs(const kv_pool *p, int layer) {
  return p->lay.sc_bytes ? (float *)((char *)layer_ks(p, layer) + p->lay.ksc_stride)
                         : nullptr;
}
inline int32_t *status_word(const kv_pool *p) {
  return (int32_t *)(p->base + p->lay.status_off);
}

// Launch `kern` on `st` so that it may be scheduled while the previous kernel
// in the stream is still running (programmatic stream serialization). The
// kernel must call grid_dependency_wait() before reading its inputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Tensor maps for the layer's K and V regions with boxes of box_rows rows,
// copied to *out (encoded on first use, then cached per box height); false +
// message on failure.
bool layer_maps(kv_pool *p, int layer, int box_rows, LayerMaps *out, kv_status *code);

// Shared-prefix pass of a cascade decode step (attn_prefill.cu): the decode
// query of each of num_seqs sequences (q [num_seqs][Hq][D], the cache dtype)
// attends the prefix_blocks blocks of prefix_table, all positions, no causal
// limit; writes each (sequence, head)'s unnormalised output to pre_o
// ([num_seqs][Hq][D] fp32) and its (maximum, sum), base 2, to pre_ml. The
// caller has checked the cache dtype, the head counts and the pointers.
kv_status prefix_pass(kv_pool *pool, int layer, const void *q, int num_seqs, int num_q_heads,
                      const int32_t *prefix_table, int prefix_blocks, float scale, float *pre_o,
                      float *pre_ml, cudaStream_t st);

}  // namespace pagedkv
