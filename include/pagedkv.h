/*
 * pagedkv.h -- C ABI of a paged KV-cache library for single-token decode on
 * NVIDIA B200 (sm_100a).
 *
 * What the library does, and where the operations are defined:
 *
 *   The KV cache of every sequence is cut into fixed-size blocks of
 *   block_size tokens that live anywhere in one preallocated pool; a per-sequence
 *   block table maps logical block i to physical block p; blocks are handed out
 *   on demand and returned when done; attention gathers the scattered blocks
 *   back into the logical sequence.
 *     [KV Cache 原理与 PagedAttention, §三 "工作方式" 1-4;
 *      aiworkagent.org q17, "Block Table", "Block Size", "KV Memory Pool"]
 *   Each decode step computes only the new token's K and V and appends them to
 *   the cache; the new query attends over every cached token.
 *     [KV Cache 原理与 PagedAttention, §一; bjdmk.com.cn/news/6246348, §2.1]
 *   Attention is softmax(q K^T * scale) V; several query heads may share one
 *   KV head (GQA / MQA).
 *     [bjdmk.com.cn/news/6246348, §2.1; KV Cache 原理与 PagedAttention, §一 GQA/MQA]
 *   Requests with a common prefix share its physical blocks; a write into a
 *   shared block first copies it (copy-on-write).
 *     [bjdmk.com.cn/news/6246348, §3.2]
 *   The cache may be stored as INT8 or FP8-E5M2 with one fp32 scale per
 *   (token, KV head), dequantized inside the attention kernel.
 *     [KV Cache 原理与 PagedAttention, §四; bjdmk.com.cn/news/6246348, §5.2, §5.3]
 *
 * Conventions for every call:
 *   - Device pointers are borrowed. The caller allocates all device memory
 *     (the pool, inputs, outputs, split-K workspace) and keeps it alive until
 *     the work queued on the stream has finished. No call allocates device memory.
 *   - Device work is queued on the given stream; calls return after enqueueing.
 *     A launch failure returns KV_ERR_CUDA.
 *   - Arguments are validated on the host before anything is queued; a
 *     rejected call queues nothing and returns KV_ERR_INVALID or
 *     KV_ERR_UNSUPPORTED. kv_last_error() then describes the problem.
 *   - Values only the device can see (block ids read from a block table,
 *     context lengths, slots) are range-checked in the kernels. A bad value
 *     never causes an out-of-bounds access: the affected row is skipped (append)
 *     or contributes nothing (attention), and a bit is set in the pool's device
 *     status word (see kv_pool_status).
 *   - Tensors are dense and row-major; the shapes below list dimensions from
 *     outermost to innermost.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st *kv_stream_t;

typedef enum {
  KV_OK = 0,
  KV_ERR_INVALID = 1,      /* bad argument (null pointer, out-of-range id, ...) */
  KV_ERR_OOM = 2,          /* the block pool has fewer free blocks than asked   */
  KV_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed       */
  KV_ERR_UNSUPPORTED = 4   /* valid but not implemented (e.g. head_dim 96)      */
} kv_status;

typedef enum {
  KV_BF16 = 0,
  KV_FP16 = 1,
  KV_FP8_E5M2 = 2,         /* 1 sign, 5 exponent (bias 15), 2 mantissa bits     */
  KV_INT8 = 3,             /* two's complement, codes in [-127, 127]            */
  KV_FP8_E5M2_CAST = 4,    /* E5M2 codes cast from the values with no scale     */
  KV_INT4 = 5,             /* 4-bit codes in [-7, 7], two per byte (element 2i  */
                           /* in the low nibble), head_dim 128 only             */
  KV_INT8_KCHAN = 6        /* INT8 keys with one fixed fp32 scale per (kv head, */
                           /* channel), INT8 values with per-token-head scales  */
} kv_dtype;

/* Bits of the device status word. */
enum {
  KV_DEVERR_BLOCK_ID = 1,  /* a block-table entry outside [0, num_blocks)        */
  KV_DEVERR_CONTEXT = 2,   /* a context length < 0 or beyond the table/maximum   */
  KV_DEVERR_SLOT = 4,      /* a slot >= num_blocks * block_size                  */
  KV_DEVERR_TIMEOUT = 8    /* a kernel gave up waiting for its own tile loads    */
};

typedef struct {
  int32_t num_layers;      /* >= 1                                              */
  int32_t num_blocks;      /* physical blocks per layer, >= 1                   */
  int32_t block_size;      /* tokens per block: 16 or 32                        */
  int32_t num_kv_heads;    /* >= 1                                              */
  int32_t head_dim;        /* 64 or 128                                         */
  int32_t cache_dtype;     /* a kv_dtype                                        */
} kv_pool_desc;

typedef struct kv_pool kv_pool;   /* opaque host object */

/* ------------------------------------------------------------------------ */
/* Pool                                                                      */
/* ------------------------------------------------------------------------ */

/* Bytes of device memory a pool with this description needs.
 *
 * Layout of the caller's buffer, for each layer in order, every region
 * starting on a 256-byte boundary:
 *   K       [num_blocks][num_kv_heads][block_size][head_dim]  cache_dtype
 *   V       same
 *   K scale [num_blocks][num_kv_heads][block_size]  fp32   (INT8 / E5M2 / INT4)
 *           [num_kv_heads][head_dim]                fp32   (INT8_KCHAN: the
 *           layer's channel scales, written by the caller before any append;
 *           per-channel granularity [bjdmk.com.cn/news/6246348, §5.2])
 *   V scale [num_blocks][num_kv_heads][block_size]  fp32   (INT8 / E5M2 / INT4 /
 *                                                            INT8_KCHAN)
 * followed by one 256-byte status region. One (block, head) tile of K or V is
 * contiguous (block_size * head_dim elements). K and V of a layer take exactly
 * 2 * num_kv_heads * head_dim * elem_bytes * (num_blocks * block_size) bytes,
 * the per-layer KV size formula of the pages applied to the pool's capacity
 * [KV Cache 原理与 PagedAttention, §一 "显存占用公式"].
 * Errors: KV_ERR_INVALID for a null pointer or a non-positive size field,
 * KV_ERR_UNSUPPORTED for a block_size, head_dim or dtype outside the lists above. */
kv_status kv_pool_required_bytes(const kv_pool_desc *desc, uint64_t *bytes);

/* Create the host-side pool object over a caller-owned device buffer: the
 * preallocated pool of fixed-size physical blocks that every sequence's cache
 * is cut into [KV Cache 原理与 PagedAttention, §三 "工作方式" 1; aiworkagent.org
 * q17, "KV Memory Pool"].
 * device_base: 256-byte aligned device pointer to >= kv_pool_required_bytes
 * bytes; borrowed, never freed by the library. Its contents are not touched;
 * the caller zeroes the status region (kv_pool_status_clear) before first use.
 * All blocks start free (refcount 0).
 * Errors: KV_ERR_INVALID (null, misaligned, too small), KV_ERR_UNSUPPORTED. */
kv_status kv_pool_create(const kv_pool_desc *desc, void *device_base,
                         uint64_t bytes, kv_pool **out);

/* Free the host object (the block pool's bookkeeping [KV Cache 原理与
 * PagedAttention, §三 "工作方式" 3]). Does not touch device memory. */
kv_status kv_pool_destroy(kv_pool *pool);

/* Device addresses of one layer's regions (the layout of kv_pool_required_bytes;
 * per-layer K and V as in the pages' KV size formula [KV Cache 原理与
 * PagedAttention, §一 "显存占用公式"]). k_scale / v_scale are set to NULL
 * for 16-bit and scale-less caches. For KV_INT8_KCHAN k_scale is the layer's
 * [num_kv_heads][head_dim] channel-scale array (caller-written). Any output
 * pointer may be NULL if not wanted. */
kv_status kv_pool_layer_ptrs(const kv_pool *pool, int32_t layer, void **k,
                             void **v, float **k_scale, float **v_scale);

/* Device address of the pool's int32 status word (bits KV_DEVERR_*). */
kv_status kv_pool_status_ptr(const kv_pool *pool, int32_t **status);

/* Queue a reset of the status word to 0 on the stream. */
kv_status kv_pool_status_clear(kv_pool *pool, kv_stream_t stream);

/* Copy the status word to *host_bits after the stream's queued work has
 * finished (synchronizes the stream). */
kv_status kv_pool_status(kv_pool *pool, kv_stream_t stream, int32_t *host_bits);

/* ------------------------------------------------------------------------ */
/* Host block allocator with reference counts                                */
/* [KV Cache 原理与 PagedAttention, §三 "工作方式" 3; bjdmk.com.cn/news/6246348,   */
/*  §3.1-§3.2]. Thread-safe; no device work.                                  */
/* ------------------------------------------------------------------------ */

/* Take n free blocks (refcount 0 -> 1) and write their ids to out_ids[0..n).
 * KV_ERR_OOM, with nothing taken, when fewer than n blocks are free. */
kv_status kv_alloc_blocks(kv_pool *pool, int32_t n, int32_t *out_ids);

/* Drop one reference from each listed block; a block reaching 0 is free again.
 * KV_ERR_INVALID, with nothing changed, if any id is out of range or free. */
kv_status kv_free_blocks(kv_pool *pool, int32_t n, const int32_t *ids);

/* Add one reference to each listed (allocated) block: sharing a prefix, or
 * forking a sequence. KV_ERR_INVALID, nothing changed, for a free/bad id. */
kv_status kv_share_blocks(kv_pool *pool, int32_t n, const int32_t *ids);

/* Before writing into `block`: if it is shared (refcount > 1), take a fresh
 * block, drop one reference from `block`, and return the fresh id in
 * *new_block; the caller then copies the contents with kv_block_copy and
 * points its block table at the copy. If the block is exclusively owned,
 * *new_block = block and nothing changes. KV_ERR_OOM when no block is free. */
kv_status kv_cow_prepare(kv_pool *pool, int32_t block, int32_t *new_block);

/* Current reference count of one block. */
kv_status kv_block_refcount(const kv_pool *pool, int32_t block, int32_t *ref);

/* used = blocks with refcount >= 1, free_ = refcount 0, shared = refcount >= 2
 * (the cache-usage figures a serving system monitors
 * [KV Cache 原理与 PagedAttention, §六]). Any pointer may be NULL. */
kv_status kv_pool_stats(const kv_pool *pool, int32_t *used, int32_t *free_,
                        int32_t *shared);

/* ------------------------------------------------------------------------ */
/* Append (reshape_and_cache), quantize, copy-on-write block copy           */
/* ------------------------------------------------------------------------ */

/* Write each new token's K and V rows into the slot it maps to: each decode
 * step computes only the new token's K and V and appends them to the cache end
 * [KV Cache 原理与 PagedAttention, §一; bjdmk.com.cn/news/6246348, §2.1], which in
 * a paged cache is a row of the block the sequence's table names for that
 * position [KV Cache 原理与 PagedAttention, §三 "工作方式" 2].
 * k_new, v_new: device [num_tokens][num_kv_heads][head_dim] of in_dtype
 *   (KV_BF16 or KV_FP16), 16-byte aligned.
 * slot_mapping: device int64 [num_tokens]; slot = physical_block * block_size
 *   + row. A negative slot skips the token; a slot >= num_blocks * block_size
 *   skips it and sets KV_DEVERR_SLOT. Slots must be distinct (duplicates race).
 * 16-bit caches: in_dtype must equal the cache dtype; the rows are copied
 *   bit for bit.
 * INT8 / E5M2 / INT4 caches: each (token, head) row x of head_dim values is
 *   quantized as kv_quantize does and its code row and fp32 scale are stored.
 * E5M2_CAST caches: each value is cast to E5M2 (saturating round to nearest
 *   even) and stored; no scale.
 * Errors: KV_ERR_INVALID (bad layer, null, misaligned, num_tokens < 0),
 *   KV_ERR_UNSUPPORTED (dtype combination), KV_ERR_CUDA. */
kv_status kv_append(kv_pool *pool, int32_t layer, const void *k_new,
                    const void *v_new, int32_t in_dtype,
                    const int64_t *slot_mapping, int32_t num_tokens,
                    kv_stream_t stream);

/* KV_INT8_KCHAN caches: each key value k of head h, channel c is stored as
 *   clamp(round-half-even(fl32(k / s[h][c])), -127, 127) (0 where s[h][c] is
 *   0) with s the layer's channel scales; each V row as for KV_INT8.
 *
 * Per-row symmetric absmax quantization [bjdmk.com.cn/news/6246348, §5.2:
 * one scale per token per head]:
 *   a = max|x|; scale = fl32(a / QMAX) (QMAX 127 for INT8, 57344 for E5M2);
 *   code = round-half-even(fl32(x / scale)), clamped to [-127, 127] (INT8) or
 *   [-7, 7] (INT4, QMAX 7: the pages' most aggressive KV row), or rounded to
 *   E5M2 with saturation to +-57344; a == 0 gives scale 0, codes 0.
 *   Both divisions are IEEE fp32 divisions, so results are bit-reproducible.
 * x: device [rows][head_dim] of in_dtype (BF16 / FP16), 16-byte aligned.
 * codes: device [rows][head_dim] bytes ([rows][head_dim / 2] for INT4: element
 *   2i in the low nibble of byte i); scales: device fp32 [rows].
 * head_dim: 64 or 128 (128 for INT4). out_dtype: KV_INT8, KV_FP8_E5M2 or KV_INT4. */
kv_status kv_quantize(const void *x, int32_t in_dtype, int64_t rows,
                      int32_t head_dim, int32_t out_dtype, void *codes,
                      float *scales, kv_stream_t stream);

/* Copy whole physical blocks, every layer, K and V (and the scales of a
 * quantized cache): block dst := block src for each pair
 * [bjdmk.com.cn/news/6246348, §3.2, copy-on-write].
 * host_pairs: HOST int32 [n_pairs][2] = {src, dst}. The pairs must be
 * disjoint: src != dst, no dst repeated, no dst that is also a src, all ids in
 * [0, num_blocks); otherwise KV_ERR_INVALID and nothing is queued. The pair
 * list is passed to the kernel by value (no device staging buffer). */
kv_status kv_block_copy(kv_pool *pool, const int32_t *host_pairs,
                        int32_t n_pairs, kv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Paged decode attention                                                    */
/* ------------------------------------------------------------------------ */
/*
 * For sequence b (context length L_b, block table row bt[b]) and query head h,
 * with g = h / (num_q_heads / num_kv_heads):
 *   out[b][h] = sum_t softmax_t(scale * q[b][h] . K_g[t]) V_g[t],  t in [0, L_b)
 * where position t lives in row t % block_size of physical block
 * bt[b][t / block_size]. L_b = 0 gives a zero output. For INT8 / E5M2 caches,
 * K_g[t] = code * k_scale and V_g[t] = code * v_scale (dequantized in-kernel).
 * [bjdmk.com.cn/news/6246348, §2.1; KV Cache 原理与 PagedAttention, §三 工作方式 4]
 *
 * Work split (split-K): a unit is one sequence and a group of its KV heads
 * (with their query heads); its positions are the sequence's KV blocks. The
 * positions of all units are laid end to end and divided evenly among
 * num_ctas persistent CTAs, so every CTA reads the same number of blocks
 * whatever the mix of lengths. A unit that one CTA covers entirely is
 * finished by it; a unit cut by CTA boundaries leaves a running max m, sum l
 * and unnormalised output o per piece, which the merge combines:
 * out = sum_i e^(m_i - M) o_i / sum_i e^(m_i - M) l_i, M = max_i m_i.
 *
 * Common arguments:
 *   q       device [num_seqs][num_q_heads][head_dim], q_dtype, 16-byte aligned.
 *           16-bit caches need q_dtype == cache dtype; INT8/E5M2 caches take
 *           KV_BF16 or KV_FP16 queries.
 *   out     device [num_seqs][num_q_heads][head_dim], q_dtype, 16-byte aligned.
 *   block_tables  device int32 [num_seqs][max_blocks_per_seq].
 *   context_lens  device int32 [num_seqs]; each must satisfy
 *           0 <= L_b <= min(max_context, max_blocks_per_seq * block_size),
 *           else KV_DEVERR_CONTEXT is set and that sequence's output is 0.
 *   max_context   host upper bound on every L_b.
 *   num_ctas      CTAs the work is divided among: 0 = one per multiprocessor
 *           of the current device (the default), else 1 .. 65535.
 *   workspace     device, 256-byte aligned, >= paged_attn_workspace_bytes
 *           bytes for the same num_seqs, num_q_heads and num_ctas. Holds the
 *           per-unit bookkeeping and the split partials between the two
 *           kernels; its contents are scratch and need no initialisation.
 *           Concurrent calls must use separate workspaces.
 */

/* Workspace bytes for these sizes: 16 B per unit plus 2 x 64 x (head_dim + 2)
 * fp32 per CTA, each part rounded up to 256 B. num_ctas = 0 queries the
 * current device (KV_ERR_CUDA without one). */
kv_status paged_attn_workspace_bytes(const kv_pool *pool, int32_t num_seqs,
                                     int32_t num_q_heads, int32_t num_ctas,
                                     uint64_t *bytes);

/* The CTA count used when num_ctas is 0 (multiprocessors of the current
 * device). */
kv_status paged_attn_default_ctas(const kv_pool *pool, int32_t *num_ctas);

/* Full decode attention: paged_attn_partition followed by paged_attn_merge on
 * the same stream (the merge kernel is launched so that it is scheduled while
 * the attention kernel drains). */
kv_status paged_attn_decode(kv_pool *pool, int32_t layer, const void *q,
                            int32_t q_dtype, int32_t num_seqs,
                            int32_t num_q_heads, const int32_t *block_tables,
                            int32_t max_blocks_per_seq,
                            const int32_t *context_lens, int32_t max_context,
                            float scale, void *out, int32_t num_ctas,
                            void *workspace, uint64_t workspace_bytes,
                            kv_stream_t stream);

/* paged_attn_decode for callers that cannot allocate a workspace -- for
 * example a serving process that has given all free GPU memory to its KV pool
 * and admits no further allocation, or an application reaching this library
 * through a plugin or foreign-function layer with no device allocator. The
 * pages have no counterpart; this is a convenience of this library.
 * The split-K scratch lives in a 16 MiB array inside the library's own device
 * memory (every GPU that loads the library holds it until the process exits).
 * The first call on each device looks up that array's device address with the
 * device current; make that first call before any stream capture. The stream
 * must belong to the current device (else KV_ERR_INVALID), and the looked-up
 * address does not survive a reset of the device (cudaDeviceReset): do not use
 * this entry point across one. Calls whose
 * scratch would exceed 16 MiB (paged_attn_workspace_bytes for the same
 * num_seqs, num_q_heads, num_ctas) return KV_ERR_INVALID and queue nothing.
 * Every call uses the same array, so calls that overlap on the GPU (on
 * different streams, or on one device from several threads without ordering)
 * race and corrupt each other's results; serialize them. No call allocates.
 * Other arguments and results are those of paged_attn_decode. */
kv_status paged_attn_decode_static(kv_pool *pool, int32_t layer, const void *q,
                                   int32_t q_dtype, int32_t num_seqs,
                                   int32_t num_q_heads, const int32_t *block_tables,
                                   int32_t max_blocks_per_seq,
                                   const int32_t *context_lens,
                                   int32_t max_context, float scale, void *out,
                                   int32_t num_ctas, kv_stream_t stream);

/* A decode step with the append folded into the attention kernel: for every
 * sequence b with a valid length L_b > 0, the new token's rows k_new[b] and
 * v_new[b] are written at position L_b - 1, i.e. row (L_b - 1) % block_size of
 * block block_tables[b][(L_b - 1) / block_size] (quantized exactly as
 * kv_append does for INT8 / E5M2 caches), and the attention over positions
 * 0 .. L_b - 1 uses them. The same results as kv_append with those slots
 * followed by paged_attn_decode, with one kernel fewer. Only the new token's
 * K and V are computed each step and put at the cache end
 * [KV Cache 原理与 PagedAttention, §一].
 * k_new, v_new: device [num_seqs][num_kv_heads][head_dim] of q_dtype (for a
 *   16-bit cache, its own dtype: rows are copied bit for bit), 16-byte aligned.
 * Needs num_q_heads / num_kv_heads <= 8 (else KV_ERR_UNSUPPORTED: use
 * kv_append and paged_attn_decode). Other arguments as paged_attn_decode. */
kv_status paged_attn_decode_append(kv_pool *pool, int32_t layer, const void *q,
                                   const void *k_new, const void *v_new,
                                   int32_t q_dtype, int32_t num_seqs,
                                   int32_t num_q_heads, const int32_t *block_tables,
                                   int32_t max_blocks_per_seq,
                                   const int32_t *context_lens,
                                   int32_t max_context, float scale, void *out,
                                   int32_t num_ctas, void *workspace,
                                   uint64_t workspace_bytes, kv_stream_t stream);

/* A decode step for sequences that share a prompt prefix: the first
 * prefix_blocks entries of every row of block_tables are the same block ids,
 * the shared prefix's blocks [bjdmk.com.cn/news/6246348, §3.2: requests with
 * one system prompt map it to the same physical blocks]. Results are those of
 * paged_attn_decode_append (k_new, v_new given) or paged_attn_decode (both
 * null) on the same arguments, within their tolerance. The work is split three
 * ways; the pages give no method for it.
 *   1. The shared positions 0 .. P - 1 (P = prefix_blocks * block_size) for
 *      all sequences at once. Per kv head this is a dense (sequences x group)
 *      by P contraction, run on the tensor cores (the chunked-prefill kernel,
 *      without its causal limit); its per-(sequence, head) partials go to the
 *      workspace. Row 0 of block_tables names the prefix's blocks.
 *   2. Each sequence's positions P .. L_b - 1, with the step's append, through
 *      the decode kernel.
 *   3. The merge, with the prefix partial folded in.
 * 16-bit caches only (a 1-byte or 4-bit cache: KV_ERR_UNSUPPORTED);
 * q_dtype must be the cache dtype. At most 128 query heads per kv head (8 with
 * an append), else KV_ERR_UNSUPPORTED.
 *   prefix_blocks  1 <= prefix_blocks < max_blocks_per_seq, and
 *                  P <= max_context, else KV_ERR_INVALID.
 *   context_lens   P <= L_b <= max_context for every sequence. L_b = P gives
 *                  the prefix's attention alone. On the device, a length
 *                  outside that range raises KV_DEVERR_CONTEXT and zeros the
 *                  sequence's outputs. With an append, L_b = P also raises
 *                  KV_DEVERR_CONTEXT: the new token would fall in the shared
 *                  blocks, so it is not written.
 *   workspace      device, 256-byte aligned, at least
 *                  paged_attn_cascade_workspace_bytes for the same num_seqs,
 *                  num_q_heads and num_ctas.
 * Other arguments as paged_attn_decode_append. Three kernels on the stream;
 * asynchronous; no allocation. */
kv_status paged_attn_decode_cascade(kv_pool *pool, int32_t layer, const void *q,
                                    const void *k_new, const void *v_new,
                                    int32_t q_dtype, int32_t num_seqs,
                                    int32_t num_q_heads, const int32_t *block_tables,
                                    int32_t max_blocks_per_seq,
                                    const int32_t *context_lens, int32_t max_context,
                                    int32_t prefix_blocks, float scale, void *out,
                                    int32_t num_ctas, void *workspace,
                                    uint64_t workspace_bytes, kv_stream_t stream);

/* Workspace bytes for paged_attn_decode_cascade: the decode workspace
 * (paged_attn_workspace_bytes) plus the prefix pass's partials,
 * num_seqs * num_q_heads * (head_dim + 2) * 4 bytes (each part rounded up to
 * 256 bytes). */
kv_status paged_attn_cascade_workspace_bytes(const kv_pool *pool, int32_t num_seqs,
                                             int32_t num_q_heads, int32_t num_ctas,
                                             uint64_t *bytes);

/* Phase 1 alone: the persistent attention kernel. Writes out for the units it
 * finishes and the workspace partials and bookkeeping for split units. */
kv_status paged_attn_partition(kv_pool *pool, int32_t layer, const void *q,
                               int32_t q_dtype, int32_t num_seqs,
                               int32_t num_q_heads, const int32_t *block_tables,
                               int32_t max_blocks_per_seq,
                               const int32_t *context_lens, int32_t max_context,
                               float scale, void *out, int32_t num_ctas,
                               void *workspace, uint64_t workspace_bytes,
                               kv_stream_t stream);

/* Phase 1 of paged_attn_decode_append alone: the attention kernel with the
 * new token's rows written as it streams the cache. Arguments as
 * paged_attn_decode_append; paged_attn_merge completes it. */
kv_status paged_attn_partition_append(kv_pool *pool, int32_t layer, const void *q,
                                      const void *k_new, const void *v_new,
                                      int32_t q_dtype, int32_t num_seqs,
                                      int32_t num_q_heads,
                                      const int32_t *block_tables,
                                      int32_t max_blocks_per_seq,
                                      const int32_t *context_lens,
                                      int32_t max_context, float scale, void *out,
                                      int32_t num_ctas, void *workspace,
                                      uint64_t workspace_bytes, kv_stream_t stream);

/* Phase 2 alone: merge split units into out (out_dtype) and write zeros for
 * empty or invalid sequences. Must follow phase 1 with the same arguments. */
kv_status paged_attn_merge(kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                           const int32_t *context_lens,
                           int32_t max_blocks_per_seq, int32_t max_context,
                           int32_t num_ctas, int32_t out_dtype, void *out,
                           void *workspace, uint64_t workspace_bytes,
                           kv_stream_t stream);

/* ------------------------------------------------------------------------ */

/* Chunked prefill over the paged cache. Sequence b's c_b = cu_q_lens[b+1] -
 * cu_q_lens[b] new tokens are the last c_b of its context_lens[b] positions;
 * their K/V rows must already be in the pool (kv_append at their slots),
 * behind a prefix that may have come from the prefix cache. New token i of
 * sequence b, at position context_lens[b] - c_b + i, attends to positions
 * 0 .. context_lens[b] - c_b + i: every token sees the tokens before it and
 * itself [KV Cache 原理与 PagedAttention, §一; bjdmk.com.cn/news/6246348, §4.1:
 * a cached prefix's prefill is skipped].
 *   q, out     device [total_q][num_q_heads][head_dim], the cache dtype
 *              (16-bit caches only, else KV_ERR_UNSUPPORTED), 16-byte aligned,
 *              sequences one after another (row cu_q_lens[b] + i).
 *   cu_q_lens  device int32 [num_seqs + 1], non-decreasing, cu_q_lens[0] = 0,
 *              cu_q_lens[num_seqs] = total_q; max_q_len >= every c_b (host).
 *   Other arguments as paged_attn_decode (any finite scale: zero weighs every
 *   attended position the same). Up to 128 query heads per kv head and 65535
 *   sequences per call (KV_ERR_UNSUPPORTED beyond).
 * A sequence with c_b > context_lens[b], a length beyond the table, or rows
 * outside [0, total_q) sets KV_DEVERR_CONTEXT and its rows are not written;
 * an invalid block id sets KV_DEVERR_BLOCK_ID and its positions are skipped.
 * One kernel launch; no workspace. */
kv_status paged_attn_prefill(kv_pool *pool, int32_t layer, const void *q,
                             int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                             const int32_t *cu_q_lens, int32_t total_q,
                             int32_t max_q_len, const int32_t *block_tables,
                             int32_t max_blocks_per_seq, const int32_t *context_lens,
                             int32_t max_context, float scale, void *out,
                             kv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Prefix cache (host only)                                                  */
/*                                                                           */
/* Requests whose prompts begin with the same tokens reuse the KV blocks      */
/* already computed for that prefix instead of prefilling it again: a radix   */
/* tree over token sequences, longest-prefix match (including part of a       */
/* block), least-recently-used leaves evicted first so a hot shared prefix    */
/* outlives the private tails below it [bjdmk.com.cn/news/6246348, §4.1,      */
/* §4.2; KV Cache 原理与 PagedAttention, §五]. KV depends on token and        */
/* position, so only exact prefixes match (§4.3).                             */
/*                                                                           */
/* The cache borrows the pool's refcounted allocator: it holds one reference  */
/* per cached block, and each block a lookup returns carries one more,        */
/* owned by the caller (release it with kv_free_blocks). Destroy the cache    */
/* before its pool. Calls on one cache are serialised internally.             */
/* ------------------------------------------------------------------------ */

typedef struct kv_prefix_cache kv_prefix_cache;

typedef struct {
  int64_t nodes;          /* radix-tree nodes (edges) */
  int64_t cached_blocks;  /* blocks the cache holds a reference on */
  int64_t lookups;        /* kv_prefix_match calls */
  int64_t hits;           /* lookups that matched at least one token */
  int64_t hit_tokens;     /* tokens matched over all lookups */
} kv_prefix_cache_stats;

kv_status kv_prefix_cache_create(kv_pool *pool, kv_prefix_cache **out);

/* Drops the cache's references (blocks held only by it become free). */
kv_status kv_prefix_cache_destroy(kv_prefix_cache *cache);

/* Longest cached prefix of tokens[0..n): *num_blocks ids in block_ids (host,
 * capacity max_blocks >= ceil(n / block_size), else KV_ERR_INVALID) covering
 * *matched_tokens tokens. Whole blocks come first; when the match continues
 * into part of one more cached block (at least one token), that block is the
 * last id: copy it (kv_cow_prepare + kv_block_copy) before appending at
 * position *matched_tokens. Ties between partial blocks go to the smallest
 * id. Each returned id carries a new reference for the caller. To keep the
 * last prompt token for the prefill to compute, pass n - 1. */
kv_status kv_prefix_match(kv_prefix_cache *cache, const int32_t *tokens, int32_t n,
                          int32_t max_blocks, int32_t *block_ids,
                          int32_t *num_blocks, int32_t *matched_tokens);

/* Record that the KV of tokens[0..n) lives in block_ids (host, one id per
 * whole block: n / block_size of them; a trailing partial block is not
 * cached). Prefixes already cached keep their blocks; the cache takes a
 * reference on each block it adds and reports their count in *newly_cached
 * (may be null). KV_ERR_INVALID, nothing changed, if an id is not allocated. */
kv_status kv_prefix_insert(kv_prefix_cache *cache, const int32_t *tokens, int32_t n,
                           const int32_t *block_ids, int32_t num_blocks,
                           int32_t *newly_cached);

/* Free up to `want` blocks, each time the least recently used leaf block
 * (ties: smallest id) that only the cache holds (refcount 1); blocks a
 * request still uses are skipped, and so are their ancestors. The freed ids,
 * in order, go to freed_ids (host, capacity want). */
kv_status kv_prefix_evict(kv_prefix_cache *cache, int32_t want, int32_t *freed_ids,
                          int32_t *num_freed);

/* Forget every cached prefix, e.g. after the model's weights change. */
kv_status kv_prefix_clear(kv_prefix_cache *cache);

kv_status kv_prefix_stats(kv_prefix_cache *cache, kv_prefix_cache_stats *out);

/* ------------------------------------------------------------------------ */

/* Failure-path self-test: launch one thread that waits on a shared-memory
 * barrier nothing completes, using the same bounded wait as the attention
 * kernel. After limit_us microseconds (1 .. 1e6) it gives up, ORs
 * KV_DEVERR_TIMEOUT into *device_status (device int32) and exits; the
 * context stays usable. No counterpart on the pages: it tests this library's
 * own failure detection. */
kv_status kv_selftest_wait_timeout(int32_t *device_status, uint32_t limit_us,
                                   kv_stream_t stream);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char *kv_last_error(void);

/* Library version string. */
const char *kv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
