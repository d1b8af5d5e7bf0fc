// Chunked prefill over the paged KV cache.
//
// Each sequence's c_b new tokens are the last c_b of its L_b positions; their
// K/V rows are already in the cache (written with kv_append), behind a prefix
// that may have come from the prefix cache, whose prefill is skipped
// [bjdmk.com.cn/news/6246348, §4.1]. New token i sits at position
// L_b - c_b + i and attends to positions 0 .. L_b - c_b + i: each token sees
// every token before it and itself [KV Cache 原理与 PagedAttention, §一].
//
// Design (sm_100a):
// * One CTA per (tile of new tokens, KV head, sequence). The tile's rows are
//   (token, query head of the KV head's group) pairs, head fastest: 128 rows
//   = 128 / G tokens x G heads, 16 rows per consumer warp.
// * One producer warp streams the KV head's cached blocks, 64 positions per
//   stage (K then V, 128-byte swizzled TMA boxes of one block-head slab), into
//   a 4-stage ring; full/empty mbarriers, every wait bounded.
// * Eight consumer warps hold their Q rows as MMA A fragments and, per 32
//   positions, compute S = Q K^T with m16n8k16 tensor-core MMAs (K read by
//   ldmatrix), the online softmax in fp32 (base 2) with the causal mask, and
//   O += P V (P from the score accumulators, as hi + lo 16-bit parts; V by
//   transposed ldmatrix). This is the dense tile of prefill: every staged K/V
//   byte serves 128 query rows.
#include <algorithm>
#include <cfloat>

#include "device.cuh"
#include "internal.h"

namespace pagedkv {
namespace {

using namespace dev;

constexpr int kPfC = 8;                 // consumer warps
constexpr int kPfThreads = (kPfC + 1) * 32;
constexpr int kPfRows = kPfC * 16;      // query rows per CTA
constexpr int kPfKeys = 64;             // positions per stage
constexpr int kPfStages = 4;

struct PrefillParams {
  const void *q;              // [T][Hq][D]
  void *out;                  // [T][Hq][D]
  const int32_t *cu_q;        // [B + 1]
  const int32_t *block_tables;
  const int32_t *context_lens;
  int *status;
  float scale_log2;
  int num_seqs, q_heads, kv_heads, group, tile_tokens, total_q;
  int max_blocks, num_blocks, limit;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait on a ring barrier; gives up (false) when another warp has
// given up or after the time limit, recording KV_DEVERR_TIMEOUT.
__device__ __forceinline__ bool ring_wait_pf(uint64_t *bar, uint32_t parity, volatile int *abort,
                                             int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicOr(status, kDevErrTimeout);
        return false;
      }
    }
  }
}

// Shared address of 16-byte chunk c of row r in a stage part of `rows` rows
// stored as 128-byte slabs (slab-major), 128-byte swizzled.
__device__ __forceinline__ uint32_t pf_chunk(uint32_t base, int r, int c, int rows) {
  return base + (c >> 3) * rows * 128 + (r << 7) + (((c & 7) ^ (r & 7)) << 4);
}

template <int D, int BS, int KV_T>
__global__ void __launch_bounds__(kPfThreads, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const PrefillParams p) {
  constexpr bool kBF = (KV_T == KV_BF16);
  constexpr int kSlabs = D / 64;                     // 128-byte slabs per row
  constexpr int kPartBytes = kPfKeys * D * 2;        // K (or V) of one stage
  constexpr int kStageBytes = 2 * kPartBytes;
  constexpr int kBlocksPerStage = kPfKeys / BS;
  constexpr int KSD = D / 16;                        // k-steps over head_dim
  constexpr unsigned kFull = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kPfStages];
  __shared__ __align__(8) uint64_t empty_bar[kPfStages];
  __shared__ uint32_t stage_mask[kPfStages];         // valid blocks of the stage
  __shared__ int s_abort;
  uint8_t *ring = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int b = blockIdx.z, g = blockIdx.y;
  const int t0 = blockIdx.x * p.tile_tokens;

  grid_dependency_wait();
  const int q0 = p.cu_q[b];
  const int cb = p.cu_q[b + 1] - q0;
  const int L = p.context_lens[b];
  if (t0 >= cb) return;  // also when cb <= 0: same for the whole CTA
  if (cb > L || L > p.limit || q0 < 0 || q0 + cb > p.total_q) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) atomicOr(p.status, kErrContext);
    return;
  }
  const int t_last = min(t0 + p.tile_tokens, cb) - 1;  // last token of the tile
  const int nkeys = L - cb + t_last + 1;               // positions the tile reads
  const int nstages = (nkeys + kPfKeys - 1) / kPfKeys;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < kPfStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kPfC);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kPfC) {
    // ============================================================ producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    const int32_t *row = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;
    bool ok = true;
    int issued = 0;
    for (int st = 0; st < nstages && ok; ++st) {
      const int s = st % kPfStages;
      int okv = 1;
      if (lane == 0 && st >= kPfStages)
        okv = ring_wait_pf(&empty_bar[s], ((st / kPfStages) - 1) & 1, &s_abort, p.status);
      okv = __shfl_sync(kFull, okv, 0);
      if (!okv) {
        ok = false;
        break;
      }
      // block ids of the stage (lanes 0 .. kBlocksPerStage-1)
      const int j0 = st * kBlocksPerStage;
      const int nblk = min(kBlocksPerStage, (nkeys - st * kPfKeys + BS - 1) / BS);
      int id = -1;
      if (lane < nblk) {
        id = row[j0 + lane];
        if (id < 0 || id >= p.num_blocks) {
          atomicOr(p.status, kErrBlockId);
          id = -1;
        }
      }
      const uint32_t valid = __ballot_sync(kFull, id >= 0);
      if (lane == 0) {
        stage_mask[s] = valid;
        mbar_arrive_expect_tx(&full_bar[s], __popc(valid) * 2 * BS * D * 2);
      }
      for (int j = 0; j < nblk; ++j) {
        const int bid = __shfl_sync(kFull, id, j);
        if (lane == 0 && bid >= 0) {
          uint8_t *kst = ring + s * kStageBytes;
          uint8_t *vst = kst + kPartBytes;
          const int y = (bid * p.kv_heads + g) * BS;
#pragma unroll
          for (int sl = 0; sl < kSlabs; ++sl) {
            const int off = (sl * kPfKeys + j * BS) * 128;
            tma_load_2d(kst + off, &kmap, &full_bar[s], sl * 64, y);
            tma_load_2d(vst + off, &vmap, &full_bar[s], sl * 64, y);
          }
        }
      }
      __syncwarp();
      ++issued;
    }
    if (!ok && lane == 0) {
      // aborted: let the loads still in flight land before the CTA can exit
      for (int st = max(0, issued - kPfStages); st < issued; ++st)
        mbar_wait(&full_bar[st % kPfStages], (st / kPfStages) & 1, nullptr, 100000000ull);
    }
    return;
  }

  // ============================================================== consumers
  const int gq = lane >> 2, cq = lane & 3;
  // rows of this lane: gq and gq + 8 of the warp's 16
  int rpos[2];
  bool rvalid[2];
  int64_t rq[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int R = warp * 16 + gq + 8 * i;
    const int tl = R / p.group, hl = R - tl * p.group;
    rvalid[i] = tl < p.tile_tokens && t0 + tl < cb;
    rpos[i] = rvalid[i] ? L - cb + t0 + tl : 0x7fffffff;
    rq[i] = (static_cast<int64_t>(q0 + t0 + tl) * p.q_heads + g * p.group + hl) * D;
  }
  // Q as A fragments: a0 (row gq, dims 16k+2cq..), a1 (row gq+8), a2, a3 (+8 dims)
  uint32_t qa[KSD][4];
  {
    const uint32_t *q32 = static_cast<const uint32_t *>(p.q);
#pragma unroll
    for (int k = 0; k < KSD; ++k) {
      qa[k][0] = rvalid[0] ? q32[(rq[0] + 16 * k + 2 * cq) >> 1] : 0u;
      qa[k][1] = rvalid[1] ? q32[(rq[1] + 16 * k + 2 * cq) >> 1] : 0u;
      qa[k][2] = rvalid[0] ? q32[(rq[0] + 16 * k + 8 + 2 * cq) >> 1] : 0u;
      qa[k][3] = rvalid[1] ? q32[(rq[1] + 16 * k + 8 + 2 * cq) >> 1] : 0u;
    }
  }
  const int wmin = min(rpos[0], rpos[1]);  // this lane's earliest row position
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float oacc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  bool alive = true;

  for (int st = 0; st < nstages; ++st) {
    const int s = st % kPfStages;
    if (alive) {
      int okv = 1;
      if (lane == 0) okv = ring_wait_pf(&full_bar[s], (st / kPfStages) & 1, &s_abort, p.status);
      okv = __shfl_sync(kFull, okv, 0);
      if (!okv) alive = false;
    }
    if (alive) {
      while (!mbar_try_wait(&full_bar[s], (st / kPfStages) & 1)) {
      }  // already complete: gives every lane the acquire
      const uint32_t kbase = smem_u32(ring + s * kStageBytes);
      const uint32_t vbase = kbase + kPartBytes;
      const uint32_t vmask_blocks = stage_mask[s];
      const int key0 = st * kPfKeys;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int hk = half * 32;  // first stage row of this half
        // -------------------------------------------- S = Q K^T (16 x 32)
        float sc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
          for (int k2 = 0; k2 < KSD / 2; ++k2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(pf_chunk(kbase, hk + nt * 8 + (lane & 7), 4 * k2 + (lane >> 3), kPfKeys),
                    b0, b1, b2, b3);
            mma16816<kBF>(sc[nt], qa[2 * k2][0], qa[2 * k2][1], qa[2 * k2][2], qa[2 * k2][3],
                          b0, b1);
            mma16816<kBF>(sc[nt], qa[2 * k2 + 1][0], qa[2 * k2 + 1][1], qa[2 * k2 + 1][2],
                          qa[2 * k2 + 1][3], b2, b3);
          }
        }
        // ------------------------------------- scale, mask, online softmax
        const int kh = key0 + hk;  // position of this half's first row
        constexpr uint32_t kAll = (1u << kBlocksPerStage) - 1u;
        const bool need_mask =
            (kh + 31 > wmin) || (kh + 32 > nkeys) || (vmask_blocks & kAll) != kAll;
        float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = e >> 1;
            const int kp = kh + nt * 8 + 2 * cq + (e & 1);
            float v = sc[nt][e] * p.scale_log2;
            if (need_mask) {
              const int blk = (kp - key0) / BS;
              const bool ok = kp <= rpos[i] && kp < nkeys && ((vmask_blocks >> blk) & 1u);
              v = ok ? v : -INFINITY;
            }
            sc[nt][e] = v;
            bm[i] = fmaxf(bm[i], v);
          }
        }
        float al[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          bm[i] = fmaxf(bm[i], __shfl_xor_sync(kFull, bm[i], 1));
          bm[i] = fmaxf(bm[i], __shfl_xor_sync(kFull, bm[i], 2));
          const float mn = fmaxf(m_run[i], bm[i]);
          al[i] = mn == m_run[i] ? 1.f : ex2f(m_run[i] - mn);
          m_run[i] = mn;
        }
        const float ms0 = m_run[0] == -INFINITY ? 0.f : m_run[0];
        const float ms1 = m_run[1] == -INFINITY ? 0.f : m_run[1];
        float ls[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          sc[nt][0] = ex2f(sc[nt][0] - ms0);
          sc[nt][1] = ex2f(sc[nt][1] - ms0);
          sc[nt][2] = ex2f(sc[nt][2] - ms1);
          sc[nt][3] = ex2f(sc[nt][3] - ms1);
          ls[0] += sc[nt][0] + sc[nt][1];
          ls[1] += sc[nt][2] + sc[nt][3];
        }
        l_run[0] = l_run[0] * al[0] + ls[0];
        l_run[1] = l_run[1] * al[1] + ls[1];
        if (__any_sync(kFull, al[0] != 1.f || al[1] != 1.f)) {
#pragma unroll
          for (int n = 0; n < D / 8; ++n) {
            oacc[n][0] *= al[0];
            oacc[n][1] *= al[0];
            oacc[n][2] *= al[1];
            oacc[n][3] *= al[1];
          }
        }
        // ---------------------------------------------------- O += P V
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {  // 16 positions each
          uint32_t ph[4], pl[4];
          split2<kBF>(sc[2 * kk][0], sc[2 * kk][1], ph[0], pl[0]);
          split2<kBF>(sc[2 * kk][2], sc[2 * kk][3], ph[1], pl[1]);
          split2<kBF>(sc[2 * kk + 1][0], sc[2 * kk + 1][1], ph[2], pl[2]);
          split2<kBF>(sc[2 * kk + 1][2], sc[2 * kk + 1][3], ph[3], pl[3]);
          // V rows this lane's B fragments cover: positions 2cq, 2cq+1 (b0)
          // and 2cq+8, 2cq+9 (b1) of the 16; zero them when not real tokens
          // (stale shared memory may hold anything)
          uint32_t vm0 = 0xffffffffu, vm1 = 0xffffffffu;
          if (need_mask) {
            const int kb = kh + kk * 16 + 2 * cq;
            auto real = [&](int kp) {
              return kp < nkeys && ((vmask_blocks >> ((kp - key0) / BS)) & 1u);
            };
            vm0 = (real(kb) ? 0xffffu : 0u) | (real(kb + 1) ? 0xffff0000u : 0u);
            vm1 = (real(kb + 8) ? 0xffffu : 0u) | (real(kb + 9) ? 0xffff0000u : 0u);
          }
#pragma unroll
          for (int n2 = 0; n2 < D / 16; ++n2) {
            uint32_t b0, b1, b2, b3;  // dims 16n2.. (b0, b1), 16n2+8.. (b2, b3)
            const int vr = hk + kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            ldsm_x4_t(pf_chunk(vbase, vr, 2 * n2 + (lane >> 4), kPfKeys), b0, b1, b2, b3);
            b0 &= vm0;
            b1 &= vm1;
            b2 &= vm0;
            b3 &= vm1;
            mma16816<kBF>(oacc[2 * n2], ph[0], ph[1], ph[2], ph[3], b0, b1);
            mma16816<kBF>(oacc[2 * n2], pl[0], pl[1], pl[2], pl[3], b0, b1);
            mma16816<kBF>(oacc[2 * n2 + 1], ph[0], ph[1], ph[2], ph[3], b2, b3);
            mma16816<kBF>(oacc[2 * n2 + 1], pl[0], pl[1], pl[2], pl[3], b2, b3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }

  // ------------------------------------------------------------- output
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_run[i] += __shfl_xor_sync(kFull, l_run[i], 1);
    l_run[i] += __shfl_xor_sync(kFull, l_run[i], 2);
  }
  const float inv0 = (alive && l_run[0] > 0.f) ? 1.f / l_run[0] : 0.f;
  const float inv1 = (alive && l_run[1] > 0.f) ? 1.f / l_run[1] : 0.f;
  uint32_t *o32 = static_cast<uint32_t *>(p.out);
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    if (rvalid[0]) o32[(rq[0] + 8 * n + 2 * cq) >> 1] = pack2<kBF>(oacc[n][0] * inv0, oacc[n][1] * inv0);
    if (rvalid[1]) o32[(rq[1] + 8 * n + 2 * cq) >> 1] = pack2<kBF>(oacc[n][2] * inv1, oacc[n][3] * inv1);
  }
}

template <int D, int BS, int KV_T>
cudaError_t launch_prefill(const CUtensorMap &km, const CUtensorMap &vm, const PrefillParams &p,
                           int tiles, cudaStream_t st) {
  constexpr int smem = kPfStages * 2 * kPfKeys * D * 2 + 1024;
  auto kern = attn_prefill_kernel<D, BS, KV_T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(tiles, p.kv_heads, p.num_seqs), dim3(kPfThreads), smem, st, km, vm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

using PrefillFn = cudaError_t (*)(const CUtensorMap &, const CUtensorMap &, const PrefillParams &,
                                  int, cudaStream_t);

template <int D>
PrefillFn pick_prefill_bs(int bs, int dt) {
  if (bs == 16) return dt == KV_BF16 ? launch_prefill<D, 16, KV_BF16> : launch_prefill<D, 16, KV_FP16>;
  return dt == KV_BF16 ? launch_prefill<D, 32, KV_BF16> : launch_prefill<D, 32, KV_FP16>;
}

}  // namespace
}  // namespace pagedkv

using namespace pagedkv;

extern "C" kv_status paged_attn_prefill(kv_pool *pool, int32_t layer, const void *q,
                                        int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                                        const int32_t *cu_q_lens, int32_t total_q,
                                        int32_t max_q_len, const int32_t *block_tables,
                                        int32_t max_blocks_per_seq,
                                        const int32_t *context_lens, int32_t max_context,
                                        float scale, void *out, kv_stream_t stream) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (layer < 0 || layer >= pool->d.num_layers) return fail(KV_ERR_INVALID, "layer %d out of range", layer);
  const int cd = pool->d.cache_dtype;
  if (is_quant(cd)) return fail(KV_ERR_UNSUPPORTED, "prefill reads 16-bit caches only");
  if (q_dtype != cd) return fail(KV_ERR_UNSUPPORTED, "q_dtype must be the cache dtype");
  const int hkv = pool->d.num_kv_heads;
  if (num_q_heads <= 0 || num_q_heads % hkv != 0)
    return fail(KV_ERR_INVALID, "num_q_heads must be a positive multiple of num_kv_heads");
  const int G = num_q_heads / hkv;
  if (G > kPfRows) return fail(KV_ERR_UNSUPPORTED, "at most %d query heads per kv head", kPfRows);
  if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || max_context < 0)
    return fail(KV_ERR_INVALID, "negative size");
  if (max_blocks_per_seq <= 0) return fail(KV_ERR_INVALID, "max_blocks_per_seq must be > 0");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(KV_ERR_INVALID, "scale must be finite");
  if (num_seqs == 0 || total_q == 0 || max_q_len == 0) return ok();
  if (!q || !out || !cu_q_lens || !block_tables || !context_lens)
    return fail(KV_ERR_INVALID, "null pointer");
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3) ||
      (reinterpret_cast<uintptr_t>(context_lens) & 3) || (reinterpret_cast<uintptr_t>(cu_q_lens) & 3))
    return fail(KV_ERR_INVALID, "q and out must be 16-byte aligned, index arrays 4-byte");
  if (num_seqs > 65535) return fail(KV_ERR_UNSUPPORTED, "at most 65535 sequences per call");
  PrefillParams p;
  p.q = q;
  p.out = out;
  p.cu_q = cu_q_lens;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.status = status_word(pool);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_seqs = num_seqs;
  p.q_heads = num_q_heads;
  p.kv_heads = hkv;
  p.group = G;
  p.tile_tokens = kPfRows / G;
  p.total_q = total_q;
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = pool->d.num_blocks;
  const int64_t tbl_cap = static_cast<int64_t>(max_blocks_per_seq) * pool->d.block_size;
  p.limit = static_cast<int>(std::min<int64_t>(max_context, tbl_cap));
  const int tiles = (max_q_len + p.tile_tokens - 1) / p.tile_tokens;
  kv_status code;
  LayerMaps maps;
  if (!layer_maps(pool, layer, pool->d.block_size, &maps, &code)) return code;
  const int D = pool->d.head_dim, bs = pool->d.block_size;
  PrefillFn fn = D == 128 ? pick_prefill_bs<128>(bs, cd) : pick_prefill_bs<64>(bs, cd);
  kv_status s = cuda_check(fn(maps.k, maps.v, p, tiles, (cudaStream_t)stream), "prefill launch");
  return s == KV_OK ? ok() : s;
}
