// Chunked prefill over the paged KV cache.
//
// Each sequence's c_b new tokens are the last c_b of its L_b positions; their
// K/V rows are already in the cache (written with kv_append), behind a prefix
// that may have come from the prefix cache, whose prefill is skipped
// [bjdmk.com.cn/news/6246348, §4.1]. New token i sits at position
// L_b - c_b + i and attends to positions 0 .. L_b - c_b + i: each token sees
// every token before it and itself [KV Cache 原理与 PagedAttention, §一].
//
// Design (sm_100a, fifth-generation tensor cores):
// * One CTA per (tile of new tokens, KV head, sequence). The tile's 128 rows
//   are (token, query head of the KV head's group) pairs, head fastest:
//   128 / G tokens x G heads. Row r lives in TMEM lane r.
// * Two producer warps (K boxes, V boxes) stream the KV head's cached
//   blocks, 64 positions per stage, into a ring of 6 (head_dim 128) or 8 (64)
//   stages; block ids are read a 32-block window ahead, each TMA box is issued
//   by its own lane. With head_dim 128 each block comes in one box for K and
//   one for V, through 4-D and 3-D views of the pool whose boxes cover both
//   128-byte slabs of a row: K lands as [block][8-row group][slab][8 rows][128
//   B], so that the 8-row groups of all keys of two adjacent stages sit 2048
//   bytes apart and form one 128-key operand; V as [block][slab][row][128 B].
//   (Where the driver declines those views: one box per block and slab, K
//   slab-major across the ring.) The copy engine's cost grows with the number
//   of boxes, not only with the bytes: one box per block streams the same
//   bytes about 25% faster than two.
// * K and V of a stage have their own full and empty barriers: a K slot is
//   released as soon as S of its unit is done, long before P V frees the V
//   slot, so the K loads run up to a ring ahead of the scores.
// * The MMA warp (one thread) issues tcgen05 MMAs with the A operand in
//   tensor memory and B in shared memory, per unit of 128 keys (two stages):
//   S_u = Q K_u^T (M 128, N 128, K head_dim; Q in TMEM, K K-major) into one
//   of two TMEM score buffers, and O += P_u V_u (M 128, N head_dim, 16 keys
//   per MMA; P in TMEM, V MN-major) into a TMEM accumulator that stays
//   resident for the whole key range. Order: S_0, S_1, then per unit u
//   O += P_u V_u followed by S_{u+2}, so the tensor core computes the next
//   scores while the softmax warps work on the current ones. Measured on
//   B200, an M 128 x N 128 x K 16 MMA takes the tensor core ~65 cycles, but
//   its issuing thread can take longer when it runs other instructions
//   between MMAs: the issue loop carries precomputed descriptors and
//   compile-time accumulate flags only.
// * 8 softmax warps (PAGEDKV_PF_GROUPS = 2 column groups; 4 gives 16 warps,
//   measured slower): warp w reads TMEM lanes 32 (w mod 4) .. + 31 (the lanes
//   a warp may access) and columns of group w / 4, so two threads share a
//   row, 64 scores each per unit, read from TMEM once (both 32-column loads
//   in flight together) and kept in registers for the max and the exp pass.
//   The row maximum of the raw scores is combined through shared memory once
//   per unit, under a named barrier of the warps sharing those TMEM lanes
//   only. The scale is applied with the maximum in one packed fused
//   multiply-add per score pair (exp2(s scale - m)); it is kept positive: a
//   negative scale enters as q's sign, a zero one as q = 0. Causal and tail
//   masks set raw scores to -inf; the online softmax runs in fp32 (base 2),
//   two lanes per instruction where the hardware has packed fp32
//   arithmetic. The running maximum is only raised
//   (and O, l rescaled in TMEM) when a new score exceeds it by more than 2^8;
//   otherwise the stale maximum stays in use, which keeps every P value below
//   256 and leaves the result unchanged up to rounding.
// * P_u overwrites S_u in TMEM, each thread in its own columns, as two
//   16-bit parts hi + lo (per 16 scores: 8 columns of packed hi pairs, then
//   8 of lo pairs, the layout of one K step of the MMA's A); O accumulates
//   P_hi V + P_lo V, so rounding P to 16 bits costs nothing measurable (bf16:
//   hi and lo by truncation, bit masks only; fp16: by rounding conversions).
// * Synchronisation is by mbarriers: TMA -> MMA (K full, V full), MMA ->
//   producers (K slot free by tcgen05.commit after S_u; V slot free after P_u
//   V, and the softmax warps wait on that commit before they rescale O or
//   read it at the end), MMA -> softmax (S_u ready), softmax -> MMA (P_u
//   written; the softmax warps wait for V full too, for the block masks and
//   the tail rows they zero). Every wait is bounded; after a timeout
//   every role runs to the end without waiting, the output is not written and
//   the CTA frees its TMEM.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "device.cuh"
#include "internal.h"

namespace pagedkv {
namespace {

using namespace dev;

constexpr int kPfRows = 128;            // query rows per CTA (TMEM lanes)
#ifndef PAGEDKV_PF_GROUPS
#define PAGEDKV_PF_GROUPS 2
#endif
constexpr int kPfGroups = PAGEDKV_PF_GROUPS;  // softmax threads per row (column groups): 2 or 4
constexpr int kPfSoftmax = 128 * kPfGroups;
constexpr int kPfProducerWarp = kPfSoftmax / 32;  // K boxes; the next warp: V boxes
constexpr int kPfMmaWarp = kPfProducerWarp + 2;
constexpr int kPfThreads = kPfSoftmax + 96;
constexpr int kPfKeys = 64;             // positions per stage (TMA ring granularity)
constexpr int kPfUnit = 128;            // positions per score tile (two stages)
// Ring depth: 6 stages of 32 KB for head_dim 128, 8 of 16 KB for 64.
__host__ __device__ constexpr int pf_stages(int D) { return D == 128 ? 6 : 8; }
constexpr int kPfSBufs = 2;             // S/P buffers in TMEM, 128 columns each
// TMEM columns: S/P 2 x 128, O head_dim, Q head_dim / 2 (packed pairs)
constexpr uint32_t kPfTmemCols = 512;
constexpr float kPfRescaleLog2 = 8.f;   // raise the running max only beyond 2^8

struct PrefillParams {
  const void *q;              // [T][Hq][D]
  void *out;                  // [T][Hq][D]
  const int32_t *cu_q;        // [B + 1]
  const int32_t *block_tables;
  const int32_t *context_lens;
  int *status;
  float scale_log2;           // |scale| log2(e), or 1 where scale is 0
  // q enters TMEM as (bits & q_keep) ^ q_sign: its sign flipped where scale <
  // 0, zeroed where scale is 0 (all scores 0), so that the scale used is > 0
  uint32_t q_keep, q_sign;
  int num_seqs, q_heads, kv_heads, group, tile_tokens, total_q;
  int max_blocks, num_blocks, limit;
  // Shared-prefix pass of a cascade decode step (prefix_len > 0): the
  // total_q "new tokens" are total_q sequences' decode queries, every one
  // attending all prefix_len positions of the one block-table row (no causal
  // limit); each row's unnormalised output goes to pre_o ([total_q][Hq][D]
  // fp32) and its (maximum, sum), base 2, to pre_ml, in place of out.
  int prefix_len;
  float *pre_o;
  float *pre_ml;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait on a pipeline barrier; gives up (false) when another role has
// given up or after the time limit, recording KV_DEVERR_TIMEOUT.
// The waiting thread sleeps in the barrier (woken when the phase completes)
// rather than spinning, leaving issue slots to the warps that do the work.
__device__ __forceinline__ bool ring_wait_pf(uint64_t *bar, uint32_t parity, volatile int *abort,
                                             int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (*abort) return false;
    if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    if (globaltimer() - t0 > kWaitLimitNs) {
      *abort = 1;
      atomicOr(status, kDevErrTimeout);
      return false;
    }
  }
}

// VBLK: K and V come one box per block (both 128-byte slabs): K through the
// 4-D map, landing per stage as [block][8-row group][slab][8 rows][128 B], V
// through the 3-D map as [block][slab][row][128 B]; otherwise one box per
// block and slab, K landing as [slab][slot * 64 + key][128 B] across the ring
// and V per stage as [slab][key][128 B].
// PRE: the shared-prefix pass of a cascade decode step (prefix_len, pre_o,
// pre_ml), a separate instantiation so the prefill kernels carry no trace of it.
template <int D, int BS, int KV_T, bool VBLK, bool PRE>
__global__ void __launch_bounds__(kPfThreads, 1)
attn_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap, const PrefillParams p) {
  constexpr bool kBF = (KV_T == KV_BF16);
  constexpr int kStages = pf_stages(D);
  constexpr int kSlabs = D / 64;                     // 128-byte slabs per row
  constexpr int kPartBytes = kPfKeys * D * 2;        // K (or V) of one stage
  constexpr int kKSlabBytes = kStages * kPfKeys * 128;  // one slab of the K ring
  constexpr int kBlocksPerStage = kPfKeys / BS;
  constexpr uint32_t kAllBlocks = (1u << (2 * kBlocksPerStage)) - 1u;  // of a full unit
  constexpr uint32_t kOCol = kPfSBufs * kPfUnit;     // first TMEM column of O
  constexpr uint32_t kQCol = kOCol + D;              // first TMEM column of Q
  constexpr uint32_t kTmemCols = kPfTmemCols;
  constexpr int kSCols = kPfUnit / kPfGroups;        // scores per thread per unit
  constexpr int kSChunk = 32;                        // scores per TMEM access
  constexpr int kOCols = D / kPfGroups;              // O columns per thread
  constexpr int kOChunk = kOCols < 32 ? kOCols : 32;  // O columns per TMEM access
  constexpr int kQGCols = D / 2 / kPfGroups < 16 ? 16 : D / 2 / kPfGroups;  // Q columns per group
  constexpr unsigned kFull = 0xffffffffu;
  static_assert(kQCol + D / 2 <= kTmemCols, "TMEM budget");
  static_assert(kSCols % kSChunk == 0 && kOCols % kOChunk == 0, "column split");
  static_assert(kStages % 2 == 0, "a unit's two stages are adjacent ring slots");
  static_assert(!VBLK || kSlabs == 2, "block boxes carry two slabs");
  // V of one stage: byte offset of (key, 16-byte chunk c) and the slab stride
  auto v_off = [](int key, int c) {
    if constexpr (VBLK)
      return (key / BS) * BS * 256 + (c >> 3) * BS * 128 + (key % BS) * 128 + (c & 7) * 16;
    else
      return (c >> 3) * kPfKeys * 128 + key * 128 + (c & 7) * 16;
  };
  constexpr uint32_t kVSlabStride = VBLK ? BS * 128 : kPfKeys * 128;
  constexpr uint32_t kKGroupStride = VBLK ? 2048 : 1024;   // 8-row groups of K
  constexpr uint32_t kKSlotBytes = VBLK ? kPartBytes : kPfKeys * 128;  // K slot stride
  constexpr uint32_t kKSlabOff = VBLK ? 1024 : kKSlabBytes;            // second 64 dims

  extern __shared__ uint8_t smem_raw[];
  // K and V of a stage land and are released separately: a K slot is free
  // once S of its unit is done, a V slot once P V is
  __shared__ __align__(8) uint64_t k_full[kStages];
  __shared__ __align__(8) uint64_t v_full[kStages];
  __shared__ __align__(8) uint64_t k_empty[kStages];
  __shared__ __align__(8) uint64_t v_empty[kStages];
  __shared__ __align__(8) uint64_t s_full[kPfSBufs];
  __shared__ __align__(8) uint64_t p_full[kPfSBufs];
  __shared__ __align__(8) uint64_t mma_idle;
  // valid blocks of a stage, written by the V warp before its full arrival:
  // a V slot (unlike a K slot) is not refilled before the softmax warps are
  // done with its unit
  __shared__ uint32_t stage_mask[kStages];
  __shared__ float red[2][kPfGroups][kPfRows];       // row maxima, then row sums
  __shared__ uint32_t tmem_slot;
  __shared__ int s_abort;
  // K ring: with block boxes [slot][block][8-row group][slab][8 rows][128 B]
  // (8-row groups 2048 bytes apart, slabs 1024), else [slab][slot * 64 + key][128
  // B] (8-row groups 1024 apart); either way the two stages of a unit (slots
  // 2i, 2i + 1) form one 128-row operand. V ring: [slot][...] as v_off says.
  uint8_t *ring_k = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring_v = ring_k + kStages * kPartBytes;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int b = blockIdx.z, g = blockIdx.y;
  const int t0 = blockIdx.x * p.tile_tokens;

  grid_dependency_wait();
  constexpr bool pre = PRE;  // shared-prefix pass: no causal limit
  const int q0 = pre ? 0 : p.cu_q[b];
  const int cb = pre ? p.total_q : p.cu_q[b + 1] - q0;
  const int L = pre ? p.prefix_len : p.context_lens[b];
  if (t0 >= cb) return;  // also when cb <= 0: same for the whole CTA
  if ((!pre && cb > L) || L > p.limit || q0 < 0 || q0 + cb > p.total_q) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && g == 0) atomicOr(p.status, kErrContext);
    return;
  }
  const int t_last = min(t0 + p.tile_tokens, cb) - 1;  // last token of the tile
  const int nkeys = pre ? L : L - cb + t_last + 1;     // positions the tile reads
  const int nstages = (nkeys + kPfKeys - 1) / kPfKeys;
  const int nunits = (nstages + 1) / 2;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < kPfSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kPfSoftmax);
    }
    mbar_init(&mma_idle, 1);
    fence_barrier_init();
  }
  if (warp == kPfMmaWarp) tmem_alloc(&tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_slot;

  // softmax threads: row and column group
  const int row = (warp & 3) * 32 + lane;
  const int cg = warp >> 2;
  bool rvalid = false;
  int rpos = 0x7fffffff;
  int64_t rq = 0;
  if (warp < kPfProducerWarp) {
    const int tl = row / p.group, hl = row - tl * p.group;
    rvalid = tl < p.tile_tokens && t0 + tl < cb;
    if (rvalid) rpos = pre ? L - 1 : L - cb + t0 + tl;
    rq = (static_cast<int64_t>(q0 + t0 + tl) * p.q_heads + g * p.group + hl) * D;
    // Q row -> TMEM as packed 16-bit pairs (zeros past the tile): the first
    // D / 2 / kQGCols groups write kQGCols columns (2 kQGCols dims) each
    if (cg < D / 2 / kQGCols) {
      const uint4 *src =
          reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.q) + rq) + cg * kQGCols / 4;
      uint32_t v[kQGCols];
#pragma unroll
      for (int i = 0; i < kQGCols / 4; ++i) {
        const uint4 x = rvalid ? src[i] : make_uint4(0u, 0u, 0u, 0u);
        v[4 * i] = (x.x & p.q_keep) ^ p.q_sign;
        v[4 * i + 1] = (x.y & p.q_keep) ^ p.q_sign;
        v[4 * i + 2] = (x.z & p.q_keep) ^ p.q_sign;
        v[4 * i + 3] = (x.w & p.q_keep) ^ p.q_sign;
      }
      tmem_st<kQGCols>(tm + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kQCol + cg * kQGCols, v);
      tmem_wait_st();
    }
  }
  // Q in TMEM before the first MMA: softmax and MMA warps only, so that the
  // producers start streaming K/V while Q is still being loaded
  if (warp != kPfProducerWarp && warp != kPfProducerWarp + 1) {
    tc_fence_before();
    bar_sync(2, kPfSoftmax + 32);
    tc_fence_after();
  }

  if (warp == kPfProducerWarp || warp == kPfProducerWarp + 1) {
    // ============================================================ producers
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&vmap);
    }
    // Two warps, one for the K boxes and one for the V boxes of every stage
    // (one box per block, or per block and slab where the block maps are not
    // available, each issued by its own lane), each warp with its own full
    // and empty barriers. Block ids travel one 32-block window per lane-wide
    // load, fetched a window ahead.
    const int kv = warp - kPfProducerWarp;
    uint64_t *fullb = kv ? v_full : k_full;
    uint64_t *emptyb = kv ? v_empty : k_empty;
    const int32_t *btab = p.block_tables + static_cast<int64_t>(b) * p.max_blocks;
    const int nblocks = (nkeys + BS - 1) / BS;
    auto load_ids = [&](int w) {
      const int jb = w * 32 + lane;
      int id = -1;
      if (jb < nblocks) {
        id = btab[jb];
        if (id < 0 || id >= p.num_blocks) {
          if (kv == 0) atomicOr(p.status, kErrBlockId);
          id = -1;
        }
      }
      return id;
    };
    int cur = load_ids(0), nxt = load_ids(1);
    uint32_t cur_ok = __ballot_sync(kFull, cur >= 0);
    int issued = 0;
    // this warp's TMA boxes of a full stage
    const int kBoxes = VBLK ? kBlocksPerStage : kBlocksPerStage * kSlabs;
    static_assert(kBlocksPerStage * kSlabs <= 32, "one box per lane");
    for (int st = 0; st < nstages; ++st) {
      const int s = st % kStages;
      const int jb0 = st * kBlocksPerStage;        // first block of the stage
      if (jb0 > 0 && (jb0 & 31) == 0) {            // next window
        cur = nxt;
        cur_ok = __ballot_sync(kFull, cur >= 0);
        nxt = load_ids(jb0 / 32 + 1);
      }
      int okv = 1;
      if (lane == 0 && st >= kStages)
        okv = ring_wait_pf(&emptyb[s], ((st / kStages) - 1) & 1, &s_abort, p.status);
      okv = __shfl_sync(kFull, okv, 0);
      if (!okv) break;
      const int nblk = min(kBlocksPerStage, nblocks - jb0);
      const uint32_t valid = (cur_ok >> (jb0 & 31)) & ((1u << nblk) - 1u);
      if (lane == 0) {
        if (kv == 1) stage_mask[s] = valid;
        mbar_arrive_expect_tx(&fullb[s], __popc(valid) * BS * D * 2);
      }
      // lane -> (block j, slab)
      const int per = VBLK ? 1 : kSlabs;
      const int j = lane / per, sl = lane % per;
      const int bid = __shfl_sync(kFull, cur, (jb0 & 31) + (j < kBlocksPerStage ? j : 0));
      if (lane < kBoxes && j < nblk && ((valid >> j) & 1u)) {
        const int y = (bid * p.kv_heads + g) * BS;
        if constexpr (VBLK) {
          if (kv == 0)
            tma_load_4d(ring_k + s * kPartBytes + j * BS * 256, &kmap, &fullb[s], 0, 0, 0, y / 8);
          else
            tma_load_3d(ring_v + s * kPartBytes + j * BS * 256, &vmap, &fullb[s], 0, y, 0);
        } else {
          if (kv == 0)
            tma_load_2d(ring_k + sl * kKSlabBytes + (s * kPfKeys + j * BS) * 128, &kmap, &fullb[s],
                        sl * 64, y);
          else
            tma_load_2d(ring_v + s * kPartBytes + (sl * kPfKeys + j * BS) * 128, &vmap, &fullb[s],
                        sl * 64, y);
        }
      }
      __syncwarp();
      ++issued;
    }
    if (lane == 0) {
      // let the loads still in flight land before the CTA can exit
      for (int st = max(0, issued - kStages); st < issued; ++st)
        mbar_wait(&fullb[st % kStages], (st / kStages) & 1, nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == kPfMmaWarp) {
    // ============================================================ MMA issue
    if (lane == 0) {
      const uint32_t idesc_s = umma_idesc_f16<kBF>(kPfRows, kPfUnit, false);
      const uint32_t idesc_o = umma_idesc_f16<kBF>(kPfRows, D, true);
      // descriptors of slot 0; other slots and K steps add their byte offset
      // / 16 to the start-address field (no carry: shared addresses stay below
      // 256 KB)
      const uint64_t kdesc0 = umma_desc_sw128(smem_u32(ring_k), 16, kKGroupStride);
      const uint64_t vdesc0 = umma_desc_sw128(smem_u32(ring_v), kVSlabStride, 1024);
      bool ok = true;
      // Between two MMAs this thread runs only immediate adds: the issuing
      // thread, not the tensor core, limits small MMAs.
      auto issue_s = [&](int u) {
        const int a = 2 * u;
        const bool two = a + 1 < nstages;
        if (!ring_wait_pf(&k_full[a % kStages], (a / kStages) & 1, &s_abort, p.status))
          return false;
        if (two &&
            !ring_wait_pf(&k_full[(a + 1) % kStages], ((a + 1) / kStages) & 1, &s_abort, p.status))
          return false;
        tc_fence_after();
        // a unit's 128 keys: rows of slots a mod kStages and the next one
        const uint64_t kd = kdesc0 + static_cast<uint64_t>(((a % kStages) * kKSlotBytes) >> 4);
        const uint32_t sd = tm + (u & 1) * kPfUnit;
        umma_f16_tmem_a_c<false>(sd, tm + kQCol, kd, idesc_s);
#pragma unroll
        for (int ks = 1; ks < D / 16; ++ks)
          umma_f16_tmem_a_c<true>(sd, tm + kQCol + ks * 8,
                                  kd + (((ks >> 2) * kKSlabOff + (ks & 3) * 32) >> 4), idesc_s);
        umma_commit(&s_full[u & 1]);
        // the unit's K slots are free once S is done
        umma_commit(&k_empty[a % kStages]);
        if (two) umma_commit(&k_empty[(a + 1) % kStages]);
        return true;
      };
      for (int u = 0; ok && u < min(nunits, kPfSBufs); ++u) ok = issue_s(u);
      for (int u = 0; ok && u < nunits; ++u) {
        if (!ring_wait_pf(&p_full[u & 1], (u >> 1) & 1, &s_abort, p.status)) break;
        tc_fence_after();
        const uint32_t pcol = tm + (u & 1) * kPfUnit;
        const int a = 2 * u, nh = a + 1 < nstages ? 2 : 1;
        // V has landed (the softmax warps waited for it too)
        if (!ring_wait_pf(&v_full[a % kStages], (a / kStages) & 1, &s_abort, p.status)) break;
        if (nh == 2 &&
            !ring_wait_pf(&v_full[(a + 1) % kStages], ((a + 1) / kStages) & 1, &s_abort, p.status))
          break;
        tc_fence_after();
        // per stage of the unit: P_hi V over its 4 K steps, then P_lo V (the
        // first MMA of the first unit starts the accumulator)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h < nh) {
            const uint64_t vd =
                vdesc0 + static_cast<uint64_t>((((a + h) % kStages) * kPartBytes) >> 4);
            const uint32_t ph = pcol + h * 64;
            if (h == 0) umma_f16_tmem_a(tm + kOCol, ph, vd, idesc_o, u > 0);
            else umma_f16_tmem_a_c<true>(tm + kOCol, ph, vd, idesc_o);
#pragma unroll
            for (int ks = 1; ks < 2 * kPfKeys / 16; ++ks) {
              const int kk = ks & (kPfKeys / 16 - 1);
              umma_f16_tmem_a_c<true>(tm + kOCol, ph + kk * 16 + (ks >= kPfKeys / 16 ? 8 : 0),
                                      vd + (v_off(kk * 16, 0) >> 4), idesc_o);
            }
          }
        }
        // the unit's V slots are free (and O holds P_0..P_u V) once these finish
        umma_commit(&v_empty[a % kStages]);
        if (nh == 2) umma_commit(&v_empty[(a + 1) % kStages]);
        // S_{u+2} reuses S_u's columns: issued after P_u V, which reads them
        if (u + kPfSBufs < nunits) ok = issue_s(u + kPfSBufs);
      }
      // every MMA issued has finished before TMEM can be released
      umma_commit(&mma_idle);
      mbar_wait(&mma_idle, 0, p.status, 100000000ull);
    }
    __syncwarp();
  } else {
    // ============================================================ softmax
    // Every softmax thread runs every unit and every named barrier, also
    // after a timeout (the waits then return at once), so none is left
    // waiting at a barrier.
    const uint32_t trow = tm + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int c0 = cg * kSCols;                      // first score column
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    float m_used = -INFINITY, l_run = 0.f;
    for (int u = 0; u < nunits; ++u) {
      const int a = 2 * u;
      const bool two = a + 1 < nstages;
      ring_wait_pf(&s_full[u & 1], (u >> 1) & 1, &s_abort, p.status);
      // the stages' V has landed (a V slot's full phase cannot advance before
      // P_u V is done; a K slot may already hold the next round, so K
      // barriers are not waited on here): gives this thread the block masks
      // and the V bytes
      ring_wait_pf(&v_full[a % kStages], (a / kStages) & 1, &s_abort, p.status);
      if (two) ring_wait_pf(&v_full[(a + 1) % kStages], ((a + 1) / kStages) & 1, &s_abort, p.status);
      tc_fence_after();
      const int key0 = u * kPfUnit;
      const uint32_t bmask =
          stage_mask[a % kStages] | (two ? stage_mask[(a + 1) % kStages] << kBlocksPerStage : 0u);
      const bool tail = key0 + kPfUnit > nkeys || bmask != kAllBlocks;
      const bool need_mask = tail || key0 + c0 + kSCols - 1 > rpos;
      const uint32_t sbuf = trow + (u & 1) * kPfUnit + c0;
      // this thread's scores of the unit, read from TMEM once and kept in
      // registers; masked positions become -inf
      uint32_t sr[kSCols / kSChunk][kSChunk];
#pragma unroll
      for (int ch = 0; ch < kSCols / kSChunk; ++ch) tmem_ld<kSChunk>(sbuf + ch * kSChunk, sr[ch]);
      tmem_wait_ld();
      if (need_mask) {
        // columns past the row's last attended key (causal or tail limit),
        // then columns of blocks whose id was invalid
        const int lim = min(rpos, nkeys - 1) - key0 - c0;
#pragma unroll
        for (int ch = 0; ch < kSCols / kSChunk; ++ch)
#pragma unroll
          for (int c = 0; c < kSChunk; ++c)
            if (ch * kSChunk + c > lim) sr[ch][c] = __float_as_uint(-INFINITY);
        if (bmask != kAllBlocks) {
#pragma unroll
          for (int ch = 0; ch < kSCols / kSChunk; ++ch)
#pragma unroll
            for (int c = 0; c < kSChunk; ++c)
              if (!((bmask >> ((c0 + ch * kSChunk + c) / BS)) & 1u))
                sr[ch][c] = __float_as_uint(-INFINITY);
        }
      }
      // the row maximum of the raw scores (the scale is not negative: a
      // negative one enters as q's sign), over this thread's columns and then
      // the row's, exchanged with the warps holding the row's other columns
      float mx = -INFINITY;
#pragma unroll
      for (int ch = 0; ch < kSCols / kSChunk; ++ch)
#pragma unroll
        for (int c = 0; c < kSChunk; c += 2)
          mx = fmax3(mx, __uint_as_float(sr[ch][c]), __uint_as_float(sr[ch][c + 1]));
      red[u & 1][cg][row] = mx;
      bar_sync(3 + (warp & 3), 32 * kPfGroups);
#pragma unroll
      for (int q = 0; q < kPfGroups; ++q) mx = fmaxf(mx, red[u & 1][q][row]);
      mx = mx == -INFINITY ? -INFINITY : mx * p.scale_log2;  // base 2
      // lazy maximum: raise it only when a score exceeds it by more than 2^8
      // (every thread of the row takes the same decision)
      float alpha = 1.f;
      if (m_used == -INFINITY) {
        m_used = mx;
      } else if (mx > m_used + kPfRescaleLog2) {
        alpha = ex2f(m_used - mx);
        m_used = mx;
        l_run *= alpha;
      }
      if (__any_sync(kFull, alpha != 1.f)) {
        // O holds P_0..P_{u-1} V: wait for the last of them (the commit that
        // freed unit u-1's first V slot), rescale this thread's columns of O
        const int pa = 2 * (u - 1);
        ring_wait_pf(&v_empty[pa % kStages], (pa / kStages) & 1, &s_abort, p.status);
        tc_fence_after();
#pragma unroll
        for (int oc = 0; oc < kOCols; oc += kOChunk) {
          uint32_t o[kOChunk];
          tmem_ld<kOChunk>(trow + kOCol + cg * kOCols + oc, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kOChunk; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st<kOChunk>(trow + kOCol + cg * kOCols + oc, o);
        }
        tmem_wait_st();
      }
      // pass 2: P = 2^(s scale - m) over the same columns (one fused
      // multiply-add per pair; the scale is positive, so masked columns give
      // 2^-inf = 0), written over S as hi + lo parts (per 16 scores: 8 hi
      // pairs, then 8 lo pairs)
      const float ms = m_used == -INFINITY ? 0.f : m_used;
      const float2 nm = make_float2(-ms, -ms);
      float2 ls = make_float2(0.f, 0.f);
#pragma unroll
      for (int ch = 0; ch < kSCols / kSChunk; ++ch) {
        uint32_t pw[kSChunk];
#pragma unroll
        for (int e = 0; e < kSChunk / 2; ++e) {
          const float2 d = fma2(make_float2(__uint_as_float(sr[ch][2 * e]),
                                            __uint_as_float(sr[ch][2 * e + 1])), sc2, nm);
          float2 pa2 = make_float2(ex2f(d.x), ex2f(d.y));
          ls = add2(ls, pa2);
          const int w = (e / 8) * 16 + (e % 8);
          if constexpr (kBF) {
            // bf16 is the upper half of fp32: truncate for hi, the exact
            // remainder truncated again for lo (hi + lo within 2^-14 relative)
            const uint32_t ua = __float_as_uint(pa2.x), ub = __float_as_uint(pa2.y);
            const float2 r = sub2(pa2, make_float2(__uint_as_float(ua & 0xFFFF0000u),
                                                   __uint_as_float(ub & 0xFFFF0000u)));
            pw[w] = prmt(ua, ub, 0x7632);
            pw[w + 8] = prmt(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
          } else {
            split2<false>(pa2.x, pa2.y, pw[w], pw[w + 8]);
          }
        }
        tmem_st<kSChunk>(sbuf + ch * kSChunk, pw);
      }
      l_run += ls.x + ls.y;
      if (tail) {
        // V rows that hold no real position of this unit (past the keys the
        // tile reads, or of a block that was not loaded) may hold anything:
        // zero them so that P = 0 there cannot meet a NaN.
        constexpr int kChunks = kPfUnit * D / 8;     // 16-byte chunks of the unit's V
#pragma unroll
        for (int i = 0; i < kChunks / kPfSoftmax; ++i) {
          const int idx = threadIdx.x + i * kPfSoftmax;
          const int kr = idx / (D / 8), c = idx % (D / 8);  // row of the unit, chunk
          const int h = kr / kPfKeys, kh = kr % kPfKeys;
          const bool real = key0 + kr < nkeys && ((bmask >> (kr / BS)) & 1u);
          if (!real && (h == 0 || two))
            *reinterpret_cast<uint4 *>(ring_v + ((a + h) % kStages) * kPartBytes + v_off(kh, c)) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();                    // zeroed V rows -> tensor core
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[u & 1]);
    }
    // ------------------------------------------------------------- output
    // row sums through the buffer the last unit's maxima did not use
    red[nunits & 1][cg][row] = l_run;
    const int la = 2 * (nunits - 1);                  // P_last V done frees this stage
    ring_wait_pf(&v_empty[la % kStages], (la / kStages) & 1, &s_abort, p.status);
    bar_sync(3 + (warp & 3), 32 * kPfGroups);
    float l_tot = 0.f;
#pragma unroll
    for (int q = 0; q < kPfGroups; ++q) l_tot += red[nunits & 1][q][row];
    if (!__any_sync(kFull, s_abort != 0)) {  // warp-uniform: TMEM loads are warp-wide
      tc_fence_after();
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      if (pre && rvalid && cg == 0) {
        p.pre_ml[rq / D * 2] = m_used;
        p.pre_ml[rq / D * 2 + 1] = l_tot;
      }
#pragma unroll
      for (int oc = 0; oc < kOCols; oc += kOChunk) {
        uint32_t o[kOChunk];
        tmem_ld<kOChunk>(trow + kOCol + cg * kOCols + oc, o);
        tmem_wait_ld();
        if (pre && rvalid) {  // the partial, against m_used: O and l as they stand
          float4 *dst = reinterpret_cast<float4 *>(p.pre_o + rq + cg * kOCols + oc);
#pragma unroll
          for (int c4 = 0; c4 < kOChunk / 4; ++c4)
            dst[c4] = make_float4(__uint_as_float(o[4 * c4]), __uint_as_float(o[4 * c4 + 1]),
                                  __uint_as_float(o[4 * c4 + 2]), __uint_as_float(o[4 * c4 + 3]));
        } else if (rvalid) {
          uint4 *dst =
              reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + rq + cg * kOCols + oc);
#pragma unroll
          for (int c4 = 0; c4 < kOChunk / 8; ++c4) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack2<kBF>(__uint_as_float(o[c4 * 8 + 2 * e]) * inv,
                                __uint_as_float(o[c4 * 8 + 2 * e + 1]) * inv);
            dst[c4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kPfMmaWarp) tmem_dealloc(tm, kTmemCols);
}

template <int D, int BS, int KV_T, bool VBLK, bool PRE>
cudaError_t launch_prefill_v(const CUtensorMap &km, const CUtensorMap &vm, const PrefillParams &p,
                             int tiles, cudaStream_t st) {
  constexpr int smem = pf_stages(D) * 2 * kPfKeys * D * 2 + 1024;
  auto kern = attn_prefill_kernel<D, BS, KV_T, VBLK, PRE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(tiles, p.kv_heads, p.num_seqs), dim3(kPfThreads), smem, st, km, vm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int BS, int KV_T, bool PRE>
cudaError_t launch_prefill(const LayerMaps &maps, const PrefillParams &p, int tiles,
                           cudaStream_t st) {
  if constexpr (D == 128) {
    if (maps.v_blk_ok && maps.k_grp_ok)
      return launch_prefill_v<D, BS, KV_T, true, PRE>(maps.k_grp, maps.v_blk, p, tiles, st);
  }
  return launch_prefill_v<D, BS, KV_T, false, PRE>(maps.k, maps.v, p, tiles, st);
}

using PrefillFn = cudaError_t (*)(const LayerMaps &, const PrefillParams &, int, cudaStream_t);

template <int D, bool PRE = false>
PrefillFn pick_prefill_bs(int bs, int dt) {
  if (bs == 16)
    return dt == KV_BF16 ? launch_prefill<D, 16, KV_BF16, PRE> : launch_prefill<D, 16, KV_FP16, PRE>;
  return dt == KV_BF16 ? launch_prefill<D, 32, KV_BF16, PRE> : launch_prefill<D, 32, KV_FP16, PRE>;
}

}  // namespace

kv_status prefix_pass(kv_pool *pool, int layer, const void *q, int num_seqs, int num_q_heads,
                      const int32_t *prefix_table, int prefix_blocks, float scale, float *pre_o,
                      float *pre_ml, cudaStream_t st) {
  const int hkv = pool->d.num_kv_heads, G = num_q_heads / hkv;
  if (G > kPfRows) return fail(KV_ERR_UNSUPPORTED, "at most %d query heads per kv head", kPfRows);
  PrefillParams p{};
  p.q = q;
  p.block_tables = prefix_table;
  p.status = status_word(pool);
  p.scale_log2 = scale == 0.f ? 1.f : std::fabs(scale) * 1.4426950408889634f;
  p.q_keep = scale == 0.f ? 0u : 0xFFFFFFFFu;
  p.q_sign = scale < 0.f ? 0x80008000u : 0u;
  p.num_seqs = 1;  // the one block-table row of the prefix
  p.q_heads = num_q_heads;
  p.kv_heads = hkv;
  p.group = G;
  p.tile_tokens = kPfRows / G;
  p.total_q = num_seqs;
  p.max_blocks = prefix_blocks;
  p.num_blocks = pool->d.num_blocks;
  p.prefix_len = prefix_blocks * pool->d.block_size;
  p.limit = p.prefix_len;
  p.pre_o = pre_o;
  p.pre_ml = pre_ml;
  const int tiles = (num_seqs + p.tile_tokens - 1) / p.tile_tokens;
  kv_status code;
  LayerMaps maps;
  if (!layer_maps(pool, layer, pool->d.block_size, &maps, &code)) return code;
  const int D = pool->d.head_dim, bs = pool->d.block_size;
  PrefillFn fn = D == 128 ? pick_prefill_bs<128, true>(bs, pool->d.cache_dtype)
                          : pick_prefill_bs<64, true>(bs, pool->d.cache_dtype);
  return cuda_check(fn(maps, p, tiles, st), "cascade prefix launch");
}

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
  PrefillParams p{};
  p.q = q;
  p.out = out;
  p.cu_q = cu_q_lens;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.status = status_word(pool);
  // scores s scale = (sign(scale) q) k |scale|: the kernel's scale is positive
  p.scale_log2 = scale == 0.f ? 1.f : std::fabs(scale) * 1.4426950408889634f;
  p.q_keep = scale == 0.f ? 0u : 0xFFFFFFFFu;
  p.q_sign = scale < 0.f ? 0x80008000u : 0u;
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
  kv_status s = cuda_check(fn(maps, p, tiles, (cudaStream_t)stream), "prefill launch");
  return s == KV_OK ? ok() : s;
}
