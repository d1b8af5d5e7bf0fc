// Paged decode attention for sm_100a.
//
// out[b][h] = softmax_t(scale * q[b][h] . K_g[t]) V_g[t] over the L_b cached
// positions of sequence b, g = h / (Hq / Hkv) [bjdmk.com.cn/news/6246348, §2.1;
// KV Cache 原理与 PagedAttention, §一 GQA/MQA], where position t sits in row
// t % block_size of physical block block_table[b][t / block_size] and the
// blocks are gathered through the table [KV Cache 原理与 PagedAttention,
// §三 工作方式 4]. Quantized caches are dequantized in the kernel
// [bjdmk.com.cn/news/6246348, §5.3].
//
// Decode reads every cached K/V byte once per step and does little arithmetic
// per byte, so the kernel is bound by HBM bandwidth [KV Cache 原理与
// PagedAttention, §四]. Design:
//
// * Grid: one CTA per (partition, kv head x head chunk, sequence). A partition
//   is `part_tokens` consecutive positions (split-K); the partials are merged
//   by a second kernel.
// * Each of the CTA's 4 warps owns every 4th block of the partition and a
//   private ring of R shared-memory stages. Lane 0 of the warp fills a stage
//   with TMA: the (block, head) K tile and V tile, each a contiguous
//   block_size x head_dim slab of the pool, land swizzled so that fragment
//   loads are bank-conflict free; the per-token scales of a quantized cache
//   come along with 1-D bulk copies. Completion is signalled on an mbarrier;
//   every wait has a time limit.
// * GQA groups (Hq / Hkv >= 2) make q K^T a dense [16 tokens x 128] x
//   [128 x 8 heads] tile: warp-level tensor-core MMA (m16n8k16) with tokens as
//   M and up to 8 query heads as N. P V runs as V^T P^T with head_dim as M,
//   the probabilities turned from accumulator to operand layout by an
//   in-register 8x8 transpose. Online softmax in fp32 (base 2) per head.
// * MHA (one query head per KV head) is a matrix-vector product; it stays on
//   CUDA cores: each half-warp covers one token row (16 lanes x head_dim/16
//   values), partial dot products are reduced with a butterfly that leaves
//   one token's score per lane.
// * INT8 / E5M2 codes convert exactly to fp16 in registers; per-token K scales
//   multiply the scores, per-token V scales are folded into the softmax
//   weights through log2(scale) so the fp16 weights stay within (0, 1].
#include <algorithm>
#include <mutex>

#include "device.cuh"
#include "internal.h"

namespace pagedkv {
namespace {

using namespace dev;

constexpr int kNW = 4;  // warps per CTA
constexpr int kThreads = kNW * 32;
constexpr int kMaxPartBlocks = 512;  // partition_tokens / block_size
constexpr float kLog2e = 1.4426950408889634f;

struct AttnParams {
  const void *q;
  void *out;
  const int32_t *block_tables;
  const int32_t *context_lens;
  const float *k_scale;
  const float *v_scale;
  float *ws_o;
  float *ws_m;
  float *ws_l;
  int *status;
  float scale_log2;  // scale * log2(e)
  int num_seqs;
  int q_heads;
  int kv_heads;
  int group;       // q heads per kv head
  int chunks;      // ceil(group / 8)
  int max_blocks;  // block-table row length
  int num_blocks;  // physical blocks in the pool
  int limit;       // min(max_context, max_blocks * block_size)
  int part_tokens;
  int max_parts;
};

constexpr int align_up_c(int x, int a) { return (x + a - 1) / a * a; }

template <int KV_T>
constexpr bool is16() {
  return KV_T == KV_BF16 || KV_T == KV_FP16;
}

template <int D, int BS, int KV_T>
struct Tile {
  static constexpr int kElt = is16<KV_T>() ? 2 : 1;
  static constexpr int kRowBytes = D * kElt;
  static constexpr int kSlab = kRowBytes >= 128 ? 128 : kRowBytes;  // TMA box width, bytes
  static constexpr int kSlabs = kRowBytes / kSlab;
  static constexpr int kTileBytes = BS * kRowBytes;
  static constexpr bool kQuant = !is16<KV_T>();
  static constexpr int kLoadBytes = 2 * kTileBytes + (kQuant ? 2 * BS * 4 : 0);
  static constexpr int kStageBytes = align_up_c(kLoadBytes, 1024);

  // Shared-memory address of 16-byte chunk c of row r of a tile, as the TMA
  // swizzle placed it (128-byte swizzle on 128-byte slabs, 64-byte swizzle on
  // 64-byte rows; a 256-byte row is two slabs, each its own BS x 128 block).
  __device__ __forceinline__ static uint32_t chunk(uint32_t tile, int r, int c) {
    if constexpr (kRowBytes == 256) {
      return tile + (((c >> 3) * BS + r) << 7) + (((c & 7) ^ (r & 7)) << 4);
    } else if constexpr (kRowBytes == 128) {
      return tile + (r << 7) + ((c ^ (r & 7)) << 4);
    } else {
      return tile + (r << 6) + ((c ^ ((r >> 1) & 3)) << 4);
    }
  }
};

template <int D, int BS, int KV_T>
constexpr int smem_bytes() {
  return kNW * 3 * Tile<D, BS, KV_T>::kStageBytes + 1024;
}

template <int D, int BS, int KV_T>
__device__ __forceinline__ void issue_stage(uint8_t *stage, uint64_t *bar, const CUtensorMap *km,
                                            const CUtensorMap *vm, int id, int g,
                                            const AttnParams &p) {
  using T = Tile<D, BS, KV_T>;
  if (id < 0) {  // invalid block: complete the phase with no data
    mbar_arrive(bar);
    return;
  }
  mbar_arrive_expect_tx(bar, T::kLoadBytes);
  const int y = (id * p.kv_heads + g) * BS;
#pragma unroll
  for (int s = 0; s < T::kSlabs; ++s) {
    tma_load_2d(stage + s * BS * T::kSlab, km, bar, s * (T::kSlab / T::kElt), y);
    tma_load_2d(stage + T::kTileBytes + s * BS * T::kSlab, vm, bar, s * (T::kSlab / T::kElt), y);
  }
  if constexpr (T::kQuant) {
    bulk_load(stage + 2 * T::kTileBytes, p.k_scale + y, BS * 4, bar);
    bulk_load(stage + 2 * T::kTileBytes + BS * 4, p.v_scale + y, BS * 4, bar);
  }
}

__device__ __forceinline__ float warp_max_xor(float v, int from) {
  for (int o = from; o < 32; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// exp2(x - m) with exp2(-inf) = 0 and no NaN when both are -inf.
__device__ __forceinline__ float exp2_rel(float x, float m) {
  return x == -INFINITY ? 0.f : exp2f(x - m);
}
// Rescale factor exp2(m_old - m_new), 1 while nothing has been seen.
__device__ __forceinline__ float rescale(float m_old, float m_new) {
  return m_new == -INFINITY ? 1.f : exp2f(m_old - m_new);
}

template <int Q_T>
__device__ __forceinline__ float load_q(const void *q, int64_t idx) {
  const uint16_t bits = static_cast<const uint16_t *>(q)[idx];
  if constexpr (Q_T == KV_BF16) return __uint_as_float(static_cast<uint32_t>(bits) << 16);
  else return __half2float(__ushort_as_half(bits));
}

template <int Q_T>
__device__ __forceinline__ void store_out(void *out, int64_t idx, float v) {
  if constexpr (Q_T == KV_BF16) static_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half *>(out)[idx] = __float2half_rn(v);
}

// Load E consecutive cache values from shared memory (address in the shared
// window) and widen them to fp32. 1-byte codes are returned as their values
// (the per-token scale is applied by the caller).
template <int KV_T, int E>
__device__ __forceinline__ void load_vals(uint32_t addr, float (&v)[E]) {
  constexpr int kBytes = E * (is16<KV_T>() ? 2 : 1);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  if constexpr (kBytes == 16) {
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "r"(addr));
  } else if constexpr (kBytes == 8) {
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
  } else {
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(addr));
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if constexpr (KV_T == KV_BF16) {
      const uint32_t x = w[e >> 1];
      v[e] = __uint_as_float((e & 1) ? (x & 0xFFFF0000u) : (x << 16));
    } else if constexpr (KV_T == KV_FP16) {
      const uint32_t x = w[e >> 1];
      v[e] = __half2float(__ushort_as_half(static_cast<uint16_t>((e & 1) ? (x >> 16) : x)));
    } else if constexpr (KV_T == KV_INT8) {
      const int32_t x = static_cast<int32_t>(w[e >> 2]);
      v[e] = static_cast<float>((x << (24 - 8 * (e & 3))) >> 24);
    } else {
      const uint32_t byte = (w[e >> 2] >> (8 * (e & 3))) & 0xFFu;
      v[e] = __half2float(__ushort_as_half(static_cast<uint16_t>(byte << 8)));
    }
  }
}

// Per-warp softmax state handed to the CTA-level combine (shared memory).
struct CombineSlot {
  float m[8];
  float l[8];
};

// ============================================================================
// Partition kernel
// ============================================================================
template <int D, int BS, int KV_T, int Q_T, bool MMA>
__global__ void __launch_bounds__(kThreads)
attn_partition_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnParams p) {
  using T = Tile<D, BS, KV_T>;
  constexpr int R = 3;  // stages per warp
  constexpr bool kQuant = T::kQuant;
  constexpr bool kBF = (KV_T == KV_BF16);  // MMA operand type (bf16, else fp16)

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kNW * R];
  __shared__ int32_t bt_s[kMaxPartBlocks];
  __shared__ CombineSlot comb[kNW];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int b = blockIdx.z;
  const int g = blockIdx.y / p.chunks;
  const int chunk = blockIdx.y - g * p.chunks;
  const int part = blockIdx.x;
  const int S = p.part_tokens;

  int L = p.context_lens[b];
  if (L < 0 || L > p.limit) {
    if (threadIdx.x == 0 && part == 0 && blockIdx.y == 0) atomicOr(p.status, kErrContext);
    L = 0;
  }
  const int nparts = L > 0 ? (L + S - 1) / S : 1;
  if (part >= nparts) return;
  const int tok0 = part * S;
  const int tok1 = min(L, tok0 + S);
  const int blk0 = tok0 / BS;
  const int nblk = L > 0 ? (tok1 - tok0 + BS - 1) / BS : 0;
  const int h0 = g * p.group + chunk * 8;
  const int nh = MMA ? min(8, p.group - chunk * 8) : 1;

  if (threadIdx.x == 0) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
    for (int i = 0; i < kNW * R; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  // The partition's slice of the block table; ids outside the pool are
  // reported and the block treated as empty (no load is issued for it).
  const int32_t *bt_row = p.block_tables + static_cast<int64_t>(b) * p.max_blocks + blk0;
  for (int i = threadIdx.x; i < nblk; i += kThreads) {
    int id = bt_row[i];
    if (id < 0 || id >= p.num_blocks) {
      atomicOr(p.status, kErrBlockId);
      id = -1;
    }
    bt_s[i] = id;
  }
  __syncthreads();

  // ------------------------------------------------------------- per warp
  const int n_it = warp < nblk ? (nblk - warp + kNW - 1) / kNW : 0;
  uint8_t *wstage = smem + warp * R * T::kStageBytes;
  uint64_t *wbar = bars + warp * R;
  if (lane == 0) {
    for (int it = 0; it < R && it < n_it; ++it)
      issue_stage<D, BS, KV_T>(wstage + it * T::kStageBytes, &wbar[it], &kmap, &vmap,
                               bt_s[warp + it * kNW], g, p);
  }
  __syncwarp();

  const int gq = lane >> 2;  // MMA fragment row group
  const int cq = lane & 3;   // MMA fragment column pair

  // softmax state (MMA: heads 2cq, 2cq+1; scalar: the one head)
  float m_run[2] = {-INFINITY, -INFINITY};   // max of scores (base 2)
  float m2_run[2] = {-INFINITY, -INFINITY};  // max of scores + log2(v scale) (quant)
  float l_run[2] = {0.f, 0.f};

  // ---------------------------------------------------------------- MMA path
  constexpr int KS = D / 16;  // k-steps over head_dim
  constexpr int MT = BS / 16;  // 16-token tiles per block
  uint32_t qb[KS][2];
  float oacc[D / 16][4];
  float s_fac[2] = {p.scale_log2, p.scale_log2};
  // ------------------------------------------------------------- scalar path
  constexpr int E = D / 16;  // values per lane in a half-warp row
  float qs[E];
  float oacc_s[E];
  const int hw = lane >> 4, jl = lane & 15;

  if constexpr (MMA) {
#pragma unroll
    for (int i = 0; i < D / 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    const bool hv = gq < nh;
    const int64_t qrow = (static_cast<int64_t>(b) * p.q_heads + h0 + gq) * D;
    if constexpr (!kQuant) {
      // B operand: k = head_dim index, n = head. Lane (gq, cq) holds dims
      // 16ks + 2cq, +1 and 16ks + 8 + 2cq, +1 of head gq.
      const uint32_t *q32 = static_cast<const uint32_t *>(p.q);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qb[ks][0] = hv ? q32[(qrow + 16 * ks + 2 * cq) >> 1] : 0u;
        qb[ks][1] = hv ? q32[(qrow + 16 * ks + 8 + 2 * cq) >> 1] : 0u;
      }
    } else {
      // fp16 operands: q scaled per head by a power of two so its largest
      // magnitude is in [2^14, 2^15) (exact), the scale folded into s_fac.
      // k-slot order matches the code fragments: lane (gq, cq) holds dims
      // 16ks + 4cq .. 16ks + 4cq + 3.
      float qv[KS][4];
      float amax = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          qv[ks][e] = hv ? load_q<Q_T>(p.q, qrow + 16 * ks + 4 * cq + e) : 0.f;
          amax = fmaxf(amax, fabsf(qv[ks][e]));
        }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      int ex = 0;
      if (amax > 0.f) {
        frexpf(amax, &ex);
        ex = 15 - ex;  // amax * 2^ex in [2^14, 2^15)
      }
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qb[ks][0] = pack2<false>(ldexpf(qv[ks][0], ex), ldexpf(qv[ks][1], ex));
        qb[ks][1] = pack2<false>(ldexpf(qv[ks][2], ex), ldexpf(qv[ks][3], ex));
      }
      // the score columns of this lane are heads 2cq and 2cq+1
      const int ex0 = __shfl_sync(0xffffffffu, ex, (2 * cq) * 4);
      const int ex1 = __shfl_sync(0xffffffffu, ex, (2 * cq + 1) * 4);
      s_fac[0] = ldexpf(p.scale_log2, -ex0);
      s_fac[1] = ldexpf(p.scale_log2, -ex1);
    }
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      qs[e] = load_q<Q_T>(p.q, (static_cast<int64_t>(b) * p.q_heads + h0) * D + jl * E + e) *
              p.scale_log2;
      oacc_s[e] = 0.f;
    }
  }

  bool alive = true;
  int it = 0;
  for (; it < n_it; ++it) {
    const int s = it % R;
    uint8_t *st = wstage + s * T::kStageBytes;
    if (!mbar_wait(&wbar[s], (it / R) & 1, p.status)) {
      alive = false;
      break;
    }
    const int j = warp + it * kNW;
    const int id = bt_s[j];
    const int tok_base = (blk0 + j) * BS;
    const int valid = id >= 0 ? min(BS, tok1 - tok_base) : 0;
    const uint32_t ktile = smem_u32(st);
    const uint32_t vtile = ktile + T::kTileBytes;
    const float *ksc = reinterpret_cast<const float *>(st + 2 * T::kTileBytes);
    const float *vsc = ksc + BS;

    if constexpr (MMA) {
      // ---------------------------------------------------- scores S = K q
      float sc[MT][4];
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int row = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        if constexpr (!kQuant) {
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(T::chunk(ktile, row, 2 * ks + (lane >> 4)), a0, a1, a2, a3);
            mma16816<kBF>(acc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
          }
        } else {
#pragma unroll
          for (int kp = 0; kp < KS / 2; ++kp) {
            uint32_t r0, r1, r2, r3;  // byte matrices: rows 0-7 / 8-15 x chunks 2kp, 2kp+1
            ldsm_x4(T::chunk(ktile, row, 2 * kp + (lane >> 4)), r0, r1, r2, r3);
            if constexpr (KV_T == KV_INT8) {
              r0 ^= 0x80808080u; r1 ^= 0x80808080u; r2 ^= 0x80808080u; r3 ^= 0x80808080u;
              mma16816<false>(acc, int8_pair<0, 1>(r0), int8_pair<0, 1>(r1),
                              int8_pair<2, 3>(r0), int8_pair<2, 3>(r1), qb[2 * kp][0],
                              qb[2 * kp][1]);
              mma16816<false>(acc, int8_pair<0, 1>(r2), int8_pair<0, 1>(r3),
                              int8_pair<2, 3>(r2), int8_pair<2, 3>(r3), qb[2 * kp + 1][0],
                              qb[2 * kp + 1][1]);
            } else {
              mma16816<false>(acc, e5m2_pair<0, 1>(r0), e5m2_pair<0, 1>(r1),
                              e5m2_pair<2, 3>(r0), e5m2_pair<2, 3>(r1), qb[2 * kp][0],
                              qb[2 * kp][1]);
              mma16816<false>(acc, e5m2_pair<0, 1>(r2), e5m2_pair<0, 1>(r3),
                              e5m2_pair<2, 3>(r2), e5m2_pair<2, 3>(r3), qb[2 * kp + 1][0],
                              qb[2 * kp + 1][1]);
            }
          }
        }
        // acc: [0],[1] = token mt*16+gq, heads 2cq, 2cq+1; [2],[3] = token +8
        const int t0 = mt * 16 + gq, t1 = t0 + 8;
        float f0 = s_fac[0], f1 = s_fac[1];
        float k0 = 1.f, k1 = 1.f;
        if constexpr (kQuant) {
          k0 = ksc[t0];
          k1 = ksc[t1];
        }
        sc[mt][0] = t0 < valid ? acc[0] * f0 * k0 : -INFINITY;
        sc[mt][1] = t0 < valid ? acc[1] * f1 * k0 : -INFINITY;
        sc[mt][2] = t1 < valid ? acc[2] * f0 * k1 : -INFINITY;
        sc[mt][3] = t1 < valid ? acc[3] * f1 * k1 : -INFINITY;
      }
      // ---------------------------------------------------- online softmax
      float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        bm0 = fmaxf(bm0, fmaxf(sc[mt][0], sc[mt][2]));
        bm1 = fmaxf(bm1, fmaxf(sc[mt][1], sc[mt][3]));
      }
      bm0 = warp_max_xor(bm0, 4);
      bm1 = warp_max_xor(bm1, 4);
      const float mn0 = fmaxf(m_run[0], bm0), mn1 = fmaxf(m_run[1], bm1);
      const float al0 = rescale(m_run[0], mn0), al1 = rescale(m_run[1], mn1);
      m_run[0] = mn0;
      m_run[1] = mn1;
      float ls0 = 0.f, ls1 = 0.f;
      // weights for P V: exp2(s - m) (16-bit), exp2(s + log2 sv - m2) (quant)
      float w[MT][4];
      float be0 = 1.f, be1 = 1.f;  // O rescale factors
      if constexpr (!kQuant) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          w[mt][0] = exp2_rel(sc[mt][0], mn0);
          w[mt][1] = exp2_rel(sc[mt][1], mn1);
          w[mt][2] = exp2_rel(sc[mt][2], mn0);
          w[mt][3] = exp2_rel(sc[mt][3], mn1);
          ls0 += w[mt][0] + w[mt][2];
          ls1 += w[mt][1] + w[mt][3];
        }
        be0 = al0;
        be1 = al1;
      } else {
        float y[MT][4];
        float bn0 = -INFINITY, bn1 = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int t0 = mt * 16 + gq, t1 = t0 + 8;
          const float lv0 = t0 < valid ? log2f(vsc[t0]) : -INFINITY;
          const float lv1 = t1 < valid ? log2f(vsc[t1]) : -INFINITY;
          y[mt][0] = sc[mt][0] + lv0;
          y[mt][1] = sc[mt][1] + lv0;
          y[mt][2] = sc[mt][2] + lv1;
          y[mt][3] = sc[mt][3] + lv1;
          bn0 = fmaxf(bn0, fmaxf(y[mt][0], y[mt][2]));
          bn1 = fmaxf(bn1, fmaxf(y[mt][1], y[mt][3]));
          ls0 += exp2_rel(sc[mt][0], mn0) + exp2_rel(sc[mt][2], mn0);
          ls1 += exp2_rel(sc[mt][1], mn1) + exp2_rel(sc[mt][3], mn1);
        }
        bn0 = warp_max_xor(bn0, 4);
        bn1 = warp_max_xor(bn1, 4);
        const float n0 = fmaxf(m2_run[0], bn0), n1 = fmaxf(m2_run[1], bn1);
        be0 = rescale(m2_run[0], n0);
        be1 = rescale(m2_run[1], n1);
        m2_run[0] = n0;
        m2_run[1] = n1;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          w[mt][0] = exp2_rel(y[mt][0], n0);
          w[mt][1] = exp2_rel(y[mt][1], n1);
          w[mt][2] = exp2_rel(y[mt][2], n0);
          w[mt][3] = exp2_rel(y[mt][3], n1);
        }
      }
      l_run[0] = l_run[0] * al0 + ls0;
      l_run[1] = l_run[1] * al1 + ls1;
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        oacc[dt][0] *= be0;
        oacc[dt][1] *= be1;
        oacc[dt][2] *= be0;
        oacc[dt][3] *= be1;
      }
      // ---------------------------------------------------- O^T += V^T P^T
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        // P^T operand (k = token, n = head) from the score layout by transpose
        const uint32_t pb0 = movmatrix_t(pack2<kBF>(w[mt][0], w[mt][1]));
        const uint32_t pb1 = movmatrix_t(pack2<kBF>(w[mt][2], w[mt][3]));
        // token rows this lane's V^T fragments cover: 2cq, 2cq+1, 2cq+8, 2cq+9
        const int tb = mt * 16 + 2 * cq;
        const bool full = (mt * 16 + 16) <= valid;
        if constexpr (!kQuant) {
#pragma unroll
          for (int dt = 0; dt < D / 16; ++dt) {
            uint32_t a0, a1, a2, a3;
            // matrices: tokens 0-7 / chunk 2dt, tokens 0-7 / 2dt+1,
            //           tokens 8-15 / 2dt, tokens 8-15 / 2dt+1
            const int vr = mt * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
            ldsm_x4_t(T::chunk(vtile, vr, 2 * dt + ((lane >> 3) & 1)), a0, a1, a2, a3);
            if (!full) {  // zero rows past the valid length (stale data may be NaN)
              const uint32_t lo0 = tb < valid ? 0xFFFFu : 0u, hi0 = tb + 1 < valid ? 0xFFFF0000u : 0u;
              const uint32_t lo1 = tb + 8 < valid ? 0xFFFFu : 0u,
                             hi1 = tb + 9 < valid ? 0xFFFF0000u : 0u;
              a0 &= lo0 | hi0;
              a1 &= lo0 | hi0;
              a2 &= lo1 | hi1;
              a3 &= lo1 | hi1;
            }
            mma16816<kBF>(oacc[dt], a0, a1, a2, a3, pb0, pb1);
          }
        } else {
#pragma unroll
          for (int cp = 0; cp < D / 32; ++cp) {
            // byte matrices: tokens 0-7 / chunk 2cp, tokens 8-15 / 2cp,
            //                tokens 0-7 / 2cp+1, tokens 8-15 / 2cp+1
            uint32_t r0, r1, r2, r3;
            const int vr = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            ldsm_x4_t(T::chunk(vtile, vr, 2 * cp + (lane >> 4)), r0, r1, r2, r3);
            // after the transpose a lane holds tokens (2cq, 2cq+1) x dims (2gq, 2gq+1)
            // of each 16-dim chunk: bytes 0,2 -> dim 2gq; bytes 1,3 -> dim 2gq+1
            uint32_t a[8];
            if constexpr (KV_T == KV_INT8) {
              r0 ^= 0x80808080u; r1 ^= 0x80808080u; r2 ^= 0x80808080u; r3 ^= 0x80808080u;
              a[0] = int8_pair<0, 2>(r0); a[1] = int8_pair<1, 3>(r0);
              a[2] = int8_pair<0, 2>(r1); a[3] = int8_pair<1, 3>(r1);
              a[4] = int8_pair<0, 2>(r2); a[5] = int8_pair<1, 3>(r2);
              a[6] = int8_pair<0, 2>(r3); a[7] = int8_pair<1, 3>(r3);
            } else {
              a[0] = e5m2_pair<0, 2>(r0); a[1] = e5m2_pair<1, 3>(r0);
              a[2] = e5m2_pair<0, 2>(r1); a[3] = e5m2_pair<1, 3>(r1);
              a[4] = e5m2_pair<0, 2>(r2); a[5] = e5m2_pair<1, 3>(r2);
              a[6] = e5m2_pair<0, 2>(r3); a[7] = e5m2_pair<1, 3>(r3);
            }
            if (!full) {
              const uint32_t m0 = (tb < valid ? 0xFFFFu : 0u) | (tb + 1 < valid ? 0xFFFF0000u : 0u);
              const uint32_t m1 =
                  (tb + 8 < valid ? 0xFFFFu : 0u) | (tb + 9 < valid ? 0xFFFF0000u : 0u);
              a[0] &= m0; a[1] &= m0; a[2] &= m1; a[3] &= m1;
              a[4] &= m0; a[5] &= m0; a[6] &= m1; a[7] &= m1;
            }
            // M rows: gq -> dim 16c + 2gq, gq+8 -> dim 16c + 2gq + 1
            mma16816<false>(oacc[2 * cp], a[0], a[1], a[2], a[3], pb0, pb1);
            mma16816<false>(oacc[2 * cp + 1], a[4], a[5], a[6], a[7], pb0, pb1);
          }
        }
      }
    } else {
      // ====================================================== scalar (MHA)
      constexpr int NV = BS / 2;  // tokens per half-warp: rows 2i + hw
      float part_s[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int r = 2 * i + hw;
        float kv[E];
        const uint32_t boff = jl * E * T::kElt;  // byte offset of this lane's values in the row
        const uint32_t addr = T::chunk(ktile, r, boff >> 4) + (boff & 15);
        load_vals<KV_T, E>(addr, kv);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) a = fmaf(qs[e], kv[e], a);
        part_s[i] = a;
      }
      // butterfly reduce-scatter over the 16 lanes of the half-warp
      int nv = NV;
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) {
        if (nv > 1) {
          const bool up = (jl & o) != 0;
#pragma unroll
          for (int k = 0; k < NV / 2; ++k) {
            if (k < nv / 2) {
              const float send = up ? part_s[k] : part_s[k + nv / 2];
              const float keep = up ? part_s[k + nv / 2] : part_s[k];
              part_s[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
          }
          nv >>= 1;
        } else {
          part_s[0] += __shfl_xor_sync(0xffffffffu, part_s[0], o);
        }
      }
      // this lane now holds row 2*idx + hw, idx = jl (16 rows) or jl >> 1 (8 rows)
      const int idx = NV == 16 ? jl : (jl >> 1);
      const int r = 2 * idx + hw;
      float kscale = 1.f;
      if constexpr (kQuant) kscale = ksc[r];
      const float sv = r < valid ? part_s[0] * kscale : -INFINITY;
      const float bm = warp_max_xor(sv, 1);
      const float mn = fmaxf(m_run[0], bm);
      const float al = rescale(m_run[0], mn);
      m_run[0] = mn;
      const float pw = exp2_rel(sv, mn);
      float lsum = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) oacc_s[e] *= al;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int src = hw * 16 + (NV == 16 ? i : 2 * i);
        float pi = __shfl_sync(0xffffffffu, pw, src);
        const int rr = 2 * i + hw;
        lsum += pi;
        if (rr < valid) {
          if constexpr (kQuant) pi *= vsc[rr];
          float vv[E];
          const uint32_t boff = jl * E * T::kElt;
          const uint32_t addr = T::chunk(vtile, rr, boff >> 4) + (boff & 15);
          load_vals<KV_T, E>(addr, vv);
#pragma unroll
          for (int e = 0; e < E; ++e) oacc_s[e] = fmaf(pi, vv[e], oacc_s[e]);
        }
      }
      l_run[0] = l_run[0] * al + lsum;
    }
    __syncwarp();
    if (lane == 0 && it + R < n_it)
      issue_stage<D, BS, KV_T>(st, &wbar[s], &kmap, &vmap, bt_s[warp + (it + R) * kNW], g, p);
  }
  if (!alive) {
    // drain the stages still in flight (bounded) before shared memory is reused
    for (int k = it + 1; k < n_it && k < it + R; ++k) mbar_wait(&wbar[k % R], (k / R) & 1, p.status);
    m_run[0] = m_run[1] = m2_run[0] = m2_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  }

  // ---------------------------------------------------- warp -> CTA combine
  // Bring every warp's state to (m, l, O) with O relative to m.
  __syncthreads();  // all warps done with their stages: reuse them
  float *obuf = reinterpret_cast<float *>(smem);  // [kNW][8][D]
  if constexpr (MMA) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 4);
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 8);
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 16);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 4);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 8);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 16);
    float f0 = 1.f, f1 = 1.f;
    if constexpr (kQuant) {
      f0 = (m2_run[0] == -INFINITY || !alive) ? 0.f : exp2f(m2_run[0] - m_run[0]);
      f1 = (m2_run[1] == -INFINITY || !alive) ? 0.f : exp2f(m2_run[1] - m_run[1]);
    } else if (!alive) {
      f0 = f1 = 0.f;
    }
    float *ow = obuf + warp * 8 * D;
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
      int d0, d1;
      if constexpr (kQuant) {  // rows gq / gq+8 are dims 16c + 2gq / + 1
        d0 = dt * 16 + 2 * gq;
        d1 = d0 + 1;
      } else {
        d0 = dt * 16 + gq;
        d1 = d0 + 8;
      }
      ow[(2 * cq) * D + d0] = oacc[dt][0] * f0;
      ow[(2 * cq + 1) * D + d0] = oacc[dt][1] * f1;
      ow[(2 * cq) * D + d1] = oacc[dt][2] * f0;
      ow[(2 * cq + 1) * D + d1] = oacc[dt][3] * f1;
    }
    if (gq == 0) {
      comb[warp].m[2 * cq] = m_run[0];
      comb[warp].m[2 * cq + 1] = m_run[1];
      comb[warp].l[2 * cq] = l_run[0];
      comb[warp].l[2 * cq + 1] = l_run[1];
    }
  } else {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 16);
    float *ow = obuf + warp * 8 * D;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float v = oacc_s[e] + __shfl_xor_sync(0xffffffffu, oacc_s[e], 16);
      if (!alive) v = 0.f;
      if (hw == 0) ow[jl * E + e] = v;
    }
    if (lane == 0) {
      comb[warp].m[0] = m_run[0];
      comb[warp].l[0] = l_run[0];
    }
  }
  __syncthreads();

  for (int idx = threadIdx.x; idx < nh * D; idx += kThreads) {
    const int n = idx / D;
    const int d = idx - n * D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kNW; ++w) M = fmaxf(M, comb[w].m[n]);
    float Ls = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kNW; ++w) {
        const float f = exp2_rel(comb[w].m[n], M);
        Ls += f * comb[w].l[n];
        O += f * obuf[(w * 8 + n) * D + d];
      }
    }
    const int h = h0 + n;
    if (nparts == 1) {
      const float v = Ls > 0.f ? O / Ls : 0.f;
      store_out<Q_T>(p.out, (static_cast<int64_t>(b) * p.q_heads + h) * D + d, v);
    } else {
      const int64_t pi = (static_cast<int64_t>(b) * p.q_heads + h) * p.max_parts + part;
      p.ws_o[pi * D + d] = O;
      if (d == 0) {
        p.ws_m[pi] = M;
        p.ws_l[pi] = Ls;
      }
    }
  }
}


// ============================================================================
// Merge kernel: one warp per (sequence, query head) with > 1 partition.
// out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p, M = max_p m_p (base 2).
// ============================================================================
constexpr int kMergeWarps = 8;

template <int D, int OUT_T>
__global__ void __launch_bounds__(kMergeWarps * 32)
attn_merge_kernel(const float *__restrict__ ws_o, const float *__restrict__ ws_m,
                  const float *__restrict__ ws_l, const int32_t *__restrict__ context_lens,
                  void *out, int num_seqs, int q_heads, int part_tokens, int max_parts,
                  int limit) {
  const int w = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= num_seqs * q_heads) return;
  const int b = w / q_heads;
  const int L = context_lens[b];
  if (L < 0 || L > limit) return;  // written as zeros by the partition kernel
  const int np = (L + part_tokens - 1) / part_tokens;
  if (np <= 1) return;  // written directly by the partition kernel
  const int64_t base = static_cast<int64_t>(w) * max_parts;
  float M = -INFINITY;
  for (int pp = lane; pp < np; pp += 32) M = fmaxf(M, ws_m[base + pp]);
  M = warp_max_xor(M, 1);
  constexpr int E = D / 32;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float Ls = 0.f;
  if (M != -INFINITY) {
    for (int p0 = 0; p0 < np; p0 += 32) {
      const int pp = p0 + lane;
      const float wgt = pp < np ? exp2_rel(ws_m[base + pp], M) : 0.f;
      Ls += pp < np ? wgt * ws_l[base + pp] : 0.f;
      const int cnt = min(32, np - p0);
      for (int k = 0; k < cnt; ++k) {
        const float wk = __shfl_sync(0xffffffffu, wgt, k);
        const float *o = ws_o + (base + p0 + k) * D + lane * E;
        if constexpr (E == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(o);
          acc[0] = fmaf(wk, v.x, acc[0]);
          acc[1] = fmaf(wk, v.y, acc[1]);
          acc[2] = fmaf(wk, v.z, acc[2]);
          acc[3] = fmaf(wk, v.w, acc[3]);
        } else {
          const float2 v = *reinterpret_cast<const float2 *>(o);
          acc[0] = fmaf(wk, v.x, acc[0]);
          acc[1] = fmaf(wk, v.y, acc[1]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
  }
#pragma unroll
  for (int e = 0; e < E; ++e)
    store_out<OUT_T>(out, static_cast<int64_t>(w) * D + lane * E + e, Ls > 0.f ? acc[e] / Ls : 0.f);
}

// ============================================================================
// Host side
// ============================================================================
using PartFn = cudaError_t (*)(const CUtensorMap &, const CUtensorMap &, const AttnParams &, dim3,
                               cudaStream_t);

template <int D, int BS, int KV_T, int Q_T, bool MMA>
cudaError_t launch_part(const CUtensorMap &km, const CUtensorMap &vm, const AttnParams &p,
                        dim3 grid, cudaStream_t st) {
  constexpr int smem = smem_bytes<D, BS, KV_T>();
  auto kern = attn_partition_kernel<D, BS, KV_T, Q_T, MMA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, st>>>(km, vm, p);
  return cudaGetLastError();
}

template <int D, int BS, int KV_T, int Q_T>
PartFn pick_path(bool mma) {
  return mma ? launch_part<D, BS, KV_T, Q_T, true> : launch_part<D, BS, KV_T, Q_T, false>;
}

template <int D, int BS>
PartFn pick_dtype(int kv, int q, bool mma) {
  switch (kv) {
    case KV_BF16: return pick_path<D, BS, KV_BF16, KV_BF16>(mma);
    case KV_FP16: return pick_path<D, BS, KV_FP16, KV_FP16>(mma);
    case KV_INT8:
      return q == KV_BF16 ? pick_path<D, BS, KV_INT8, KV_BF16>(mma)
                          : pick_path<D, BS, KV_INT8, KV_FP16>(mma);
    default:
      return q == KV_BF16 ? pick_path<D, BS, KV_FP8_E5M2, KV_BF16>(mma)
                          : pick_path<D, BS, KV_FP8_E5M2, KV_FP16>(mma);
  }
}

PartFn pick_partition(int D, int BS, int kv, int q, bool mma) {
  if (D == 128) return BS == 16 ? pick_dtype<128, 16>(kv, q, mma) : pick_dtype<128, 32>(kv, q, mma);
  return BS == 16 ? pick_dtype<64, 16>(kv, q, mma) : pick_dtype<64, 32>(kv, q, mma);
}

cudaError_t launch_merge(int D, int out_t, const float *o, const float *m, const float *l,
                         const int32_t *lens, void *out, int B, int Hq, int S, int Pmax, int limit,
                         cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(B) * Hq;
  const unsigned grid = static_cast<unsigned>((warps + kMergeWarps - 1) / kMergeWarps);
  const int th = kMergeWarps * 32;
  if (D == 128) {
    if (out_t == KV_BF16)
      attn_merge_kernel<128, KV_BF16><<<grid, th, 0, st>>>(o, m, l, lens, out, B, Hq, S, Pmax, limit);
    else
      attn_merge_kernel<128, KV_FP16><<<grid, th, 0, st>>>(o, m, l, lens, out, B, Hq, S, Pmax, limit);
  } else {
    if (out_t == KV_BF16)
      attn_merge_kernel<64, KV_BF16><<<grid, th, 0, st>>>(o, m, l, lens, out, B, Hq, S, Pmax, limit);
    else
      attn_merge_kernel<64, KV_FP16><<<grid, th, 0, st>>>(o, m, l, lens, out, B, Hq, S, Pmax, limit);
  }
  return cudaGetLastError();
}

// Workspace: o [B][Hq][Pmax][D], m and l [B][Hq][Pmax], fp32, 256-aligned parts.
struct WsLayout {
  uint64_t o_off, m_off, l_off, total;
};

WsLayout ws_layout(int B, int Hq, int Pmax, int D) {
  WsLayout w{};
  if (Pmax <= 1) return w;
  const uint64_t n = static_cast<uint64_t>(B) * Hq * Pmax;
  w.o_off = 0;
  w.m_off = round_up(n * D * sizeof(float), 256);
  w.l_off = w.m_off + round_up(n * sizeof(float), 256);
  w.total = w.l_off + round_up(n * sizeof(float), 256);
  return w;
}

int heads_per_cta_chunks(int group) { return group >= 2 ? (group + 7) / 8 : 1; }

int default_partition(const kv_pool *pool, int B, int Hq, int max_ctx) {
  const int bs = pool->d.block_size;
  const int group = Hq / pool->d.num_kv_heads;
  const int64_t units =
      static_cast<int64_t>(B) * pool->d.num_kv_heads * heads_per_cta_chunks(group);
  // Enough CTAs to fill 148 SMs, two resident each, four times over; never
  // below four blocks per partition.
  const int64_t want = 4LL * 148 * 2;
  int S = 512;
  while (S > 4 * bs && units * ((max_ctx + S - 1) / S) < want) S /= 2;
  return S;
}

// Shared argument checks of the attention entry points. Fills S and Pmax.
kv_status check_attn(const kv_pool *pool, int num_seqs, int num_q_heads, int max_context,
                     int partition_tokens, int *S, int *Pmax) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (num_seqs < 0 || num_seqs > 65535) return fail(KV_ERR_INVALID, "num_seqs must be in [0, 65535]");
  const int hkv = pool->d.num_kv_heads;
  if (num_q_heads <= 0 || num_q_heads % hkv != 0)
    return fail(KV_ERR_INVALID, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                num_q_heads, hkv);
  if (static_cast<int64_t>(hkv) * heads_per_cta_chunks(num_q_heads / hkv) > 65535)
    return fail(KV_ERR_INVALID, "too many heads");
  if (max_context < 0) return fail(KV_ERR_INVALID, "negative max_context");
  const int bs = pool->d.block_size;
  int s = partition_tokens;
  if (s == 0) s = default_partition(pool, num_seqs, num_q_heads, max_context);
  if (s < bs || s % bs != 0 || s / bs > kMaxPartBlocks)
    return fail(KV_ERR_INVALID, "partition_tokens %d must be a multiple of block_size %d, at most %d",
                partition_tokens, bs, kMaxPartBlocks * bs);
  *S = s;
  *Pmax = max_context > 0 ? (max_context + s - 1) / s : 1;
  if (*Pmax > 0x7fffffff / 2) return fail(KV_ERR_INVALID, "max_context too large");
  return KV_OK;
}

kv_status run_partition(kv_pool *pool, int32_t layer, const void *q, int32_t q_dtype,
                        int32_t num_seqs, int32_t num_q_heads, const int32_t *block_tables,
                        int32_t max_blocks_per_seq, const int32_t *context_lens,
                        int32_t max_context, float scale, void *out, int32_t partition_tokens,
                        void *workspace, uint64_t workspace_bytes, cudaStream_t st,
                        int *S_out, int *Pmax_out) {
  int S = 0, Pmax = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, partition_tokens, &S, &Pmax);
  if (s != KV_OK) return s;
  if (layer < 0 || layer >= pool->d.num_layers) return fail(KV_ERR_INVALID, "layer %d out of range", layer);
  const int cd = pool->d.cache_dtype;
  if (q_dtype != KV_BF16 && q_dtype != KV_FP16)
    return fail(KV_ERR_UNSUPPORTED, "q_dtype must be KV_BF16 or KV_FP16");
  if (!is_quant(cd) && q_dtype != cd)
    return fail(KV_ERR_UNSUPPORTED, "a 16-bit cache takes queries of its own dtype");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(KV_ERR_INVALID, "scale must be finite");
  if (max_blocks_per_seq <= 0) return fail(KV_ERR_INVALID, "max_blocks_per_seq must be > 0");
  *S_out = S;
  *Pmax_out = Pmax;
  if (num_seqs == 0) return KV_OK;
  if (!q || !out || !block_tables || !context_lens) return fail(KV_ERR_INVALID, "null pointer");
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(context_lens) & 3))
    return fail(KV_ERR_INVALID, "q and out must be 16-byte aligned, tables and lengths 4-byte");
  const int D = pool->d.head_dim;
  const WsLayout wl = ws_layout(num_seqs, num_q_heads, Pmax, D);
  if (wl.total > 0) {
    if (!workspace || workspace_bytes < wl.total)
      return fail(KV_ERR_INVALID, "workspace of %llu bytes needed, %llu given",
                  static_cast<unsigned long long>(wl.total), static_cast<unsigned long long>(workspace_bytes));
    if (reinterpret_cast<uintptr_t>(workspace) & 255)
      return fail(KV_ERR_INVALID, "workspace must be 256-byte aligned");
  }
  kv_status code;
  const LayerMaps *maps = layer_maps(pool, layer, &code);
  if (!maps) return code;
  const int group = num_q_heads / pool->d.num_kv_heads;
  const bool mma = group >= 2;
  AttnParams p{};
  p.q = q;
  p.out = out;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.k_scale = layer_ks(pool, layer);
  p.v_scale = layer_vs(pool, layer);
  char *ws = static_cast<char *>(workspace);
  p.ws_o = wl.total ? reinterpret_cast<float *>(ws + wl.o_off) : nullptr;
  p.ws_m = wl.total ? reinterpret_cast<float *>(ws + wl.m_off) : nullptr;
  p.ws_l = wl.total ? reinterpret_cast<float *>(ws + wl.l_off) : nullptr;
  p.status = status_word(pool);
  p.scale_log2 = scale * kLog2e;
  p.num_seqs = num_seqs;
  p.q_heads = num_q_heads;
  p.kv_heads = pool->d.num_kv_heads;
  p.group = group;
  p.chunks = heads_per_cta_chunks(group);
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = pool->d.num_blocks;
  const int64_t tbl_cap = static_cast<int64_t>(max_blocks_per_seq) * pool->d.block_size;
  p.limit = static_cast<int>(std::min<int64_t>(max_context, tbl_cap));
  p.part_tokens = S;
  p.max_parts = Pmax;
  PartFn fn = pick_partition(D, pool->d.block_size, cd, q_dtype, mma);
  dim3 grid(Pmax, p.kv_heads * p.chunks, num_seqs);
  return cuda_check(fn(maps->k, maps->v, p, grid, st), "paged attention launch");
}

kv_status run_merge(const kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                    const int32_t *context_lens, int32_t max_blocks_per_seq,
                    int32_t max_context, int32_t partition_tokens,
                    int32_t out_dtype, void *out, const void *workspace, uint64_t workspace_bytes,
                    cudaStream_t st) {
  int S = 0, Pmax = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, partition_tokens, &S, &Pmax);
  if (s != KV_OK) return s;
  if (out_dtype != KV_BF16 && out_dtype != KV_FP16)
    return fail(KV_ERR_UNSUPPORTED, "out_dtype must be KV_BF16 or KV_FP16");
  if (max_blocks_per_seq <= 0) return fail(KV_ERR_INVALID, "max_blocks_per_seq must be > 0");
  if (num_seqs == 0 || Pmax <= 1) return KV_OK;
  if (!out || !context_lens) return fail(KV_ERR_INVALID, "null pointer");
  const int D = pool->d.head_dim;
  const WsLayout wl = ws_layout(num_seqs, num_q_heads, Pmax, D);
  if (!workspace || workspace_bytes < wl.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(KV_ERR_INVALID, "workspace missing, too small or misaligned");
  const char *ws = static_cast<const char *>(workspace);
  // same validity limit on lengths as phase 1 (invalid lengths were zeroed there)
  const int64_t tbl_cap = static_cast<int64_t>(max_blocks_per_seq) * pool->d.block_size;
  const int limit = static_cast<int>(std::min<int64_t>(max_context, tbl_cap));
  return cuda_check(
      launch_merge(D, out_dtype, reinterpret_cast<const float *>(ws + wl.o_off),
                   reinterpret_cast<const float *>(ws + wl.m_off),
                   reinterpret_cast<const float *>(ws + wl.l_off), context_lens, out, num_seqs,
                   num_q_heads, S, Pmax, limit, st),
      "merge launch");
}

}  // namespace
}  // namespace pagedkv

using namespace pagedkv;

extern "C" {

kv_status paged_attn_workspace_bytes(const kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                                     int32_t max_context, int32_t partition_tokens,
                                     uint64_t *bytes) {
  if (!bytes) return fail(KV_ERR_INVALID, "null bytes");
  int S = 0, Pmax = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, partition_tokens, &S, &Pmax);
  if (s != KV_OK) return s;
  *bytes = ws_layout(num_seqs, num_q_heads, Pmax, pool->d.head_dim).total;
  return ok();
}

kv_status paged_attn_default_partition(const kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                                       int32_t max_context, int32_t *partition_tokens) {
  if (!partition_tokens) return fail(KV_ERR_INVALID, "null partition_tokens");
  int S = 0, Pmax = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, 0, &S, &Pmax);
  if (s != KV_OK) return s;
  *partition_tokens = S;
  return ok();
}

kv_status paged_attn_partition(kv_pool *pool, int32_t layer, const void *q, int32_t q_dtype,
                               int32_t num_seqs, int32_t num_q_heads, const int32_t *block_tables,
                               int32_t max_blocks_per_seq, const int32_t *context_lens,
                               int32_t max_context, float scale, void *out,
                               int32_t partition_tokens, void *workspace, uint64_t workspace_bytes,
                               kv_stream_t stream) {
  int S, Pmax;
  kv_status s = run_partition(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                              max_blocks_per_seq, context_lens, max_context, scale, out,
                              partition_tokens, workspace, workspace_bytes,
                              (cudaStream_t)stream, &S, &Pmax);
  return s == KV_OK ? ok() : s;
}

kv_status paged_attn_merge(const kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                           const int32_t *context_lens, int32_t max_blocks_per_seq,
                           int32_t max_context, int32_t partition_tokens, int32_t out_dtype,
                           void *out, const void *workspace, uint64_t workspace_bytes,
                           kv_stream_t stream) {
  kv_status s = run_merge(pool, num_seqs, num_q_heads, context_lens, max_blocks_per_seq,
                          max_context, partition_tokens, out_dtype, out, workspace,
                          workspace_bytes, (cudaStream_t)stream);
  return s == KV_OK ? ok() : s;
}

kv_status paged_attn_decode(kv_pool *pool, int32_t layer, const void *q, int32_t q_dtype,
                            int32_t num_seqs, int32_t num_q_heads, const int32_t *block_tables,
                            int32_t max_blocks_per_seq, const int32_t *context_lens,
                            int32_t max_context, float scale, void *out, int32_t partition_tokens,
                            void *workspace, uint64_t workspace_bytes, kv_stream_t stream) {
  int S, Pmax;
  kv_status s = run_partition(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                              max_blocks_per_seq, context_lens, max_context, scale, out,
                              partition_tokens, workspace, workspace_bytes,
                              (cudaStream_t)stream, &S, &Pmax);
  if (s != KV_OK) return s;
  if (num_seqs > 0 && Pmax > 1) {
    s = run_merge(pool, num_seqs, num_q_heads, context_lens, max_blocks_per_seq, max_context, S,
                  q_dtype, out, workspace, workspace_bytes, (cudaStream_t)stream);
    if (s != KV_OK) return s;
  }
  return ok();
}

}  // extern "C"
