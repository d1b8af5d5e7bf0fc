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
// * Work: a "unit" is one sequence and a group of HG consecutive KV heads
//   (with all their query heads, in chunks of up to 8). Its positions are the
//   sequence's ceil(L / block_size) blocks. All units' positions are laid end
//   to end and split evenly over a persistent grid (by default one CTA per
//   SM): every CTA streams the same number of positions, whatever the length
//   mix. A CTA's range can cut a unit only at its two ends, so each CTA emits
//   at most two partial results per head (split-K); a unit inside one CTA is
//   finished there. A merge kernel combines the split units.
// * Inside a CTA one producer warp streams, for each position, the K and V
//   rows of all HG heads of that block -- contiguous in the pool -- into a
//   ring of shared-memory stages with a few large TMA box loads (16 KB each
//   for bf16, 128-byte swizzled so fragment loads are bank-conflict free);
//   the per-token scales of a quantized cache come with 1-D bulk copies.
//   Large requests matter: the copy engine spends a roughly fixed time per
//   request, so small tiles cannot keep HBM busy. Eight consumer warps each
//   own one (KV head, query-head chunk) of the unit and keep its online
//   softmax state in registers across the unit's blocks; full/empty
//   mbarriers link producer and consumers, every wait has a time limit.
// * q K^T for the query heads of one KV head is a [16 tokens x head_dim] x
//   [head_dim x 8 heads] tile: warp-level tensor-core MMA (m16n8k16) with
//   tokens as M and up to 8 query heads as N (MHA uses one of the 8 columns:
//   the tensor pipe is otherwise idle, and one MMA replaces the CUDA-core
//   dot products and their reductions). P V runs as V^T P^T with head_dim as
//   M, the probabilities turned from accumulator to operand layout by an
//   in-register 8x8 transpose and fed as two 16-bit parts (hi + lo) so P V
//   keeps fp32-level accuracy. Online softmax in fp32 (base 2) per head.
// * INT8 and INT4 keys meet the query on the 8-bit integer tensor core
//   (m16n8k32, int32 accumulation): the key codes enter as stored (INT4 as
//   offset nibbles), the query as two exact signed 8-bit digits of its value
//   against the head's absmax, so no key code is converted. E5M2 keys and all
//   value codes convert exactly to fp16 in registers. Per-token K scales
//   multiply the scores, per-token V scales are folded into the softmax
//   weights through log2(scale) so the fp16 weights stay within (0, 1].
#include <algorithm>
#include <cfloat>

#include "device.cuh"
#include "internal.h"

namespace pagedkv {
namespace {

using namespace dev;

constexpr int kNC = 8;                    // consumer warps (one per slot of a unit)
constexpr int kWarps = kNC + 1;           // + one producer warp
constexpr int kThreads = kWarps * 32;
constexpr int kRingBytes = 200 * 1024;    // shared-memory stages per CTA
constexpr int kMaxStageBytes = 96 * 1024; // at least two stages
constexpr int kMaxStages = 8;
constexpr int kChunkHeads = 8;            // query heads of one slot (MMA N)
constexpr float kLog2e = 1.4426950408889634f;

struct AttnParams {
  const void *q;
  void *out;
  const int32_t *block_tables;
  const int32_t *context_lens;
  const float *k_scale;  // per-token K scales, or (INT8_KCHAN) the [kv_heads][D] channel scales
  const float *v_scale;
  float *part_o;   // [num_ctas][2][kNC][8][D]   unnormalised outputs of split units
  float *part_ml;  // [num_ctas][2][kNC][8][2]   their (max, sum), base 2
  int4 *meta;      // [num_seqs * units_per_seq]: first CTA, #CTAs, first side
  int *status;
  // fused append (paged_attn_decode_append): each sequence's new token, written
  // at position L - 1 before it is attended; null when not fused
  const void *k_new;  // [num_seqs][kv_heads][D], the query dtype
  const void *v_new;
  char *k_cache;      // the layer's K / V regions and scales, for the writes
  char *v_cache;
  float *k_scale_w;
  float *v_scale_w;
  float scale_log2;  // scale * log2(e)
  int num_seqs;
  int q_heads;
  int kv_heads;
  int group;           // q heads per kv head
  int chunks;          // 8-head chunks per kv head: ceil(group / 8), 1 for MHA
  int hg;              // kv heads per unit (HG)
  int cpg;             // chunks per unit (<= kNC)
  int cgroups;         // chunk groups per kv head: ceil(chunks / cpg)
  int units_per_seq;   // (kv_heads / hg) * cgroups
  int stage_bytes;     // bytes between ring stages (load size rounded to 1024)
  int stages;          // ring stages (R)
  int unit_cost;       // positions charged for starting a unit (see Walk)
  int max_blocks;      // block-table row length
  int num_blocks;      // physical blocks in the pool
  int limit;           // valid lengths: 0 < L <= min(max_context, max_blocks * bs)
  int num_ctas;
  // Cascade step (paged_attn_decode_cascade): the first len_off positions of
  // every sequence (a shared prefix) are attended by the prefix pass, this
  // call attends positions len_off .. L - 1 through tables that start at
  // them (lengths below are L - len_off), every unit leaves partials, and
  // the merge folds in each (sequence, head)'s prefix partial from pre_o
  // ([num_seqs][q_heads][D], unnormalised) and pre_ml ((max, sum), base 2).
  int len_off;
  const float *pre_o;
  const float *pre_ml;
};

// Positions of sequence b this call attends.
__device__ __forceinline__ int seq_len(const AttnParams &p, int b) {
  return p.context_lens[b] - p.len_off;
}

template <int KV_T>
constexpr bool is16() {
  return KV_T == KV_BF16 || KV_T == KV_FP16;
}

template <int D, int BS, int KV_T>
struct Tile {
  static constexpr int kElt = is16<KV_T>() ? 2 : 1;  // tensor-map element bytes
  static constexpr int kRowBytes = KV_T == KV_INT4 ? D / 2 : D * kElt;
  static constexpr int kSlab = kRowBytes >= 128 ? 128 : kRowBytes;  // TMA box width, bytes
  static constexpr int kSlabs = kRowBytes / kSlab;
  static constexpr bool kQuant = !is16<KV_T>();                 // 1-byte codes
  static constexpr bool kScaled = kQuant && KV_T != KV_FP8_E5M2_CAST;  // with fp32 scales
  // per-token K scale rows (INT8_KCHAN keys use the layer's channel scales)
  static constexpr bool kKRowScales = kScaled && KV_T != KV_INT8_KCHAN;

  // A stage holds `rows` = HG * BS rows (HG heads of one block) of K, then of
  // V, each as kSlabs slabs of rows x kSlab bytes, then (quantized caches) the
  // K scales (per-token ones only) and the V scales of those rows.
  __host__ __device__ static constexpr int load_bytes(int rows) {
    return 2 * rows * kRowBytes + (kScaled ? (kKRowScales ? 2 : 1) * rows * 4 : 0);
  }
  __host__ __device__ static constexpr int vscale_off(int rows) {
    return 2 * rows * kRowBytes + (kKRowScales ? rows * 4 : 0);
  }

  // Shared-memory address of 16-byte chunk c of row r of the K (or V) part of
  // a stage, as the TMA swizzle placed it: 128-byte swizzle on 128-byte slabs,
  // 64-byte swizzle on 64-byte rows. Rows of one head start at a multiple of
  // BS (a multiple of 8), so the swizzle phase of a head's row r is r's.
  __device__ __forceinline__ static uint32_t chunk(uint32_t tile, int r, int c, int rows) {
    if constexpr (kRowBytes == 256) {
      return tile + (c >> 3) * rows * 128 + (r << 7) + (((c & 7) ^ (r & 7)) << 4);
    } else if constexpr (kRowBytes == 128) {
      return tile + (r << 7) + ((c ^ (r & 7)) << 4);
    } else {
      return tile + (r << 6) + ((c ^ ((r >> 1) & 3)) << 4);
    }
  }
};

// Fill one stage with block `id` of the unit's HG heads (rows row0 ..
// row0 + rows - 1 of the pool's 2-D view); an invalid id completes the phase
// without data.
template <int D, int BS, int KV_T>
__device__ __forceinline__ void issue_stage(uint8_t *stage, uint64_t *bar, const CUtensorMap *km,
                                            const CUtensorMap *vm, int id, int row0, int rows,
                                            const AttnParams &p) {
  using T = Tile<D, BS, KV_T>;
  if (id < 0) {
    mbar_arrive(bar);
    return;
  }
  mbar_arrive_expect_tx(bar, T::load_bytes(rows));
  const int kv = rows * T::kRowBytes;
#pragma unroll
  for (int s = 0; s < T::kSlabs; ++s) {
    tma_load_2d(stage + s * rows * T::kSlab, km, bar, s * (T::kSlab / T::kElt), row0);
    tma_load_2d(stage + kv + s * rows * T::kSlab, vm, bar, s * (T::kSlab / T::kElt), row0);
  }
  if constexpr (T::kKRowScales) bulk_load(stage + 2 * kv, p.k_scale + row0, rows * 4, bar);
  if constexpr (T::kScaled) bulk_load(stage + T::vscale_off(rows), p.v_scale + row0, rows * 4, bar);
}

__device__ __forceinline__ float warp_max_xor(float v, int from) {
  for (int o = from; o < 32; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// exp2(x - m) with exp2(-inf) = 0 and no NaN when both are -inf.
__device__ __forceinline__ float exp2_rel(float x, float m) {
  return x == -INFINITY ? 0.f : exp2f(x - m);
}

// The SFU's base-2 exponential and logarithm (relative error about 2^-22,
// ample for softmax weights that are rounded to 16 bits for the MMA).
// ex2(-inf) = 0 and lg2(0) = -inf; subnormal inputs and results are zero.
__device__ __forceinline__ float ex2_sfu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_sfu(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int Q_T>
__device__ __forceinline__ float load_q(const void *q, int64_t idx) {
  const uint16_t bits = static_cast<const uint16_t *>(q)[idx];
  if constexpr (Q_T == KV_BF16) return __uint_as_float(static_cast<uint32_t>(bits) << 16);
  else return __half2float(__ushort_as_half(bits));
}

// Query elements idx .. idx + 3 (idx a multiple of 4) with one 8-byte load.
template <int Q_T>
__device__ __forceinline__ void load_q4(const void *q, int64_t idx, float (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(q) + idx);
  const uint32_t w[2] = {u.x, u.y};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t bits = static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1)));
    if constexpr (Q_T == KV_BF16) v[i] = __uint_as_float(static_cast<uint32_t>(bits) << 16);
    else v[i] = __half2float(__ushort_as_half(bits));
  }
}

template <int Q_T>
__device__ __forceinline__ void store_out(void *out, int64_t idx, float v) {
  if constexpr (Q_T == KV_BF16) static_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16_rn(v);
  else static_cast<__half *>(out)[idx] = __float2half_rn(v);
}

// KV blocks of sequence b; 0 for an empty or invalid length.
template <int BS>
__device__ __forceinline__ int seq_blocks(const AttnParams &p, int b) {
  const int L = seq_len(p, b);
  return (L > 0 && L <= p.limit) ? (L + BS - 1) / BS : 0;
}

// Even split of T blocks over G CTAs: CTA c gets q + 1 blocks if c < r, else q.
__device__ __forceinline__ long long cta_start(long long c, long long T, long long G) {
  const long long q = T / G, r = T % G;
  return c * q + (c < r ? c : r);
}
__device__ __forceinline__ int cta_of(long long x, long long T, long long G) {
  const long long q = T / G, r = T % G;
  if (x < r * (q + 1)) return static_cast<int>(x / (q + 1));
  return static_cast<int>(r + (x - r * (q + 1)) / q);
}

__device__ __forceinline__ long long block_sum(long long v, long long *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  long long t = 0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) t += red[i];
  __syncthreads();
  return t;
}

// Exclusive prefix sum over the CTA's threads; *total gets the CTA's sum.
__device__ __forceinline__ long long block_excl_scan(long long v, long long *red,
                                                     long long *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  long long before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) {
    before += i < warp ? red[i] : 0;
    tot += red[i];
  }
  __syncthreads();
  *total = tot;
  return before + x - v;
}

// Waits on a ring barrier; gives up when another warp has aborted or the time
// limit passes (then raises the CTA's abort flag and the device status bit).
__device__ __forceinline__ bool ring_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicOr(status, kErrTimeout);
        return false;
      }
    }
  }
}

// ============================================================================
// Consumer: per-warp state and the work on one staged block.
// ============================================================================
template <int D, int BS, int KV_T, int Q_T>
struct Consumer {
  using T = Tile<D, BS, KV_T>;
  static constexpr bool kQuant = T::kQuant;    // 1-byte codes (fp16 MMA, scaled q)
  static constexpr bool kScaled = T::kScaled;  // per-token-head scales
  static constexpr bool kBF = (KV_T == KV_BF16);  // MMA operand type (bf16, else fp16)
  static constexpr int KS = D / 16;  // k-steps over head_dim
  static constexpr int MT = BS / 16;  // 16-token tiles per block
  static constexpr bool KCH = (KV_T == KV_INT8_KCHAN);  // keys with channel scales
  static constexpr bool kInt8Codes = (KV_T == KV_INT8 || KCH);  // INT8 codes (K and V)
  // integer keys (INT8, INT4) meet the query on the 8-bit integer tensor core:
  // the query as three signed 8-bit digits, int32 accumulation
  static constexpr bool kIntK = kInt8Codes || KV_T == KV_INT4;
  static constexpr int kDig = 3;
  // Lazy running maxima (FP8-E5M2 and INT4 codes): a maximum moves only when a
  // block's exceeds it by more than 2^8, so most blocks skip the O rescale and
  // the weights stay below 2^8. Measured: E5M2 kernels 2.3 % faster, INT4
  // 1.3 %; INT8 4.4 % slower, 16-bit caches unchanged, so only these use it.
  static constexpr bool kLazy =
      KV_T == KV_FP8_E5M2 || KV_T == KV_FP8_E5M2_CAST || KV_T == KV_INT4;
  static constexpr float kLazyLog2 = 8.f;

  float m_run[2], m2_run[2], l_run[2];
  float oacc[D / 16][4];
  uint32_t qb[kIntK ? 1 : KS][2];           // 16-bit query operands (fp16 / bf16 MMA)
  uint32_t qi[kIntK ? D / 32 : 1][2][kDig];  // [k32 step][b0 / b1][digit, most significant first]
  float qcf[2];  // INT4: what the offset codes add to each score column
  float s_fac[2];

  __device__ __forceinline__ void reset() {
    m_run[0] = m_run[1] = m2_run[0] = m2_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  }

  // Query fragments of heads h0 .. h0 + nh - 1 of sequence b.
  __device__ __forceinline__ void load_query(const AttnParams &p, int b, int h0, int nh, int lane) {
    const int gq = lane >> 2, cq = lane & 3;
    s_fac[0] = s_fac[1] = p.scale_log2;
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
    } else if constexpr (kIntK) {
      // Three signed 8-bit digits per query value: x = rint(q * qs) with
      // qs = 127 * 2^16 / max|q| of the head (about 23 bits, as fp32 holds
      // q), split as x = 2^16 h + 2^8 m + l (h in [-127, 127], m and l in
      // [-128, 127]). The key codes enter as they are stored (INT8), or as
      // offset nibbles code + 8 (INT4, unsigned), so each digit's dot product
      // is exact in int32 and a score is (2^16 acc_h + 2^8 acc_m + acc_l) / qs
      // (INT4: less 8 * the same combination of the digit sums). Two digits
      // (15 bits) measured up to 2e-2 relative error on near-zero outputs of
      // per-channel keys; three keep it near 1e-5.
      // B fragment of k32 step kp: lane (gq, cq) holds 4 k-slots of head gq
      // in each half; INT8 slot (kp, half, e) is dim 32kp + 16half + 4cq + e;
      // INT4 nibbles split into even and odd dims, slot (kp, half, e) is dim
      // 64(kp / 2) + 32half + 8cq + 2e + kp % 2.
      float qv[D / 32][2][4];
      float amax = 0.f;
      // INT8 slots (kp, hf, 0..3) are 4 consecutive dims; INT4 slots (kp, hf,
      // 0..3) of kp = 2c and 2c + 1 interleave 8 consecutive dims
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          if constexpr (KV_T == KV_INT4) {
            if ((kp & 1) == 0) {
              float lo[4] = {0.f, 0.f, 0.f, 0.f}, hi4[4] = {0.f, 0.f, 0.f, 0.f};
              const int64_t base = qrow + (kp >> 1) * 64 + 32 * hf + 8 * cq;
              if (hv) {
                load_q4<Q_T>(p.q, base, lo);
                load_q4<Q_T>(p.q, base + 4, hi4);
              }
              qv[kp][hf][0] = lo[0]; qv[kp][hf][1] = lo[2]; qv[kp][hf][2] = hi4[0]; qv[kp][hf][3] = hi4[2];
              qv[kp + 1][hf][0] = lo[1]; qv[kp + 1][hf][1] = lo[3];
              qv[kp + 1][hf][2] = hi4[1]; qv[kp + 1][hf][3] = hi4[3];
            }
          } else {
            float v4[4] = {0.f, 0.f, 0.f, 0.f};
            if (hv) load_q4<Q_T>(p.q, qrow + 32 * kp + 16 * hf + 4 * cq, v4);
#pragma unroll
            for (int e = 0; e < 4; ++e) qv[kp][hf][e] = v4[e];
          }
        }
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int dim = KV_T == KV_INT4 ? (kp >> 1) * 64 + 32 * hf + 8 * cq + 2 * e + (kp & 1)
                                            : 32 * kp + 16 * hf + 4 * cq + e;
            float v = qv[kp][hf][e];
            if constexpr (KCH) {
              // keys code k / s_c: the channel scale moves to the query,
              // q . k = sum_c (q_c s_c) code_c
              v *= p.k_scale[(h0 / p.group) * D + dim];
            }
            qv[kp][hf][e] = v;
            amax = fmaxf(amax, fabsf(v));
          }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const float qs = amax > 0.f ? __fdiv_rn(8323072.f, amax) : 0.f;  // 127 * 2^16
      int dsum[kDig] = {0, 0, 0};
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t w[kDig] = {0u, 0u, 0u};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int x = __float2int_rn(qv[kp][hf][e] * qs);
            const int h = (x + 32896) >> 16;  // floors: h in [-127, 127]
            const int r = x - (h << 16);       // [-32896, 32639]
            const int m = (r + 128) >> 8;      // [-128, 127]
            const int l = r - (m << 8);        // [-128, 127]
            w[0] |= (static_cast<uint32_t>(h) & 0xFFu) << (8 * e);
            w[1] |= (static_cast<uint32_t>(m) & 0xFFu) << (8 * e);
            w[2] |= (static_cast<uint32_t>(l) & 0xFFu) << (8 * e);
            dsum[0] += h;
            dsum[1] += m;
            dsum[2] += l;
          }
#pragma unroll
          for (int d = 0; d < kDig; ++d) qi[kp][hf][d] = w[d];
        }
      // the score columns of this lane are heads 2cq and 2cq+1
      const float f = qs > 0.f ? __fdiv_rn(p.scale_log2, qs) : 0.f;
      s_fac[0] = __shfl_sync(0xffffffffu, f, (2 * cq) * 4);
      s_fac[1] = __shfl_sync(0xffffffffu, f, (2 * cq + 1) * 4);
      if constexpr (KV_T == KV_INT4) {
#pragma unroll
        for (int d = 0; d < kDig; ++d) {
          dsum[d] += __shfl_xor_sync(0xffffffffu, dsum[d], 1);
          dsum[d] += __shfl_xor_sync(0xffffffffu, dsum[d], 2);
        }
        const float corr = 8.f * fmaf(static_cast<float>(dsum[0]), 65536.f,
                                      fmaf(static_cast<float>(dsum[1]), 256.f,
                                           static_cast<float>(dsum[2])));
        qcf[0] = __shfl_sync(0xffffffffu, corr, (2 * cq) * 4);
        qcf[1] = __shfl_sync(0xffffffffu, corr, (2 * cq + 1) * 4);
      }
    } else {
      // E5M2 codes are exact fp16 values: fp16 operands, q scaled per head by
      // a power of two so its largest magnitude is in [2^14, 2^15) (exact),
      // the scale folded into s_fac. k-slot order matches the code fragments:
      // lane (gq, cq) holds dims 16ks + 4cq .. 16ks + 4cq + 3.
      float qv[KS][4];
      float amax = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        float v4[4] = {0.f, 0.f, 0.f, 0.f};
        if (hv) load_q4<Q_T>(p.q, qrow + 16 * ks + 4 * cq, v4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          qv[ks][e] = v4[e];
          amax = fmaxf(amax, fabsf(v4[e]));
        }
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      int ex = 0;
      if (amax > 0.f) {
        frexpf(amax, &ex);
        ex = 15 - ex;  // amax * 2^ex in [2^14, 2^15)
      }
      // x * 2^ex is exact while 2^ex is a normal float (ex >= -113 here, as
      // amax * 2^ex < 2^15); ex > 127 only for amax below 2^-112
      const bool pw = ex <= 127;
      const float p2 = __int_as_float((127 + (pw ? ex : 0)) << 23);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int e = 0; e < 4; ++e) qv[ks][e] = pw ? qv[ks][e] * p2 : ldexpf(qv[ks][e], ex);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qb[ks][0] = pack2<false>(qv[ks][0], qv[ks][1]);
        qb[ks][1] = pack2<false>(qv[ks][2], qv[ks][3]);
      }
      // the score columns of this lane are heads 2cq and 2cq+1
      const int ex0 = __shfl_sync(0xffffffffu, ex, (2 * cq) * 4);
      const int ex1 = __shfl_sync(0xffffffffu, ex, (2 * cq + 1) * 4);
      s_fac[0] = ldexpf(p.scale_log2, -ex0);
      s_fac[1] = ldexpf(p.scale_log2, -ex1);
    }
  }

  // One staged block of head `hi` of the stage's `rows`-row group: rows
  // [0, valid) of the head's BS rows are real tokens.
  __device__ __forceinline__ void block(const uint8_t *st, int rows, int hi, int valid, int lane) {
    if (valid <= 0) return;  // no token (an invalid block id): nothing to add
    const uint32_t ktile = smem_u32(st);
    const uint32_t vtile = ktile + rows * T::kRowBytes;
    const int r0 = hi * BS;  // the head's first row in the stage
    const float *ksc = reinterpret_cast<const float *>(st + 2 * rows * T::kRowBytes) + r0;
    const float *vsc = reinterpret_cast<const float *>(st + T::vscale_off(rows)) + r0;
    const int gq = lane >> 2, cq = lane & 3;
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
          ldsm_x4(T::chunk(ktile, r0 + row, 2 * ks + (lane >> 4), rows), a0, a1, a2, a3);
          mma16816<kBF>(acc, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
        }
      } else if constexpr (kIntK) {
        // ldmatrix.x4 of rows 0-7 / 8-15 x 16-byte chunks 2c, 2c+1 gives the
        // A fragments of one k32 step as stored bytes
        int ai[kDig][4] = {};  // one accumulator per query digit
        if constexpr (KV_T == KV_INT4) {
          // a chunk holds 32 dims as nibbles (dim 2i low, 2i + 1 high nibble of
          // byte i); offset to u = code + 8 and split into even / odd dims:
          // k32 steps 2c (even dims) and 2c + 1 (odd dims)
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t w0, w1, w2, w3;
            ldsm_x4(T::chunk(ktile, r0 + row, 2 * c + (lane >> 4), rows), w0, w1, w2, w3);
            // u = code + 8: mask the nibbles and flip their top bit in one op
            const uint32_t e0 = (w0 & 0x0F0F0F0Fu) ^ 0x08080808u, e1 = (w1 & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t e2 = (w2 & 0x0F0F0F0Fu) ^ 0x08080808u, e3 = (w3 & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t o0 = ((w0 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t o1 = ((w1 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t o2 = ((w2 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
            const uint32_t o3 = ((w3 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
#pragma unroll
            for (int d = 0; d < kDig; ++d) {
              mma16832_i8<true>(ai[d], e0, e1, e2, e3, qi[2 * c][0][d], qi[2 * c][1][d]);
              mma16832_i8<true>(ai[d], o0, o1, o2, o3, qi[2 * c + 1][0][d], qi[2 * c + 1][1][d]);
            }
          }
        } else {
#pragma unroll
          for (int kp = 0; kp < D / 32; ++kp) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(T::chunk(ktile, r0 + row, 2 * kp + (lane >> 4), rows), a0, a1, a2, a3);
#pragma unroll
            for (int d = 0; d < kDig; ++d)
              mma16832_i8<false>(ai[d], a0, a1, a2, a3, qi[kp][0][d], qi[kp][1][d]);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i] = fmaf(static_cast<float>(ai[0][i]), 65536.f,
                        fmaf(static_cast<float>(ai[1][i]), 256.f, static_cast<float>(ai[2][i])));
          if constexpr (KV_T == KV_INT4) acc[i] -= qcf[i & 1];  // columns 2cq, 2cq + 1
        }
      } else {
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
          uint32_t q0, q1, q2, q3;  // byte matrices: rows 0-7 / 8-15 x chunks 2kp, 2kp+1
          ldsm_x4(T::chunk(ktile, r0 + row, 2 * kp + (lane >> 4), rows), q0, q1, q2, q3);
          mma16816<false>(acc, e5m2_pair<0, 1>(q0), e5m2_pair<0, 1>(q1), e5m2_pair<2, 3>(q0),
                          e5m2_pair<2, 3>(q1), qb[2 * kp][0], qb[2 * kp][1]);
          mma16816<false>(acc, e5m2_pair<0, 1>(q2), e5m2_pair<0, 1>(q3), e5m2_pair<2, 3>(q2),
                          e5m2_pair<2, 3>(q3), qb[2 * kp + 1][0], qb[2 * kp + 1][1]);
        }
      }
      // acc: [0],[1] = token mt*16+gq, heads 2cq, 2cq+1; [2],[3] = token +8
      const int t0 = mt * 16 + gq, t1 = t0 + 8;
      float k0 = 1.f, k1 = 1.f;
      if constexpr (T::kKRowScales) {
        k0 = ksc[t0];
        k1 = ksc[t1];
      }
      sc[mt][0] = t0 < valid ? acc[0] * s_fac[0] * k0 : -INFINITY;
      sc[mt][1] = t0 < valid ? acc[1] * s_fac[1] * k0 : -INFINITY;
      sc[mt][2] = t1 < valid ? acc[2] * s_fac[0] * k1 : -INFINITY;
      sc[mt][3] = t1 < valid ? acc[3] * s_fac[1] * k1 : -INFINITY;
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
    // a block holds at least one valid token, so the new maxima are finite;
    // a factor is exactly 1 when its maximum did not move
    const float mn0 = kLazy ? (bm0 > m_run[0] + kLazyLog2 ? bm0 : m_run[0]) : fmaxf(m_run[0], bm0);
    const float mn1 = kLazy ? (bm1 > m_run[1] + kLazyLog2 ? bm1 : m_run[1]) : fmaxf(m_run[1], bm1);
    const float al0 = mn0 == m_run[0] ? 1.f : ex2_sfu(m_run[0] - mn0);
    const float al1 = mn1 == m_run[1] ? 1.f : ex2_sfu(m_run[1] - mn1);
    m_run[0] = mn0;
    m_run[1] = mn1;
    float ls0 = 0.f, ls1 = 0.f;
    // weights for P V: exp2(s - m) (16-bit), exp2(s + log2 sv - m2) (quant)
    float w[MT][4];
    float be0 = 1.f, be1 = 1.f;  // O rescale factors
    if constexpr (!kScaled) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        w[mt][0] = ex2_sfu(sc[mt][0] - mn0);
        w[mt][1] = ex2_sfu(sc[mt][1] - mn1);
        w[mt][2] = ex2_sfu(sc[mt][2] - mn0);
        w[mt][3] = ex2_sfu(sc[mt][3] - mn1);
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
        const float lv0 = t0 < valid ? lg2_sfu(vsc[t0]) : -INFINITY;
        const float lv1 = t1 < valid ? lg2_sfu(vsc[t1]) : -INFINITY;
        y[mt][0] = sc[mt][0] + lv0;
        y[mt][1] = sc[mt][1] + lv0;
        y[mt][2] = sc[mt][2] + lv1;
        y[mt][3] = sc[mt][3] + lv1;
        bn0 = fmaxf(bn0, fmaxf(y[mt][0], y[mt][2]));
        bn1 = fmaxf(bn1, fmaxf(y[mt][1], y[mt][3]));
        ls0 += ex2_sfu(sc[mt][0] - mn0) + ex2_sfu(sc[mt][2] - mn0);
        ls1 += ex2_sfu(sc[mt][1] - mn1) + ex2_sfu(sc[mt][3] - mn1);
      }
      bn0 = warp_max_xor(bn0, 4);
      bn1 = warp_max_xor(bn1, 4);
      // the second maxima stay -inf while every V scale seen is 0; a finite
      // stand-in keeps y - n from becoming NaN (all such y are -inf)
      const float n0 = kLazy ? (bn0 > m2_run[0] + kLazyLog2 ? bn0 : m2_run[0]) : fmaxf(m2_run[0], bn0);
      const float n1 = kLazy ? (bn1 > m2_run[1] + kLazyLog2 ? bn1 : m2_run[1]) : fmaxf(m2_run[1], bn1);
      const float f0 = fmaxf(n0, -FLT_MAX), f1 = fmaxf(n1, -FLT_MAX);
      be0 = n0 == m2_run[0] ? 1.f : ex2_sfu(m2_run[0] - f0);
      be1 = n1 == m2_run[1] ? 1.f : ex2_sfu(m2_run[1] - f1);
      m2_run[0] = n0;
      m2_run[1] = n1;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        w[mt][0] = ex2_sfu(y[mt][0] - f0);
        w[mt][1] = ex2_sfu(y[mt][1] - f1);
        w[mt][2] = ex2_sfu(y[mt][2] - f0);
        w[mt][3] = ex2_sfu(y[mt][3] - f1);
      }
    }
    l_run[0] = l_run[0] * al0 + ls0;
    l_run[1] = l_run[1] * al1 + ls1;
    // once the running maxima settle, most blocks move none of them: the whole
    // warp then skips the O rescale
    if (__any_sync(0xffffffffu, be0 != 1.f || be1 != 1.f)) {
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt) {
        oacc[dt][0] *= be0;
        oacc[dt][1] *= be1;
        oacc[dt][2] *= be0;
        oacc[dt][3] *= be1;
      }
    }
    // ---------------------------------------------------- O^T += V^T P^T
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      // P^T operand (k = token, n = head) from the score layout by transpose,
      // as a hi and a lo part so that the weights keep ~fp32 accuracy
      uint32_t h0, l0, h1, l1;
      split2<kBF>(w[mt][0], w[mt][1], h0, l0);
      split2<kBF>(w[mt][2], w[mt][3], h1, l1);
      const uint32_t pb0 = movmatrix_t(h0), pb1 = movmatrix_t(h1);
      const uint32_t pl0 = movmatrix_t(l0), pl1 = movmatrix_t(l1);
      // token rows this lane's V^T fragments cover: 2cq, 2cq+1, 2cq+8, 2cq+9
      const int tb = mt * 16 + 2 * cq;
      const bool full = (mt * 16 + 16) <= valid;
      const uint32_t m0 = (tb < valid ? 0xFFFFu : 0u) | (tb + 1 < valid ? 0xFFFF0000u : 0u);
      const uint32_t m1 = (tb + 8 < valid ? 0xFFFFu : 0u) | (tb + 9 < valid ? 0xFFFF0000u : 0u);
      if constexpr (!kQuant) {
#pragma unroll
        for (int dt = 0; dt < D / 16; ++dt) {
          uint32_t a0, a1, a2, a3;
          // matrices: tokens 0-7 / chunk 2dt, tokens 0-7 / 2dt+1,
          //           tokens 8-15 / 2dt, tokens 8-15 / 2dt+1
          const int vr = mt * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
          ldsm_x4_t(T::chunk(vtile, r0 + vr, 2 * dt + ((lane >> 3) & 1), rows), a0, a1, a2, a3);
          if (!full) {  // zero rows past the valid length (stale data may be NaN)
            a0 &= m0;
            a1 &= m0;
            a2 &= m1;
            a3 &= m1;
          }
          mma16816<kBF>(oacc[dt], a0, a1, a2, a3, pb0, pb1);
          mma16816<kBF>(oacc[dt], a0, a1, a2, a3, pl0, pl1);
        }
      } else if constexpr (KV_T == KV_INT4) {
        // after the transpose a lane holds, for tokens 2cq and 2cq+1 (low /
        // high half), the 4 nibbles of dims 32c + 4gq .. + 3; m-tile 2c + t
        // takes dims 32c + 4gq + 2t (rows gq) and + 1 (rows gq + 8)
#pragma unroll
        for (int cp = 0; cp < D / 64; ++cp) {
          uint32_t w0, w1, w2, w3;  // tokens 0-7 / 8-15 x chunks 2cp, 2cp+1
          const int vr = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          ldsm_x4_t(T::chunk(vtile, r0 + vr, 2 * cp + (lane >> 4), rows), w0, w1, w2, w3);
          uint32_t a[16];  // codes as fp16 (the offset flip is inside int4_pair)
          a[0] = int4_pair<0>(w0); a[1] = int4_pair<1>(w0); a[2] = int4_pair<0>(w1); a[3] = int4_pair<1>(w1);
          a[4] = int4_pair<2>(w0); a[5] = int4_pair<3>(w0); a[6] = int4_pair<2>(w1); a[7] = int4_pair<3>(w1);
          a[8] = int4_pair<0>(w2); a[9] = int4_pair<1>(w2); a[10] = int4_pair<0>(w3); a[11] = int4_pair<1>(w3);
          a[12] = int4_pair<2>(w2); a[13] = int4_pair<3>(w2); a[14] = int4_pair<2>(w3); a[15] = int4_pair<3>(w3);
          if (!full) {
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
              a[i] &= m0; a[i + 1] &= m0; a[i + 2] &= m1; a[i + 3] &= m1;
            }
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {  // m-tiles 4cp + t
            mma16816<false>(oacc[4 * cp + t], a[4 * t], a[4 * t + 1], a[4 * t + 2], a[4 * t + 3],
                            pb0, pb1);
            mma16816<false>(oacc[4 * cp + t], a[4 * t], a[4 * t + 1], a[4 * t + 2], a[4 * t + 3],
                            pl0, pl1);
          }
        }
      } else {
#pragma unroll
        for (int cp = 0; cp < D / 32; ++cp) {
          // byte matrices: tokens 0-7 / chunk 2cp, tokens 8-15 / 2cp,
          //                tokens 0-7 / 2cp+1, tokens 8-15 / 2cp+1
          uint32_t q0, q1, q2, q3;
          const int vr = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          ldsm_x4_t(T::chunk(vtile, r0 + vr, 2 * cp + (lane >> 4), rows), q0, q1, q2, q3);
          // after the transpose a lane holds tokens (2cq, 2cq+1) x dims (2gq, 2gq+1)
          // of each 16-dim chunk: bytes 0,2 -> dim 2gq; bytes 1,3 -> dim 2gq+1
          uint32_t a[8];
          if constexpr (kInt8Codes) {
            q0 ^= 0x80808080u; q1 ^= 0x80808080u; q2 ^= 0x80808080u; q3 ^= 0x80808080u;
            a[0] = int8_pair<0, 2>(q0); a[1] = int8_pair<1, 3>(q0);
            a[2] = int8_pair<0, 2>(q1); a[3] = int8_pair<1, 3>(q1);
            a[4] = int8_pair<0, 2>(q2); a[5] = int8_pair<1, 3>(q2);
            a[6] = int8_pair<0, 2>(q3); a[7] = int8_pair<1, 3>(q3);
          } else {
            a[0] = e5m2_pair<0, 2>(q0); a[1] = e5m2_pair<1, 3>(q0);
            a[2] = e5m2_pair<0, 2>(q1); a[3] = e5m2_pair<1, 3>(q1);
            a[4] = e5m2_pair<0, 2>(q2); a[5] = e5m2_pair<1, 3>(q2);
            a[6] = e5m2_pair<0, 2>(q3); a[7] = e5m2_pair<1, 3>(q3);
          }
          if (!full) {
            a[0] &= m0; a[1] &= m0; a[2] &= m1; a[3] &= m1;
            a[4] &= m0; a[5] &= m0; a[6] &= m1; a[7] &= m1;
          }
          // M rows: gq -> dim 16c + 2gq, gq+8 -> dim 16c + 2gq + 1
          mma16816<false>(oacc[2 * cp], a[0], a[1], a[2], a[3], pb0, pb1);
          mma16816<false>(oacc[2 * cp], a[0], a[1], a[2], a[3], pl0, pl1);
          mma16816<false>(oacc[2 * cp + 1], a[4], a[5], a[6], a[7], pb0, pb1);
          mma16816<false>(oacc[2 * cp + 1], a[4], a[5], a[6], a[7], pl0, pl1);
        }
      }
    }
  }

  // End of the unit's piece in this CTA: write the normalised output of heads
  // h0 .. h0 + nh - 1 (whole unit) or the unnormalised partial (m, l, O) to
  // record `pbase` + head of the workspace.
  template <bool CASC>
  __device__ __forceinline__ void finish(const AttnParams &p, bool whole, int b, int h0, int nh,
                                         int64_t pbase, bool alive, int lane) {
    const int gq = lane >> 2, cq = lane & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 4);
      l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 8);
      l_run[i] += __shfl_xor_sync(0xffffffffu, l_run[i], 16);
    }
    float f[2] = {alive ? 1.f : 0.f, alive ? 1.f : 0.f};
    if constexpr (kScaled) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
        f[i] = (m2_run[i] == -INFINITY || !alive) ? 0.f : exp2f(m2_run[i] - m_run[i]);
    }
    // cascade step (16-bit caches): a whole unit folds in the shared prefix's
    // partial of each of its heads here (the prefix pass finished before this
    // kernel passed its dependency wait); fp weights that partial's output
    float fp[2] = {0.f, 0.f};
    int64_t prow[2] = {0, 0};
    const bool pre = CASC && !kScaled && whole;  // (cascade kernels: O against m_run)
    if (whole) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        if (!pre) {
          f[i] = l_run[i] > 0.f ? f[i] / l_run[i] : 0.f;
          continue;
        }
        float lp = 0.f, wp = 0.f, ws = 0.f;
        if (2 * cq + i < nh) {
          prow[i] = (static_cast<int64_t>(b) * p.q_heads + h0 + 2 * cq + i) * D;
          const float2 ml = *reinterpret_cast<const float2 *>(p.pre_ml + prow[i] / D * 2);
          const float M = fmaxf(alive ? m_run[i] : -INFINITY, ml.x);
          if (M != -INFINITY) {
            ws = alive ? exp2_rel(m_run[i], M) : 0.f;
            wp = exp2_rel(ml.x, M);
            lp = ml.y * wp;
          }
        }
        const float den = l_run[i] * ws + lp;
        f[i] = den > 0.f ? ws / den : 0.f;
        fp[i] = den > 0.f ? wp / den : 0.f;
      }
    }
    // the prefix partial's values this lane adds, all loaded before the first
    // output store (the stores could alias them, so later loads would wait)
    float pv[D / 16][2][2];
    if (pre) {
#pragma unroll
      for (int dt = 0; dt < D / 16; ++dt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int d0 = dt * 16 + gq;  // 16-bit caches: rows gq / gq + 8
          const bool hv = 2 * cq + i < nh;
          pv[dt][i][0] = hv ? p.pre_o[prow[i] + d0] * fp[i] : 0.f;
          pv[dt][i][1] = hv ? p.pre_o[prow[i] + d0 + 8] * fp[i] : 0.f;
        }
    }
#pragma unroll
    for (int dt = 0; dt < D / 16; ++dt) {
      int d0, d1;
      if constexpr (KV_T == KV_INT4) {  // rows gq / gq+8: dims 32c + 4gq + 2t / + 1
        d0 = (dt >> 1) * 32 + 4 * gq + 2 * (dt & 1);
        d1 = d0 + 1;
      } else if constexpr (kQuant) {  // rows gq / gq+8 are dims 16c + 2gq / + 1
        d0 = dt * 16 + 2 * gq;
        d1 = d0 + 1;
      } else {
        d0 = dt * 16 + gq;
        d1 = d0 + 8;
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int n = 2 * cq + i;
        if (n < nh) {
          const float v0 = oacc[dt][i] * f[i], v1 = oacc[dt][i + 2] * f[i];
          if (whole) {
            const int64_t o = (static_cast<int64_t>(b) * p.q_heads + h0 + n) * D;
            if (pre) {
              store_out<Q_T>(p.out, o + d0, v0 + pv[dt][i][0]);
              store_out<Q_T>(p.out, o + d1, v1 + pv[dt][i][1]);
            } else {
              store_out<Q_T>(p.out, o + d0, v0);
              store_out<Q_T>(p.out, o + d1, v1);
            }
          } else {
            float *po = p.part_o + (pbase + n) * D;
            po[d0] = v0;
            po[d1] = v1;
          }
        }
      }
    }
    if (!whole && gq == 0) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int n = 2 * cq + i;
        if (n < nh) {
          p.part_ml[(pbase + n) * 2] = alive ? m_run[i] : -INFINITY;
          p.part_ml[(pbase + n) * 2 + 1] = l_run[i];
        }
      }
    }
  }
};

// The new token's K and V rows for one kv head, as this lane's share: lane l
// holds elements l * D/32 .. of the row (16-bit bits, or codes and scales).
template <int D, int BS, int KV_T, int Q_T>
struct NewRow {
  static constexpr int E = D / 32;
  static constexpr bool kQuant = !is16<KV_T>();
  static constexpr bool kScaled = Tile<D, BS, KV_T>::kScaled;
  uint32_t k[2], v[2];  // 16-bit: E * 2 bytes; 1-byte: E codes in k[0] / v[0]
  float ks, vs;

  __device__ __forceinline__ void load(const AttnParams &p, int b, int g, int lane) {
    const int64_t row = (static_cast<int64_t>(b) * p.kv_heads + g) * D;
    const uint16_t *kn = static_cast<const uint16_t *>(p.k_new) + row;
    const uint16_t *vn = static_cast<const uint16_t *>(p.v_new) + row;
    if constexpr (!kQuant) {
      if constexpr (E == 4) {
        const uint2 a = *reinterpret_cast<const uint2 *>(kn + lane * 4);
        const uint2 c = *reinterpret_cast<const uint2 *>(vn + lane * 4);
        k[0] = a.x; k[1] = a.y; v[0] = c.x; v[1] = c.y;
      } else {
        k[0] = *reinterpret_cast<const uint32_t *>(kn + lane * 2);
        v[0] = *reinterpret_cast<const uint32_t *>(vn + lane * 2);
        k[1] = v[1] = 0u;
      }
    } else if constexpr (KV_T == KV_INT8_KCHAN) {
      // keys with the layer's channel scales, values per row as INT8
      float x[E];
      load_row<D, Q_T>(kn, lane, x);
      k[0] = quantize_row_chan<D>(x, p.k_scale + g * D, lane);
      ks = 1.f;
      load_row<D, Q_T>(vn, lane, x);
      v[0] = quantize_row<D, KV_INT8>(x, &vs);
      k[1] = v[1] = 0u;
    } else {
      float x[E];
      load_row<D, Q_T>(kn, lane, x);
      k[0] = quantize_row<D, KV_T>(x, &ks);
      load_row<D, Q_T>(vn, lane, x);
      v[0] = quantize_row<D, KV_T>(x, &vs);
      k[1] = v[1] = 0u;
    }
  }

  // Park this lane's share in shared memory (buf: this warp's [6][32] words)
  // from the piece start to the block that takes it, so that it holds no
  // registers through the blocks before.
  __device__ __forceinline__ void stash(uint32_t *buf, int lane) const {
    buf[lane] = k[0];
    buf[32 + lane] = k[1];
    buf[64 + lane] = v[0];
    buf[96 + lane] = v[1];
    buf[128 + lane] = __float_as_uint(ks);
    buf[160 + lane] = __float_as_uint(vs);
  }
  __device__ __forceinline__ void unstash(const uint32_t *buf, int lane) {
    k[0] = buf[lane];
    k[1] = buf[32 + lane];
    v[0] = buf[64 + lane];
    v[1] = buf[96 + lane];
    ks = __uint_as_float(buf[128 + lane]);
    vs = __uint_as_float(buf[160 + lane]);
  }

  // Put the row in the stage (row r0 + rl of the stage's K / V parts, where the
  // load brought whatever the pool held) and in the pool (block id, head g).
  __device__ __forceinline__ void store(const AttnParams &p, uint8_t *st, int rows, int r, int id,
                                        int g, int rl, int lane) const {
    using T = Tile<D, BS, KV_T>;
    const uint32_t ktile = smem_u32(st);
    const uint32_t vtile = ktile + rows * T::kRowBytes;
    // this lane's bytes within the row (INT4: two codes per byte)
    const uint32_t off = lane * (KV_T == KV_INT4 ? E / 2 : E * T::kElt);
    const uint32_t ka = T::chunk(ktile, r, off >> 4, rows) + (off & 15);
    const uint32_t va = T::chunk(vtile, r, off >> 4, rows) + (off & 15);
    const int64_t grow = (static_cast<int64_t>(id) * p.kv_heads + g) * BS + rl;
    char *kg = p.k_cache + grow * T::kRowBytes + off;
    char *vg = p.v_cache + grow * T::kRowBytes + off;
    constexpr int kBytes = KV_T == KV_INT4 ? E / 2 : E * T::kElt;
    if constexpr (kBytes == 8) {
      asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(ka), "r"(k[0]), "r"(k[1]) : "memory");
      asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(va), "r"(v[0]), "r"(v[1]) : "memory");
      *reinterpret_cast<uint2 *>(kg) = make_uint2(k[0], k[1]);
      *reinterpret_cast<uint2 *>(vg) = make_uint2(v[0], v[1]);
    } else if constexpr (kBytes == 4) {
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(ka), "r"(k[0]) : "memory");
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(va), "r"(v[0]) : "memory");
      *reinterpret_cast<uint32_t *>(kg) = k[0];
      *reinterpret_cast<uint32_t *>(vg) = v[0];
    } else {
      asm volatile("st.shared.u16 [%0], %1;" ::"r"(ka), "h"(static_cast<uint16_t>(k[0])) : "memory");
      asm volatile("st.shared.u16 [%0], %1;" ::"r"(va), "h"(static_cast<uint16_t>(v[0])) : "memory");
      *reinterpret_cast<uint16_t *>(kg) = static_cast<uint16_t>(k[0]);
      *reinterpret_cast<uint16_t *>(vg) = static_cast<uint16_t>(v[0]);
    }
    if constexpr (kScaled) {
      if (lane == 0) {
        if constexpr (T::kKRowScales) {
          reinterpret_cast<float *>(st + 2 * rows * T::kRowBytes)[r] = ks;
          p.k_scale_w[grow] = ks;
        }
        reinterpret_cast<float *>(st + T::vscale_off(rows))[r] = vs;
        p.v_scale_w[grow] = vs;
      }
    }
  }
};

// Position of a CTA's walk over the flattened (unit, block) list. Each unit
// with blocks occupies unit_cost + nb positions: unit_cost positions that
// stand for the fixed work of starting a unit (query load, partial write),
// then one per block. The even split of positions over CTAs thus gives a CTA
// whose share starts a unit fewer blocks.
struct Walk {
  int b;         // sequence
  int gc;        // unit within the sequence: kv head * chunks + chunk
  int j;         // block within the unit
  int nb;        // blocks of sequence b
  long long pos; // flattened position of block j of unit (b, gc)
};

// Positions of one unit of a sequence with nb blocks.
__device__ __forceinline__ int unit_len(int nb, const AttnParams &p) {
  return nb > 0 ? nb + p.unit_cost : 0;
}

template <int BS>
__device__ __forceinline__ void walk_advance(Walk &w, int seg, const AttnParams &p) {
  w.pos += seg;
  w.j += seg;
  if (w.j == w.nb) {
    w.j = 0;
    w.pos += p.unit_cost;  // the next unit's first block
    if (++w.gc == p.units_per_seq) {
      w.gc = 0;
      do {
        ++w.b;
        w.nb = w.b < p.num_seqs ? seq_blocks<BS>(p, w.b) : 0;
      } while (w.b < p.num_seqs && w.nb == 0);
    }
  }
}

// ============================================================================
// Partition kernel: persistent, one producer warp + kNC consumer warps.
// CASC: the attention pass of a cascade step (whole units fold in the shared
// prefix's partials); a separate instantiation, so the plain kernels carry no
// trace of it.
// ============================================================================
template <int D, int BS, int KV_T, int Q_T, bool CASC>
__global__ void __launch_bounds__(kThreads, 1)
attn_partition_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnParams p) {
  using T = Tile<D, BS, KV_T>;
  constexpr unsigned kFull = 0xffffffffu;

  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
  __shared__ int stage_id[kMaxStages];
  __shared__ long long red[kWarps];
  __shared__ long long s_loc[2];
  __shared__ int s_abort;
  __shared__ uint32_t s_newrow[kNC][6 * 32];  // fused append: each warp's new row
  uint8_t *ring = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int c = blockIdx.x;
  const int B = p.num_seqs;
  const int UH = p.units_per_seq;
  const long long G = p.num_ctas;
  const int rows = p.hg * BS;           // rows of one stage's K (or V) part
  const int stride = p.stage_bytes;     // bytes between stages (1024-aligned)
  const int R = p.stages;

  // ---------------------------------------------------------------- prologue
  launch_dependents();      // let the merge kernel be scheduled early
  grid_dependency_wait();   // inputs may come from the previous kernel
  // Total positions over all units, then this CTA's even share [s0, s1).
  long long part = 0;
  for (int b = threadIdx.x; b < B; b += kThreads) {
    const int L = seq_len(p, b);
    // (cascade with an append: the new token must lie past the shared prefix)
    if (L < 0 || L > p.limit || (L == 0 && p.len_off > 0 && p.k_new != nullptr)) {
      if (c == 0) atomicOr(p.status, kErrContext);
    } else {
      part += unit_len((L + BS - 1) / BS, p);
    }
  }
  const long long total = block_sum(part, red) * UH;
  const long long s0 = cta_start(c, total, G), s1 = cta_start(c + 1, total, G);
  if (s0 >= s1) return;  // same for every thread of the CTA

  if (threadIdx.x == 0) {
    s_loc[0] = -1;
    s_abort = 0;
    for (int i = 0; i < R; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kNC);
    }
    fence_barrier_init();
  }
  if (warp == kNC && lane == 0) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
  }
  __syncthreads();
  // Sequence holding position s0 (chunked scan over the sequences).
  long long run = 0;
  for (int base = 0; base < B; base += kThreads) {
    const int b = base + threadIdx.x;
    const int ln = b < B ? unit_len(seq_blocks<BS>(p, b), p) : 0;
    long long tot;
    const long long excl = run + block_excl_scan(ln, red, &tot);
    if (ln > 0 && excl * UH <= s0 && s0 < (excl + ln) * UH) {
      s_loc[0] = b;
      s_loc[1] = excl;
    }
    run += tot;
    __syncthreads();
    if (s_loc[0] >= 0) break;
  }
  if (s_loc[0] < 0) {  // lengths changed under the kernel: nothing consistent to do
    if (threadIdx.x == 0) atomicOr(p.status, kErrContext);
    return;
  }
  Walk w0;
  w0.b = static_cast<int>(s_loc[0]);
  w0.nb = seq_blocks<BS>(p, w0.b);
  {
    // s0 may fall on the unit's start positions: the walk then begins at its
    // first block (possibly past s1: nothing to do here)
    const int ln = unit_len(w0.nb, p);
    const long long off = s0 - s_loc[1] * UH;
    w0.gc = static_cast<int>(off / ln);
    const int jv = static_cast<int>(off - static_cast<long long>(w0.gc) * ln) - p.unit_cost;
    w0.j = jv > 0 ? jv : 0;
    w0.pos = s0 + (jv < 0 ? -jv : 0);
  }

  if (warp == kNC) {
    // ============================================================ producer
    Walk w = w0;
    uint32_t k = 0;
    bool ok = true;
    while (w.pos < s1 && ok) {
      if (w.b >= B || w.nb <= 0) break;  // lengths changed under the kernel
      const int seg = static_cast<int>(min(static_cast<long long>(w.nb - w.j), s1 - w.pos));
      const int head0 = (w.gc / p.cgroups) * p.hg;  // first kv head of the unit
      const int32_t *btrow = p.block_tables + static_cast<int64_t>(w.b) * p.max_blocks + w.j;
      for (int i0 = 0; i0 < seg && ok; i0 += 32) {
        const int cnt = min(32, seg - i0);
        int myid = -1;
        if (lane < cnt) {
          myid = btrow[i0 + lane];
          if (myid < 0 || myid >= p.num_blocks) {
            atomicOr(p.status, kErrBlockId);
            myid = -1;
          }
        }
        for (int i = 0; i < cnt; ++i) {
          const int id = __shfl_sync(kFull, myid, i);
          const int s = k % R;
          int okv = 1;
          if (lane == 0 && k >= static_cast<uint32_t>(R))
            okv = ring_wait(&empty_bar[s], ((k / R) - 1) & 1, &s_abort, p.status);
          okv = __shfl_sync(kFull, okv, 0);
          if (!okv) {
            ok = false;
            break;
          }
          if (lane == 0) {
            stage_id[s] = id;
            const int row0 = id >= 0 ? (id * p.kv_heads + head0) * BS : 0;
            issue_stage<D, BS, KV_T>(ring + s * stride, &full_bar[s], &kmap, &vmap, id, row0,
                                     rows, p);
          }
          __syncwarp();
          ++k;
        }
      }
      walk_advance<BS>(w, seg, p);
    }
    if (!ok && lane == 0) {
      // aborted: let the loads still in flight land before the CTA can exit
      for (uint32_t kk = k > static_cast<uint32_t>(R) ? k - R : 0; kk < k; ++kk)
        mbar_wait(&full_bar[kk % R], (kk / R) & 1, nullptr, 100000000ull);
    }
    return;
  }

  // ============================================================== consumers
  // Consumer warp `warp` owns slot `warp` of each unit: kv head hi = warp / cpg
  // of the unit's group, query-head chunk cl = warp % cpg. Every consumer visits
  // every position (an idle one only releases the stage).
  Consumer<D, BS, KV_T, Q_T> cs;
  Walk w = w0;
  uint32_t k = 0;
  bool alive = true;
  int side = 0;  // the CTA's first piece goes to side 0, the others to side 1
  while (w.pos < s1) {
    if (w.b >= B || w.nb <= 0) {  // same test as the producer: both stop here
      if (warp == 0 && lane == 0) atomicOr(p.status, kErrContext);
      break;
    }
    const int seg = static_cast<int>(min(static_cast<long long>(w.nb - w.j), s1 - w.pos));
    const int hgi = w.gc / p.cgroups;
    const int cgi = w.gc - hgi * p.cgroups;
    const int cpg = min(p.cpg, p.chunks - cgi * p.cpg);
    const bool active = warp < p.hg * cpg;
    const int hi = active ? warp / cpg : 0;
    const int cl = warp - hi * cpg;
    const int g = hgi * p.hg + hi;
    const int chunk = cgi * p.cpg + cl;
    const int h0 = g * p.group + chunk * kChunkHeads;
    const int nh = min(kChunkHeads, p.group - chunk * kChunkHeads);
    const int L = seq_len(p, w.b);
    // fused append: the new token (position L - 1) is in block jl of the unit;
    // with one query-head chunk per kv head this warp alone uses its rows
    const int jl = (L - 1) / BS;
    const bool has_new =
        p.k_new != nullptr && active && L > 0 && jl >= w.j && jl < w.j + seg;
    if (has_new) {  // loaded (quantized) now, parked until its block arrives
      NewRow<D, BS, KV_T, Q_T> nr;
      nr.load(p, w.b, g, lane);
      nr.stash(s_newrow[warp], lane);
    }
    if (active) {
      cs.reset();
      cs.load_query(p, w.b, h0, nh, lane);
    }
    for (uint32_t kk = k; kk < k + seg; ++kk) {
      const int s = kk % R;
      if (alive) {
        int okv = 1;
        if (lane == 0) okv = ring_wait(&full_bar[s], (kk / R) & 1, &s_abort, p.status);
        okv = __shfl_sync(kFull, okv, 0);
        if (!okv) alive = false;
      }
      if (alive) {
        while (!mbar_try_wait(&full_bar[s], (kk / R) & 1)) {
        }  // already complete: gives every lane the acquire
        if (active) {
          const int jb = w.j + static_cast<int>(kk - k);
          const int id = stage_id[s];
          const int valid = id >= 0 ? min(BS, L - jb * BS) : 0;
          if (has_new && jb == jl && id >= 0) {
            const int rl = (L - 1) - jl * BS;
            NewRow<D, BS, KV_T, Q_T> nr;
            nr.unstash(s_newrow[warp], lane);
            nr.store(p, ring + s * stride, rows, hi * BS + rl, id, g, rl, lane);
            // the producer's next TMA into this stage must come after these writes
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
          }
          cs.block(ring + s * stride, rows, hi, valid, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);
      }
    }
    // ------------------------------------------ end of the unit's piece here
    const bool whole = (w.j == 0 && seg == w.nb);
    if (active) {
      const int64_t pbase = ((static_cast<int64_t>(c) * 2 + side) * kNC + warp) * kChunkHeads;
      cs.template finish<CASC>(p, whole, w.b, h0, nh, pbase, alive, lane);
    }
    if (warp == 0 && lane == 0 && w.j == 0) {  // this CTA holds the unit's first block
      const int nu = cta_of(w.pos + w.nb - 1, total, G) - c + 1;
      p.meta[static_cast<int64_t>(w.b) * UH + w.gc] = make_int4(c, nu, side, 0);
    }
    k += seg;
    side = 1;
    walk_advance<BS>(w, seg, p);
  }
}

// ============================================================================
// Merge kernel: one warp per (sequence, query head). Writes zeros for empty or
// invalid sequences; combines the partials of units split across CTAs:
// out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i, M = max_i m_i.
// ============================================================================
constexpr int kMergeWarps = 4;  // small CTAs: one fits beside a partition CTA

template <int D, int OUT_T>
__global__ void __launch_bounds__(kMergeWarps * 32) attn_merge_kernel(const AttnParams p) {
  launch_dependents();
  grid_dependency_wait();  // the partials come from the partition kernel
  const int w = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= p.num_seqs * p.q_heads) return;
  constexpr int E = D / 32;
  const int b = w / p.q_heads;
  const int h = w - b * p.q_heads;
  // (unit, slot, head) of query head h, as the partition kernel assigned them
  const int g = h / p.group;
  const int r = h - g * p.group;
  const int chunk = r / kChunkHeads;
  const int n = r - chunk * kChunkHeads;
  const int hgi = g / p.hg, hi = g - hgi * p.hg;
  const int cgi = chunk / p.cpg, cl = chunk - cgi * p.cpg;
  const int cpg = min(p.cpg, p.chunks - cgi * p.cpg);
  const int slot = hi * cpg + cl;
  // length and bookkeeping in one round trip (the bookkeeping is used only
  // for a valid, non-empty length: it is rewritten for such units every call)
  const int L = seq_len(p, b);
  const int4 mt = p.meta[static_cast<int64_t>(b) * p.units_per_seq + hgi * p.cgroups + cgi];
  const int64_t orow = static_cast<int64_t>(w) * D + lane * E;
  const bool pre = p.pre_o != nullptr;  // cascade: fold in the prefix partial
  const bool valid = L > 0 && L <= p.limit;
  if (!valid && !(pre && L == 0)) {     // (cascade: no position past the prefix)
#pragma unroll
    for (int e = 0; e < E; ++e) store_out<OUT_T>(p.out, orow + e, 0.f);
    return;
  }
  const int nu = valid ? mt.y : 0;
  if (valid && nu <= 1) return;  // finished by the partition kernel
  if (valid && (mt.x < 0 || mt.x >= p.num_ctas || nu < 1 || nu > p.num_ctas - mt.x || (mt.z & ~1))) {
    if (lane == 0) atomicOr(p.status, kErrTimeout);  // bookkeeping not written: phase 1 aborted
    return;
  }
  auto rec = [&](int i) -> int64_t {
    return ((static_cast<int64_t>(mt.x + i) * 2 + (i == 0 ? mt.z : 0)) * kNC + slot) * kChunkHeads + n;
  };
  auto load_o = [&](int i, float (&v)[E]) {
    const float *o = p.part_o + rec(i) * D + lane * E;
    if constexpr (E == 4) {
      const float4 x = *reinterpret_cast<const float4 *>(o);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2 *>(o);
      v[0] = x.x; v[1] = x.y;
    }
  };
  // One online pass over the pieces in order: running max M, sum Ls and
  // output acc. The loads of up to kBatch pieces are issued together, so a
  // unit costs one round trip per kBatch pieces rather than one per piece
  // (10 keeps the kernel at about 90 registers, so a CTA still fits beside an
  // attention CTA's 48k).
  constexpr int kBatch = 10;
  float M = -INFINITY, Ls = 0.f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int i0 = 0; i0 < nu; i0 += kBatch) {
    float2 ml[kBatch];
    float o[kBatch][E];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (i0 + k < nu) {
        ml[k] = *reinterpret_cast<const float2 *>(p.part_ml + rec(i0 + k) * 2);
        load_o(i0 + k, o[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (i0 + k < nu) {
        const float Mn = fmaxf(M, ml[k].x);
        if (Mn != -INFINITY) {
          const float a = exp2_rel(M, Mn), wt = exp2_rel(ml[k].x, Mn);
          Ls = Ls * a + ml[k].y * wt;
#pragma unroll
          for (int e = 0; e < E; ++e) acc[e] = acc[e] * a + o[k][e] * wt;
          M = Mn;
        }
      }
    }
  }
  if (pre) {  // the prefix pass's piece, last
    const float2 ml = *reinterpret_cast<const float2 *>(p.pre_ml + static_cast<int64_t>(w) * 2);
    float o[E];
    const float *src = p.pre_o + orow;
#pragma unroll
    for (int e = 0; e < E; ++e) o[e] = src[e];
    const float Mn = fmaxf(M, ml.x);
    if (Mn != -INFINITY) {
      const float a = exp2_rel(M, Mn), wt = exp2_rel(ml.x, Mn);
      Ls = Ls * a + ml.y * wt;
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = acc[e] * a + o[e] * wt;
    }
  }
  const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) store_out<OUT_T>(p.out, orow + e, acc[e] * inv);
}

// ============================================================================
// Host side
// ============================================================================
using PartFn = cudaError_t (*)(const CUtensorMap &, const CUtensorMap &, const AttnParams &,
                               cudaStream_t);

template <int D, int BS, int KV_T, int Q_T, bool CASC = false>
cudaError_t launch_part(const CUtensorMap &km, const CUtensorMap &vm, const AttnParams &p,
                        cudaStream_t st) {
  const int smem = p.stages * p.stage_bytes + 1024;
  auto kern = attn_partition_kernel<D, BS, KV_T, Q_T, CASC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(p.num_ctas), dim3(kThreads), smem, st, km, vm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int BS>
PartFn pick_dtype(int kv, int q) {
  switch (kv) {
    case KV_BF16: return launch_part<D, BS, KV_BF16, KV_BF16>;
    case KV_FP16: return launch_part<D, BS, KV_FP16, KV_FP16>;
    case KV_INT8:
      return q == KV_BF16 ? launch_part<D, BS, KV_INT8, KV_BF16> : launch_part<D, BS, KV_INT8, KV_FP16>;
    case KV_FP8_E5M2:
      return q == KV_BF16 ? launch_part<D, BS, KV_FP8_E5M2, KV_BF16>
                          : launch_part<D, BS, KV_FP8_E5M2, KV_FP16>;
    case KV_INT8_KCHAN:
      return q == KV_BF16 ? launch_part<D, BS, KV_INT8_KCHAN, KV_BF16>
                          : launch_part<D, BS, KV_INT8_KCHAN, KV_FP16>;
    case KV_INT4:  // pools reject INT4 unless head_dim is 128
      if constexpr (D == 128)
        return q == KV_BF16 ? launch_part<D, BS, KV_INT4, KV_BF16> : launch_part<D, BS, KV_INT4, KV_FP16>;
      else
        return nullptr;
    default:
      return q == KV_BF16 ? launch_part<D, BS, KV_FP8_E5M2_CAST, KV_BF16>
                          : launch_part<D, BS, KV_FP8_E5M2_CAST, KV_FP16>;
  }
}

PartFn pick_partition(int D, int BS, int kv, int q) {
  if (D == 128) return BS == 16 ? pick_dtype<128, 16>(kv, q) : pick_dtype<128, 32>(kv, q);
  return BS == 16 ? pick_dtype<64, 16>(kv, q) : pick_dtype<64, 32>(kv, q);
}

// The cascade step's attention pass: 16-bit caches only.
template <int D, int BS>
PartFn pick_cascade_dtype(int kv) {
  return kv == KV_BF16 ? launch_part<D, BS, KV_BF16, KV_BF16, true>
                       : launch_part<D, BS, KV_FP16, KV_FP16, true>;
}
PartFn pick_cascade(int D, int BS, int kv) {
  if (kv != KV_BF16 && kv != KV_FP16) return nullptr;
  if (D == 128) return BS == 16 ? pick_cascade_dtype<128, 16>(kv) : pick_cascade_dtype<128, 32>(kv);
  return BS == 16 ? pick_cascade_dtype<64, 16>(kv) : pick_cascade_dtype<64, 32>(kv);
}

// Dynamic shared memory a merge CTA reserves without using it: it caps how
// many merge CTAs one SM takes when the attention CTAs drain (measured: CTAs
// piling onto the first SMs to free up made slow outlier steps), while two
// still fit beside a resident attention CTA, so the merge is scheduled early.
constexpr int kMergeSmemReserve = 12 * 1024;

cudaError_t launch_merge(int D, int out_t, const AttnParams &p, cudaStream_t st) {
  const int64_t warps = static_cast<int64_t>(p.num_seqs) * p.q_heads;
  const unsigned grid = static_cast<unsigned>((warps + kMergeWarps - 1) / kMergeWarps);
  const int th = kMergeWarps * 32;
  const int sm = kMergeSmemReserve;
  cudaError_t e;
  if (D == 128) {
    e = out_t == KV_BF16 ? launch_pdl(attn_merge_kernel<128, KV_BF16>, dim3(grid), dim3(th), sm, st, p)
                         : launch_pdl(attn_merge_kernel<128, KV_FP16>, dim3(grid), dim3(th), sm, st, p);
  } else {
    e = out_t == KV_BF16 ? launch_pdl(attn_merge_kernel<64, KV_BF16>, dim3(grid), dim3(th), sm, st, p)
                         : launch_pdl(attn_merge_kernel<64, KV_FP16>, dim3(grid), dim3(th), sm, st, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// How a call's heads are grouped into units (see the kernel's notes).
struct UnitGeom {
  int chunks, cpg, cgroups, hg, units_per_seq, rows, stage_bytes, stages;
};

UnitGeom unit_geom(const kv_pool *pool, int num_q_heads) {
  const kv_pool_desc &d = pool->d;
  UnitGeom u{};
  const int group = num_q_heads / d.num_kv_heads;
  u.chunks = (group + kChunkHeads - 1) / kChunkHeads;
  u.cpg = std::min(u.chunks, kNC);
  u.cgroups = (u.chunks + u.cpg - 1) / u.cpg;
  const int row_bytes = row_bytes_of(d.cache_dtype, d.head_dim);
  const bool quant = has_scales(d.cache_dtype);  // scale rows ride with the stage
  auto load = [&](int hg) { return 2 * hg * d.block_size * (row_bytes + (quant ? 4 : 0)); };
  // the largest group of kv heads (a divisor of Hkv) with one slot per consumer
  // warp, a stage of at most kMaxStageBytes and a TMA box of at most 256 rows
  u.hg = 1;
  for (int hg = 1; hg <= d.num_kv_heads; ++hg) {
    if (d.num_kv_heads % hg) continue;
    if (hg * u.cpg > kNC || load(hg) > kMaxStageBytes || hg * d.block_size > 256) break;
    u.hg = hg;
  }
  u.units_per_seq = (d.num_kv_heads / u.hg) * u.cgroups;
  u.rows = u.hg * d.block_size;
  u.stage_bytes = static_cast<int>(round_up(load(u.hg), 1024));
  u.stages = std::min(kMaxStages, kRingBytes / u.stage_bytes);
  return u;
}

// Workspace: unit metadata, then per-CTA partials (two sides x kNC slots x 8 heads).
struct WsLayout {
  uint64_t meta_off, ml_off, o_off, total;
};

WsLayout ws_layout(int B, int units_per_seq, int G, int D) {
  WsLayout w{};
  const uint64_t recs = static_cast<uint64_t>(G) * 2 * kNC * kChunkHeads;
  w.meta_off = 0;
  w.ml_off = round_up(static_cast<uint64_t>(B) * units_per_seq * 16, 256);
  w.o_off = w.ml_off + round_up(recs * 2 * 4, 256);
  w.total = w.o_off + round_up(recs * D * 4, 256);
  return w;
}

kv_status sm_count(int *n) {
  int dev = 0;
  kv_status s = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (s != KV_OK) return s;
  return cuda_check(cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev),
                    "multiprocessor count");
}

// Shared checks; resolves num_ctas (0 = one per SM).
kv_status check_attn(const kv_pool *pool, int num_seqs, int num_q_heads, int max_context,
                     int num_ctas, int *G) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (num_seqs < 0) return fail(KV_ERR_INVALID, "negative num_seqs");
  const int hkv = pool->d.num_kv_heads;
  if (num_q_heads <= 0 || num_q_heads % hkv != 0)
    return fail(KV_ERR_INVALID, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                num_q_heads, hkv);
  if (static_cast<int64_t>(num_seqs) * num_q_heads > 0x7fffffffLL / 32)
    return fail(KV_ERR_INVALID, "num_seqs * num_q_heads too large");
  if (max_context < 0) return fail(KV_ERR_INVALID, "negative max_context");
  if (num_ctas < 0 || num_ctas > 65535) return fail(KV_ERR_INVALID, "num_ctas must be in [0, 65535]");
  if (num_ctas == 0) {
    kv_status s = sm_count(G);
    if (s != KV_OK) return s;
  } else {
    *G = num_ctas;
  }
  return KV_OK;
}

kv_status fill_params(kv_pool *pool, int layer, const void *q, int num_seqs, int num_q_heads,
                      const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *context_lens, int max_context, float scale, void *out,
                      int G, void *workspace, uint64_t workspace_bytes, AttnParams *pp) {
  const int D = pool->d.head_dim;
  const int group = num_q_heads / pool->d.num_kv_heads;
  const UnitGeom u = unit_geom(pool, num_q_heads);
  const WsLayout wl = ws_layout(num_seqs, u.units_per_seq, G, D);
  if (!workspace || workspace_bytes < wl.total)
    return fail(KV_ERR_INVALID, "workspace of %llu bytes needed, %llu given",
                static_cast<unsigned long long>(wl.total),
                static_cast<unsigned long long>(workspace_bytes));
  if (reinterpret_cast<uintptr_t>(workspace) & 255)
    return fail(KV_ERR_INVALID, "workspace must be 256-byte aligned");
  AttnParams &p = *pp;
  p = AttnParams{};
  p.q = q;
  p.out = out;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.k_scale = layer >= 0 ? layer_ks(pool, layer) : nullptr;
  p.v_scale = layer >= 0 ? layer_vs(pool, layer) : nullptr;
  char *ws = static_cast<char *>(workspace);
  p.meta = reinterpret_cast<int4 *>(ws + wl.meta_off);
  p.part_ml = reinterpret_cast<float *>(ws + wl.ml_off);
  p.part_o = reinterpret_cast<float *>(ws + wl.o_off);
  p.status = status_word(pool);
  p.scale_log2 = scale * kLog2e;
  p.num_seqs = num_seqs;
  p.q_heads = num_q_heads;
  p.kv_heads = pool->d.num_kv_heads;
  p.group = group;
  p.chunks = u.chunks;
  p.hg = u.hg;
  p.cpg = u.cpg;
  p.cgroups = u.cgroups;
  p.units_per_seq = u.units_per_seq;
  p.stage_bytes = u.stage_bytes;
  p.stages = u.stages;
  // starting a unit (query load, partial write) costs about as much as
  // streaming 192 KB on one SM: charged as that many blocks in the split
  p.unit_cost = std::max(1, std::min(8, (192 * 1024 + u.stage_bytes / 2) / u.stage_bytes));
  p.max_blocks = max_blocks_per_seq;
  p.num_blocks = pool->d.num_blocks;
  const int64_t tbl_cap = static_cast<int64_t>(max_blocks_per_seq) * pool->d.block_size;
  p.limit = static_cast<int>(std::min<int64_t>(max_context, tbl_cap));
  p.num_ctas = G;
  return KV_OK;
}

// A cascade step's view of the call: the shared prefix's blocks and where the
// prefix pass leaves its partials.
struct Cascade {
  int prefix_blocks;
  float *pre_o;
  float *pre_ml;
};

// Suffix view of a cascade step: tables from the first block past the prefix
// (same row stride), lengths and limit counted from there.
void apply_cascade(const kv_pool *pool, const Cascade *cas, int32_t max_blocks_per_seq,
                   int32_t max_context, AttnParams *p) {
  if (!cas) return;
  const int bs = pool->d.block_size;
  p->len_off = cas->prefix_blocks * bs;
  if (p->block_tables) p->block_tables += cas->prefix_blocks;
  const int64_t cap = static_cast<int64_t>(max_blocks_per_seq - cas->prefix_blocks) * bs;
  p->limit = static_cast<int>(std::min<int64_t>(max_context - p->len_off, cap));
  p->pre_o = cas->pre_o;
  p->pre_ml = cas->pre_ml;
}

kv_status run_partition(kv_pool *pool, int32_t layer, const void *q, int32_t q_dtype,
                        int32_t num_seqs, int32_t num_q_heads, const int32_t *block_tables,
                        int32_t max_blocks_per_seq, const int32_t *context_lens,
                        int32_t max_context, float scale, void *out, int32_t num_ctas,
                        void *workspace, uint64_t workspace_bytes, const void *k_new,
                        const void *v_new, cudaStream_t st, const Cascade *cas = nullptr) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (layer < 0 || layer >= pool->d.num_layers) return fail(KV_ERR_INVALID, "layer %d out of range", layer);
  const int cd = pool->d.cache_dtype;
  if (q_dtype != KV_BF16 && q_dtype != KV_FP16)
    return fail(KV_ERR_UNSUPPORTED, "q_dtype must be KV_BF16 or KV_FP16");
  if (!is_quant(cd) && q_dtype != cd)
    return fail(KV_ERR_UNSUPPORTED, "a 16-bit cache takes queries of its own dtype");
  if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
    return fail(KV_ERR_INVALID, "scale must be finite");
  if (max_blocks_per_seq <= 0) return fail(KV_ERR_INVALID, "max_blocks_per_seq must be > 0");
  if (num_seqs < 0) return fail(KV_ERR_INVALID, "negative num_seqs");
  if (num_seqs > 0 && (!q || !out || !block_tables || !context_lens))
    return fail(KV_ERR_INVALID, "null pointer");
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(context_lens) & 3))
    return fail(KV_ERR_INVALID, "q and out must be 16-byte aligned, tables and lengths 4-byte");
  int G = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, num_ctas, &G);
  if (s != KV_OK) return s;
  AttnParams p;
  s = fill_params(pool, layer, q, num_seqs, num_q_heads, block_tables, max_blocks_per_seq,
                  context_lens, max_context, scale, out, G, workspace, workspace_bytes, &p);
  if (s != KV_OK) return s;
  apply_cascade(pool, cas, max_blocks_per_seq, max_context, &p);
  if (k_new || v_new) {
    if (!k_new || !v_new) return fail(KV_ERR_INVALID, "k_new and v_new go together");
    if ((reinterpret_cast<uintptr_t>(k_new) & 15) || (reinterpret_cast<uintptr_t>(v_new) & 15))
      return fail(KV_ERR_INVALID, "k_new and v_new must be 16-byte aligned");
    if (p.cpg != 1)
      return fail(KV_ERR_UNSUPPORTED,
                  "the fused append supports up to 8 query heads per kv head; use kv_append "
                  "and paged_attn_decode");
    p.k_new = k_new;
    p.v_new = v_new;
    p.k_cache = layer_k(pool, layer);
    p.v_cache = layer_v(pool, layer);
    p.k_scale_w = layer_ks(pool, layer);
    p.v_scale_w = layer_vs(pool, layer);
  }
  if (num_seqs == 0) return KV_OK;
  kv_status code;
  LayerMaps maps;
  if (!layer_maps(pool, layer, p.hg * pool->d.block_size, &maps, &code)) return code;
  PartFn fn = cas ? pick_cascade(pool->d.head_dim, pool->d.block_size, cd)
                  : pick_partition(pool->d.head_dim, pool->d.block_size, cd, q_dtype);
  if (!fn) return fail(KV_ERR_UNSUPPORTED, "no attention kernel for this cache shape");
  return cuda_check(fn(maps.k, maps.v, p, st), "paged attention launch");
}

kv_status run_merge(kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                    const int32_t *context_lens, int32_t max_blocks_per_seq, int32_t max_context,
                    int32_t num_ctas, int32_t out_dtype, void *out, void *workspace,
                    uint64_t workspace_bytes, cudaStream_t st, const Cascade *cas = nullptr) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (out_dtype != KV_BF16 && out_dtype != KV_FP16)
    return fail(KV_ERR_UNSUPPORTED, "out_dtype must be KV_BF16 or KV_FP16");
  if (max_blocks_per_seq <= 0) return fail(KV_ERR_INVALID, "max_blocks_per_seq must be > 0");
  int G = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, num_ctas, &G);
  if (s != KV_OK) return s;
  if (num_seqs == 0) return KV_OK;
  if (!out || !context_lens) return fail(KV_ERR_INVALID, "null pointer");
  if ((reinterpret_cast<uintptr_t>(out) & 15)) return fail(KV_ERR_INVALID, "out must be 16-byte aligned");
  AttnParams p;
  s = fill_params(pool, -1, nullptr, num_seqs, num_q_heads, nullptr, max_blocks_per_seq,
                  context_lens, max_context, 1.f, out, G, workspace, workspace_bytes, &p);
  if (s != KV_OK) return s;
  apply_cascade(pool, cas, max_blocks_per_seq, max_context, &p);
  return cuda_check(launch_merge(pool->d.head_dim, out_dtype, p, st), "merge launch");
}

// Workspace of a cascade step: the decode workspace, then the prefix pass's
// outputs [num_seqs][Hq][D] and (max, sum) pairs [num_seqs][Hq][2], fp32.
uint64_t cascade_ws(int B, int Hq, int units_per_seq, int G, int D, uint64_t *o_off,
                    uint64_t *ml_off) {
  *o_off = round_up(ws_layout(B, units_per_seq, G, D).total, 256);
  *ml_off = *o_off + round_up(static_cast<uint64_t>(B) * Hq * D * 4, 256);
  return *ml_off + round_up(static_cast<uint64_t>(B) * Hq * 2 * 4, 256);
}

kv_status run_cascade(kv_pool *pool, int32_t layer, const void *q, const void *k_new,
                      const void *v_new, int32_t q_dtype, int32_t num_seqs, int32_t num_q_heads,
                      const int32_t *block_tables, int32_t max_blocks_per_seq,
                      const int32_t *context_lens, int32_t max_context, int32_t prefix_blocks,
                      float scale, void *out, int32_t num_ctas, void *workspace,
                      uint64_t workspace_bytes, cudaStream_t st) {
  if (!pool) return fail(KV_ERR_INVALID, "null pool");
  if (layer < 0 || layer >= pool->d.num_layers) return fail(KV_ERR_INVALID, "layer %d out of range", layer);
  if (is_quant(pool->d.cache_dtype))
    return fail(KV_ERR_UNSUPPORTED, "the cascade step reads 16-bit caches only");
  if (q_dtype != pool->d.cache_dtype) return fail(KV_ERR_UNSUPPORTED, "q_dtype must be the cache dtype");
  if (prefix_blocks < 1 || prefix_blocks >= max_blocks_per_seq)
    return fail(KV_ERR_INVALID, "prefix_blocks must be in [1, max_blocks_per_seq)");
  if (static_cast<int64_t>(prefix_blocks) * pool->d.block_size > max_context)
    return fail(KV_ERR_INVALID, "max_context is shorter than the prefix");
  int G = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, num_ctas, &G);
  if (s != KV_OK) return s;
  if (num_q_heads / pool->d.num_kv_heads > 128)
    return fail(KV_ERR_UNSUPPORTED, "at most 128 query heads per kv head");
  if (num_seqs == 0) return KV_OK;
  if (!q || !out || !block_tables || !context_lens) return fail(KV_ERR_INVALID, "null pointer");
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(out) & 15) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3) || (reinterpret_cast<uintptr_t>(context_lens) & 3))
    return fail(KV_ERR_INVALID, "q and out must be 16-byte aligned, tables and lengths 4-byte");
  if (k_new || v_new) {  // checked before any launch
    if (!k_new || !v_new) return fail(KV_ERR_INVALID, "k_new and v_new go together");
    if ((reinterpret_cast<uintptr_t>(k_new) & 15) || (reinterpret_cast<uintptr_t>(v_new) & 15))
      return fail(KV_ERR_INVALID, "k_new and v_new must be 16-byte aligned");
    if (num_q_heads / pool->d.num_kv_heads > kChunkHeads)
      return fail(KV_ERR_UNSUPPORTED, "the fused append supports up to 8 query heads per kv head");
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255))
    return fail(KV_ERR_INVALID, "workspace must be 256-byte aligned");
  const UnitGeom u = unit_geom(pool, num_q_heads);
  uint64_t o_off = 0, ml_off = 0;
  const uint64_t need = cascade_ws(num_seqs, num_q_heads, u.units_per_seq, G, pool->d.head_dim,
                                   &o_off, &ml_off);
  if (!workspace || workspace_bytes < need)
    return fail(KV_ERR_INVALID, "workspace of %llu bytes needed, %llu given",
                static_cast<unsigned long long>(need), static_cast<unsigned long long>(workspace_bytes));
  Cascade cas{prefix_blocks, reinterpret_cast<float *>(static_cast<char *>(workspace) + o_off),
              reinterpret_cast<float *>(static_cast<char *>(workspace) + ml_off)};
  // 1. the shared prefix, once for all sequences, on the tensor cores (row 0
  //    of the tables names the prefix's blocks, as every row does)
  s = prefix_pass(pool, layer, q, num_seqs, num_q_heads, block_tables, prefix_blocks, scale,
                  cas.pre_o, cas.pre_ml, st);
  if (s != KV_OK) return s;
  // 2. each sequence's positions past the prefix (with the step's append):
  //    a unit finished in one CTA folds in its prefix partials there, split
  //    units leave partials; 3. the merge folds the prefix partial into those
  s = run_partition(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                    max_blocks_per_seq, context_lens, max_context, scale, out, num_ctas,
                    workspace, workspace_bytes, k_new, v_new, st, &cas);
  if (s != KV_OK) return s;
  return run_merge(pool, num_seqs, num_q_heads, context_lens, max_blocks_per_seq, max_context,
                   num_ctas, q_dtype, out, workspace, workspace_bytes, st, &cas);
}

}  // namespace
}  // namespace pagedkv

using namespace pagedkv;

extern "C" {

kv_status paged_attn_workspace_bytes(const kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                                     int32_t num_ctas, uint64_t *bytes) {
  if (!bytes) return fail(KV_ERR_INVALID, "null bytes");
  int G = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, 0, num_ctas, &G);
  if (s != KV_OK) return s;
  const UnitGeom u = unit_geom(pool, num_q_heads);
  *bytes = ws_layout(num_seqs, u.units_per_seq, G, pool->d.head_dim).total;
  return ok();
}

kv_status paged_attn_cascade_workspace_bytes(const kv_pool *pool, int32_t num_seqs,
                                             int32_t num_q_heads, int32_t num_ctas,
                                             uint64_t *bytes) {
  if (!bytes) return fail(KV_ERR_INVALID, "null bytes");
  int G = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, 0, num_ctas, &G);
  if (s != KV_OK) return s;
  const UnitGeom u = unit_geom(pool, num_q_heads);
  uint64_t o_off = 0, ml_off = 0;
  *bytes = cascade_ws(num_seqs, num_q_heads, u.units_per_seq, G, pool->d.head_dim, &o_off, &ml_off);
  return ok();
}

kv_status paged_attn_decode_cascade(kv_pool *pool, int32_t layer, const void *q,
                                    const void *k_new, const void *v_new, int32_t q_dtype,
                                    int32_t num_seqs, int32_t num_q_heads,
                                    const int32_t *block_tables, int32_t max_blocks_per_seq,
                                    const int32_t *context_lens, int32_t max_context,
                                    int32_t prefix_blocks, float scale, void *out,
                                    int32_t num_ctas, void *workspace, uint64_t workspace_bytes,
                                    kv_stream_t stream) {
  kv_status s = run_cascade(pool, layer, q, k_new, v_new, q_dtype, num_seqs, num_q_heads,
                            block_tables, max_blocks_per_seq, context_lens, max_context,
                            prefix_blocks, scale, out, num_ctas, workspace, workspace_bytes,
                            (cudaStream_t)stream);
  return s == KV_OK ? ok() : s;
}

kv_status paged_attn_default_ctas(const kv_pool *pool, int32_t *num_ctas) {
  if (!pool || !num_ctas) return fail(KV_ERR_INVALID, "null argument");
  int n = 0;
  kv_status s = sm_count(&n);
  if (s != KV_OK) return s;
  *num_ctas = n;
  return ok();
}

kv_status paged_attn_partition(kv_pool *pool, int32_t layer, const void *q, int32_t q_dtype,
                               int32_t num_seqs, int32_t num_q_heads, const int32_t *block_tables,
                               int32_t max_blocks_per_seq, const int32_t *context_lens,
                               int32_t max_context, float scale, void *out, int32_t num_ctas,
                               void *workspace, uint64_t workspace_bytes, kv_stream_t stream) {
  kv_status s = run_partition(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                              max_blocks_per_seq, context_lens, max_context, scale, out, num_ctas,
                              workspace, workspace_bytes, nullptr, nullptr, (cudaStream_t)stream);
  return s == KV_OK ? ok() : s;
}

kv_status paged_attn_partition_append(kv_pool *pool, int32_t layer, const void *q,
                                      const void *k_new, const void *v_new, int32_t q_dtype,
                                      int32_t num_seqs, int32_t num_q_heads,
                                      const int32_t *block_tables, int32_t max_blocks_per_seq,
                                      const int32_t *context_lens, int32_t max_context,
                                      float scale, void *out, int32_t num_ctas, void *workspace,
                                      uint64_t workspace_bytes, kv_stream_t stream) {
  if (num_seqs > 0 && (!k_new || !v_new)) return fail(KV_ERR_INVALID, "null k_new / v_new");
  kv_status s = run_partition(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                              max_blocks_per_seq, context_lens, max_context, scale, out, num_ctas,
                              workspace, workspace_bytes, k_new, v_new, (cudaStream_t)stream);
  return s == KV_OK ? ok() : s;
}

kv_status paged_attn_merge(kv_pool *pool, int32_t num_seqs, int32_t num_q_heads,
                           const int32_t *context_lens, int32_t max_blocks_per_seq,
                           int32_t max_context, int32_t num_ctas, int32_t out_dtype, void *out,
                           void *workspace, uint64_t workspace_bytes, kv_stream_t stream) {
  kv_status s = run_merge(pool, num_seqs, num_q_heads, context_lens, max_blocks_per_seq,
                          max_context, num_ctas, out_dtype, out, workspace, workspace_bytes,
                          (cudaStream_t)stream);
  return s == KV_OK ? ok() : s;
}

kv_status paged_attn_decode(kv_pool *pool, int32_t layer, const void *q, int32_t q_dtype,
                            int32_t num_seqs, int32_t num_q_heads, const int32_t *block_tables,
                            int32_t max_blocks_per_seq, const int32_t *context_lens,
                            int32_t max_context, float scale, void *out, int32_t num_ctas,
                            void *workspace, uint64_t workspace_bytes, kv_stream_t stream) {
  kv_status s = run_partition(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                              max_blocks_per_seq, context_lens, max_context, scale, out, num_ctas,
                              workspace, workspace_bytes, nullptr, nullptr, (cudaStream_t)stream);
  if (s != KV_OK) return s;
  if (num_seqs > 0) {
    s = run_merge(pool, num_seqs, num_q_heads, context_lens, max_blocks_per_seq, max_context,
                  num_ctas, q_dtype, out, workspace, workspace_bytes, (cudaStream_t)stream);
    if (s != KV_OK) return s;
  }
  return ok();
}

kv_status paged_attn_decode_append(kv_pool *pool, int32_t layer, const void *q,
                                   const void *k_new, const void *v_new, int32_t q_dtype,
                                   int32_t num_seqs, int32_t num_q_heads,
                                   const int32_t *block_tables, int32_t max_blocks_per_seq,
                                   const int32_t *context_lens, int32_t max_context, float scale,
                                   void *out, int32_t num_ctas, void *workspace,
                                   uint64_t workspace_bytes, kv_stream_t stream) {
  if (num_seqs > 0 && (!k_new || !v_new)) return fail(KV_ERR_INVALID, "null k_new / v_new");
  kv_status s = run_partition(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                              max_blocks_per_seq, context_lens, max_context, scale, out, num_ctas,
                              workspace, workspace_bytes, k_new, v_new, (cudaStream_t)stream);
  if (s != KV_OK) return s;
  if (num_seqs > 0) {
    s = run_merge(pool, num_seqs, num_q_heads, context_lens, max_blocks_per_seq, max_context,
                  num_ctas, q_dtype, out, workspace, workspace_bytes, (cudaStream_t)stream);
    if (s != KV_OK) return s;
  }
  return ok();
}

}  // extern "C"

// ============================================================================
// Decode attention for callers that cannot allocate a workspace.
//
// Some callers cannot hand this library a workspace: a serving process that
// has already given all of the GPU's free memory to its KV pool and admits no
// further allocation, or a host application that reaches this library through
// a plugin or foreign-function interface with no access to a device
// allocator. For them, paged_attn_decode_static keeps the split-K scratch in a
// fixed array compiled into this library instead. Every GPU that loads the
// library holds that array until the process exits.
// ============================================================================

// The scratch: unit bookkeeping and split partials, as for a caller workspace.
static __device__ __align__(256) unsigned char g_decode_scratch[16u << 20];

namespace pagedkv {
namespace {

constexpr uint64_t kStaticScratchBytes = 16ull << 20;
constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxScratchDevices];  // device address of the array, per device

// Device address of the scratch array on the current device. Host code cannot
// use the array's name as a device pointer (it is a host-side stand-in), so the
// address is looked up once per device, with that device current. The stream
// the kernels go to must belong to that device (another device's stream would
// be handed this device's array).
kv_status scratch_address(cudaStream_t stream, void **out) {
  int dev = 0;
  kv_status s = cuda_check(cudaGetDevice(&dev), "cudaGetDevice");
  if (s != KV_OK) return s;
  if (dev < 0 || dev >= kMaxScratchDevices)
    return fail(KV_ERR_UNSUPPORTED, "device %d: at most %d devices", dev, kMaxScratchDevices);
  if (stream) {
    int sdev = -1;
    s = cuda_check(cudaStreamGetDevice(stream, &sdev), "cudaStreamGetDevice");
    if (s != KV_OK) return s;
    if (sdev != dev)
      return fail(KV_ERR_INVALID, "the stream belongs to device %d, the current device is %d",
                  sdev, dev);
  }
  std::lock_guard<std::mutex> g(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void *ptr = nullptr;
    s = cuda_check(cudaGetSymbolAddress(&ptr, g_decode_scratch), "scratch address");
    if (s != KV_OK) return s;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return KV_OK;
}

}  // namespace
}  // namespace pagedkv

extern "C" kv_status paged_attn_decode_static(kv_pool *pool, int32_t layer, const void *q,
                                              int32_t q_dtype, int32_t num_seqs,
                                              int32_t num_q_heads, const int32_t *block_tables,
                                              int32_t max_blocks_per_seq,
                                              const int32_t *context_lens, int32_t max_context,
                                              float scale, void *out, int32_t num_ctas,
                                              kv_stream_t stream) {
  int G = 0;
  kv_status s = check_attn(pool, num_seqs, num_q_heads, max_context, num_ctas, &G);
  if (s != KV_OK) return s;
  const UnitGeom u = unit_geom(pool, num_q_heads);
  const uint64_t need = ws_layout(num_seqs, u.units_per_seq, G, pool->d.head_dim).total;
  if (need > kStaticScratchBytes)
    return fail(KV_ERR_INVALID,
                "these sizes need %llu bytes of scratch; the built-in scratch holds %llu "
                "(use fewer sequences or CTAs, or paged_attn_decode with a workspace)",
                static_cast<unsigned long long>(need),
                static_cast<unsigned long long>(kStaticScratchBytes));
  void *ws = nullptr;
  s = scratch_address((cudaStream_t)stream, &ws);
  if (s != KV_OK) return s;
  // Nothing in the scratch needs to start at zero: the partition kernel writes
  // every bookkeeping entry and partial that the merge kernel then reads.
  return paged_attn_decode(pool, layer, q, q_dtype, num_seqs, num_q_heads, block_tables,
                           max_blocks_per_seq, context_lens, max_context, scale, out, num_ctas,
                           ws, kStaticScratchBytes, stream);
}
