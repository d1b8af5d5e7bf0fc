// Device-side building blocks for sm_100a: mbarrier waits with a time limit,
// TMA tile loads and 1-D bulk copies into shared memory (CTA-local, never
// multicast), warp-level fragment loads and tensor-core MMA, and the
// conversions of 1-byte KV codes to fp16.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "pagedkv.h"

namespace pagedkv {
namespace dev {

// Status bits (mirror KV_DEVERR_* of pagedkv.h plus the timeout bit).
constexpr int kErrBlockId = 1;
constexpr int kErrContext = 2;
constexpr int kErrSlot = 4;
constexpr int kErrTimeout = 8;

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------- programmatic dependent launch
// Kernels of this library are launched so that the next kernel in the stream
// may be scheduled before they finish (launch_dependents). Each kernel waits
// for the previous grid to complete, with its memory visible, before it reads
// any input (grid_dependency_wait); without such a launch both are no-ops.

__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase with the given parity to complete. Gives up after
// limit_ns, sets kErrTimeout in *status and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63) == 0 && globaltimer() - t0 > limit_ns) {
      if (status) atomicOr(status, kErrTimeout);
      return false;
    }
  }
}

// ------------------------------------------------------------------ TMA / bulk

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled tensor load global -> shared (this CTA), completion on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 1-D bulk copy global -> shared (this CTA). dst, src 16-byte aligned; bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------ fragments

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                          uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose an 8x8 matrix of 16-bit elements held one 32-bit pair per lane.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// D = A(16x16, row) * B(16x8, col) + D, fp32 accumulate.
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Pack two floats into a 16-bit pair (low half = lo), round to nearest even.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
  }
}

// Split two floats into 16-bit pairs hi + lo with hi = round(x) and
// lo = round(x - hi): hi + lo carries x to about 2^-17 (bf16) or 2^-22 (fp16)
// relative, so an MMA on both parts loses almost nothing to operand rounding.
template <bool BF16>
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
  hi = pack2<BF16>(a, b);
  float ha, hb;
  if constexpr (BF16) {
    ha = __uint_as_float(hi << 16);
    hb = __uint_as_float(hi & 0xFFFF0000u);
  } else {
    ha = __half2float(__ushort_as_half(static_cast<unsigned short>(hi & 0xFFFFu)));
    hb = __half2float(__ushort_as_half(static_cast<unsigned short>(hi >> 16)));
  }
  lo = pack2<BF16>(a - ha, b - hb);
}

// -------------------------------------------------- 4-bit codes -> fp16 pairs
//
// INT4 codes (two's complement nibbles) become offset binary u = code + 8 when
// the caller xors the word with 0x88888888. Nibbles K and K + 4 of a 32-bit
// word, placed under the fp16 exponent byte 0x64, are 1024 + u: an exact pair,
// 1032 above the codes.
template <int K>
__device__ __forceinline__ uint32_t int4_pair_biased(uint32_t w_biased) {
  return ((w_biased >> (4 * K)) & 0x000F000Fu) | 0x64006400u;
}
template <int K>
__device__ __forceinline__ uint32_t int4_pair(uint32_t w_biased) {
  uint32_t h = int4_pair_biased<K>(w_biased);
  __half2 v = *reinterpret_cast<__half2 *>(&h);
  const __half2 bias = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
  v = __hsub2(v, bias);
  return *reinterpret_cast<uint32_t *>(&v);
}

// -------------------------------------------------- 1-byte codes -> fp16 pairs
//
// An E5M2 byte is the high byte of the fp16 with the same value (same sign,
// exponent width and bias; the two mantissa bits are fp16's top two), so
// placing the byte in the high half of a 16-bit lane is an exact conversion.
// An INT8 code c in [-127, 127] becomes exact fp16 through the biased byte
// u = c + 128 (the caller xors the source word with 0x80808080): the fp16 with
// bits 0x64:u is 1024 + u, and subtracting 1152 leaves c.
//
// Both take bytes A and B (0..3) of the 32-bit source and return them as an
// fp16 pair, byte A in the low half.

template <int A, int B>
__device__ __forceinline__ uint32_t e5m2_pair(uint32_t src) {
  // result bytes: [0] = 0, [1] = src[A], [2] = 0, [3] = src[B]
  return prmt(src, 0u, (B << 12) | (4 << 8) | (A << 4) | 4);
}

// Two INT8 codes (sign bit flipped by the caller) as fp16 1152 + code, exact:
// the bias stays in and is removed from the dot product by the caller.
template <int A, int B>
__device__ __forceinline__ uint32_t int8_pair_biased(uint32_t src_biased) {
  // result bytes: [0] = u[A], [1] = 0x64, [2] = u[B], [3] = 0x64 -> 1024 + u
  return prmt(src_biased, 0x64646464u, (4 << 12) | (B << 8) | (4 << 4) | A);
}

template <int A, int B>
__device__ __forceinline__ uint32_t int8_pair(uint32_t src_biased) {
  // result bytes: [0] = u[A], [1] = 0x64, [2] = u[B], [3] = 0x64
  uint32_t h = prmt(src_biased, 0x64646464u, (4 << 12) | (B << 8) | (4 << 4) | A);
  __half2 v = *reinterpret_cast<__half2 *>(&h);
  const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
  v = __hsub2(v, bias);
  return *reinterpret_cast<uint32_t *>(&v);
}

// ------------------------------------------------ per-row KV quantization
// One warp handles one row of D values, lane l holding elements
// l * D/32 .. l * D/32 + D/32 - 1 (used by the append kernel and by the
// attention kernel's fused append, so both produce the same bytes).

template <int IN_T>
__device__ __forceinline__ float to_f32(uint16_t bits) {
  if constexpr (IN_T == KV_BF16) {
    return __uint_as_float(static_cast<uint32_t>(bits) << 16);
  } else {
    return __half2float(__ushort_as_half(bits));
  }
}

// Quantize one row of D values held as D/32 per lane; returns the packed codes
// of this lane (D/32 bytes, little-endian in order) and the row scale.
template <int D, int OUT_T>
__device__ __forceinline__ uint32_t quantize_row(const float (&x)[D / 32], float *scale_out) {
  constexpr int E = D / 32;
  if constexpr (OUT_T == KV_FP8_E5M2_CAST) {  // plain cast: no scale, saturating RNE
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < E; ++i)
      packed |= static_cast<uint32_t>(__nv_cvt_float_to_fp8(x[i], __NV_SATFINITE, __NV_E5M2))
                << (8 * i);
    *scale_out = 1.f;
    return packed;
  }
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  constexpr float kQmax = OUT_T == KV_INT8 ? 127.0f : OUT_T == KV_INT4 ? 7.0f : 57344.0f;
  uint32_t packed = 0;
  float scale = 0.f;
  if (a > 0.f) {
    scale = __fdiv_rn(a, kQmax);
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float y = __fdiv_rn(x[i], scale);
      uint32_t code;
      if constexpr (OUT_T == KV_INT8) {
        int q = __float2int_rn(y);
        q = max(-127, min(127, q));
        code = static_cast<uint32_t>(q) & 0xFFu;
      } else if constexpr (OUT_T == KV_INT4) {
        int q = __float2int_rn(y);
        q = max(-7, min(7, q));
        code = static_cast<uint32_t>(q) & 0xFu;
        packed |= code << (4 * i);  // two codes per byte, element 2i low
        continue;
      } else {
        code = static_cast<uint32_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E5M2));
      }
      packed |= code << (8 * i);
    }
  }
  *scale_out = scale;
  return packed;
}

template <int D, int IN_T>
__device__ __forceinline__ void load_row(const uint16_t *__restrict__ src, int lane,
                                         float (&x)[D / 32]) {
  constexpr int E = D / 32;
  if constexpr (E == 4) {
    uint2 v = *reinterpret_cast<const uint2 *>(src + lane * 4);
    x[0] = to_f32<IN_T>(v.x & 0xFFFF);
    x[1] = to_f32<IN_T>(v.x >> 16);
    x[2] = to_f32<IN_T>(v.y & 0xFFFF);
    x[3] = to_f32<IN_T>(v.y >> 16);
  } else {
    uint32_t v = *reinterpret_cast<const uint32_t *>(src + lane * 2);
    x[0] = to_f32<IN_T>(v & 0xFFFF);
    x[1] = to_f32<IN_T>(v >> 16);
  }
}

// Store this lane's codes of one row (row base `dst`): D/32 bytes, or D/64
// for INT4 (4 bits per code).
template <int D, int OUT_T = KV_INT8>
__device__ __forceinline__ void store_codes(uint8_t *dst, int lane, uint32_t packed) {
  if constexpr (OUT_T == KV_INT4) {
    static_assert(D == 128, "INT4 rows need head_dim 128");
    reinterpret_cast<uint16_t *>(dst)[lane] = static_cast<uint16_t>(packed);
  } else if constexpr (D == 128) {
    reinterpret_cast<uint32_t *>(dst)[lane] = packed;
  } else {
    reinterpret_cast<uint16_t *>(dst)[lane] = static_cast<uint16_t>(packed);
  }
}

}  // namespace dev
}  // namespace pagedkv
