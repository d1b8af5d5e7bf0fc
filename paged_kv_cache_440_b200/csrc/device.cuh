// Device-side building blocks for sm_100a: mbarrier waits with a time limit,
// TMA tile loads and 1-D bulk copies into this CTA's own shared memory only,
// warp-level fragment loads and tensor-core MMA, and the
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

// As mbar_try_wait, but the thread may sleep up to `ns` nanoseconds for the
// phase to complete (it wakes as soon as it does) instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
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

// 3-D tiled tensor load global -> shared (this CTA), completion on `bar`.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 4-D tiled tensor load global -> shared (this CTA), completion on `bar`.
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
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

// D = A(16x32, row) * B(32x8, col) + D on 8-bit integers, exact int32
// accumulation. A signed (s8) or unsigned (u8) as kUnsignedA says, B signed.
// A's four registers are what one ldmatrix.x4 of a 16-row x 32-byte tile
// gives (rows 0-7 / 8-15 of bytes 0-15, then of bytes 16-31).
template <bool kUnsignedA>
__device__ __forceinline__ void mma16832_i8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
  if constexpr (kUnsignedA) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
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
// An INT4 code c (two's complement nibble) is offset binary u = c + 8 after
// flipping its top bit. Nibbles K and K + 4 of a 32-bit word of codes, masked,
// flipped and placed under the fp16 exponent byte 0x64 in one logic op
// ((x & 0x000F000F) ^ 0x64086408), are 1024 + u: an exact pair, 1032 above the
// codes.
template <int K>
__device__ __forceinline__ uint32_t int4_pair_biased(uint32_t w) {
  return ((w >> (4 * K)) & 0x000F000Fu) ^ 0x64086408u;
}
template <int K>
__device__ __forceinline__ uint32_t int4_pair(uint32_t w) {
  uint32_t h = int4_pair_biased<K>(w);
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

// One row's D/32 16-bit values of this lane, as loaded (the loads of the
// next row can be in flight while this one is converted and quantized).
template <int D>
struct RawRow {
  uint32_t w[D / 64];
};

template <int D>
__device__ __forceinline__ RawRow<D> load_row_raw(const uint16_t *__restrict__ src, int lane) {
  RawRow<D> r;
  if constexpr (D / 32 == 4) {
    const uint2 v = *reinterpret_cast<const uint2 *>(src + lane * 4);
    r.w[0] = v.x;
    r.w[1] = v.y;
  } else {
    r.w[0] = *reinterpret_cast<const uint32_t *>(src + lane * 2);
  }
  return r;
}

template <int D, int IN_T>
__device__ __forceinline__ void raw_to_f32(const RawRow<D> &r, float (&x)[D / 32]) {
#pragma unroll
  for (int i = 0; i < D / 64; ++i) {
    x[2 * i] = to_f32<IN_T>(r.w[i] & 0xFFFF);
    x[2 * i + 1] = to_f32<IN_T>(r.w[i] >> 16);
  }
}

template <int D, int IN_T>
__device__ __forceinline__ void load_row(const uint16_t *__restrict__ src, int lane,
                                         float (&x)[D / 32]) {
  raw_to_f32<D, IN_T>(load_row_raw<D>(src, lane), x);
}

// INT8 codes of this lane's share of a key row with one fixed scale per
// channel: code = clamp(round-half-even(fl32(x / s)), -127, 127), 0 where the
// scale is not positive. cs: the head's head_dim channel scales.
template <int D>
__device__ __forceinline__ uint32_t quantize_row_chan(const float (&x)[D / 32], const float *cs,
                                                      int lane) {
  constexpr int E = D / 32;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const float s = cs[lane * E + i];
    int q = 0;
    if (s > 0.f) {
      q = __float2int_rn(__fdiv_rn(x[i], s));
      q = max(-127, min(127, q));
    }
    packed |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * i);
  }
  return packed;
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

// ------------------------------------------------------------ packed fp32
// Two fp32 lanes per instruction (sm_100 f32x2 arithmetic), round to nearest.

#define PAGEDKV_F32X2(NAME, OP)                                                          \
  __device__ __forceinline__ float2 NAME(float2 a, float2 b) {                            \
    float2 r;                                                                             \
    asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t" OP \
        " d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"                                          \
        : "=f"(r.x), "=f"(r.y)                                                            \
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));                                        \
    return r;                                                                             \
  }
PAGEDKV_F32X2(mul2, "mul.rn.f32x2")
PAGEDKV_F32X2(add2, "add.rn.f32x2")
PAGEDKV_F32X2(sub2, "sub.rn.f32x2")
#undef PAGEDKV_F32X2

// a * b + c on two lanes, one rounding (sm_100 f32x2 fused multiply-add).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mov.b64 c, {%6, %7};\n\tfma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return r;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ------------------------------------------------------------------ tcgen05
// Fifth-generation tensor core: MMAs issued by one thread read both operands
// from shared memory through 64-bit matrix descriptors and accumulate in
// tensor memory (TMEM: 128 lanes x 512 columns of 32 bits per SM).

// Shared-memory matrix descriptor, 128-byte swizzle (the layout TMA writes
// with CU_TENSOR_MAP_SWIZZLE_128B): start address, leading and stride byte
// offsets (16-byte units), descriptor version 1, layout type 2. Operand tiles
// start on 1024-byte boundaries; a K offset inside a 128-byte row moves the
// start address. K-major: 8-row groups `sbo` bytes apart, `lbo` unused (1).
// MN-major: `lbo` is the distance between 64-element column slabs, `sbo`
// between 8-row groups along K.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16 with fp32 accumulation: A and B both
// bf16 (or both fp16), M x N tile, A K-major, B K-major or MN-major.
template <bool BF16>
__device__ __forceinline__ uint32_t umma_idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (BF16 ? (1u << 7) | (1u << 10) : 0u) | (b_mn_major ? (1u << 16) : 0u) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]: A is M x 16 with row r in lane r and two
// 16-bit K elements per 32-bit column (the lower K index in the low half).
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                                uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// As umma_f16_tmem_a with a compile-time accumulate flag (no predicate setup).
template <bool ACC>
__device__ __forceinline__ void umma_f16_tmem_a_c(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                                  uint32_t idesc) {
  if constexpr (ACC) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, 0, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.u32 p, 0, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc)
        : "memory");
  }
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Make this thread's shared-memory writes visible to the async proxy (TMA,
// tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Whole-warp TMEM allocation of `cols` columns; the base address lands in *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols)
               : "memory");
}

// 32 consecutive columns of this warp's 32 lanes: lane i gets row i's values.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
        "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
        "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// 16 consecutive columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
        "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}

// N (16 or 32) consecutive columns.
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&v)[N]) {
  if constexpr (N == 32) tmem_ld32(taddr, v);
  else tmem_ld16(taddr, v);
}
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[N]) {
  if constexpr (N == 32) tmem_st32(taddr, v);
  else tmem_st16(taddr, v);
}

// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace dev
}  // namespace pagedkv
