"""KV-cache quantization reference: INT8 and FP8-E5M2 with per-token-head scales,
INT8 keys with per-channel scales.

Test infrastructure only (see ``oracle/__init__``).

What the pages fix:
* KV can be stored as FP8 or INT8 and is dequantized before use
  [KV Cache 原理与 PagedAttention, §四 "KV Cache 量化" table; the FP8 flavour named
  there is ``fp8_e5m2``].
* The finest granularity listed, one scale per token per attention head
  ("per-token-head"), is the one in mainstream use
  [bjdmk.com.cn/news/6246348, §5.2].

What they leave open, and the reading taken here (plain symmetric absmax):
* a = max |x| over the D values of one (token, head) row;
* scale = fl32(a / QMAX), QMAX = 127 for INT8 and 57344 (largest finite E5M2) for FP8;
* y = fl32(x / scale) (IEEE fp32 division, correctly rounded);
* INT8 code = clamp(round-half-even(y), -127, 127);
  E5M2 code = round-half-even of y to 1-5-2 with saturation to +-57344;
* a == 0 gives scale 0 and all-zero codes;
* dequantized value = code * scale.

The E5M2 encoder/decoder below are written from the format definition (OCP 8-bit
floating point specification, E5M2: 1 sign bit, 5 exponent bits with bias 15,
2 mantissa bits, subnormals when the exponent field is 0, exponent field 31 for
Inf/NaN), working on the raw fp32 bits.
"""
import numpy as np

QMAX_INT8 = np.float32(127.0)
QMAX_INT4 = np.float32(7.0)
QMAX_E5M2 = np.float32(57344.0)       # (1 + 3/4) * 2**15
E5M2_MAX_CODE = 0x7B                  # exponent field 30, mantissa 3


def e5m2_decode(codes):
    """E5M2 byte(s) -> float64 value(s), from the format definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 2) & 0x1F
    m = (c & 3).astype(np.float64)
    normal = np.ldexp(1.0 + m / 4.0, (e - 15).astype(np.int64))
    subnormal = np.ldexp(m / 4.0, -14)
    val = np.where(e == 0, subnormal, normal)
    val = np.where(e == 31, np.where(m == 0, np.inf, np.nan), val)
    return sign * val


def e5m2_encode(y):
    """float32 value(s) -> E5M2 byte(s): round to nearest, ties to even, saturating.

    Magnitudes that round above the largest finite value (57344) saturate to it;
    infinities saturate as well. NaN maps to 0x7F (never produced by quantize).
    """
    y = np.asarray(y, dtype=np.float32)
    bits = y.view(np.uint32).astype(np.int64)
    sign = (bits >> 31) & 1
    E = (bits >> 23) & 0xFF
    M = bits & 0x7FFFFF
    is_nan = (E == 0xFF) & (M != 0)
    is_inf = (E == 0xFF) & (M == 0)

    # Normal results: E5M2 exponent field = E - 127 + 15 = E - 112 >= 1.
    # Keep the top 2 mantissa bits, round on the 21 dropped bits (ties to even).
    # A carry out of the mantissa correctly bumps the exponent field.
    mag_n = ((E - 112) << 2) | (M >> 21)
    rem = M & ((1 << 21) - 1)
    half = 1 << 20
    up = (rem > half) | ((rem == half) & ((mag_n & 1) == 1))
    mag_n = mag_n + up.astype(np.int64)

    # Subnormal results (E <= 112): the value in units of 2**-16 (the E5M2
    # subnormal step) is sig * 2**(E - 134), sig the 24-bit significand; round
    # that to an integer, ties to even. A result of 4 is the smallest normal
    # (exponent field 1, mantissa 0), which the plain integer already encodes.
    sig = np.where(E == 0, M, M | (1 << 23))
    e_eff = np.where(E == 0, 1, E)             # fp32 subnormals share exponent -126
    sh = np.clip(134 - e_eff, 0, 62)
    q = sig >> sh
    r = sig - (q << sh)
    halfs = np.where(sh > 0, np.left_shift(np.int64(1), np.maximum(sh - 1, 0)), 0)
    up_s = (sh > 0) & ((r > halfs) | ((r == halfs) & ((q & 1) == 1)))
    mag_s = q + up_s.astype(np.int64)

    mag = np.where(E >= 113, mag_n, mag_s)
    mag = np.minimum(mag, E5M2_MAX_CODE)       # saturate (covers rounding into Inf)
    mag = np.where(is_inf, E5M2_MAX_CODE, mag)
    code = (sign << 7) | mag
    code = np.where(is_nan, 0x7F, code)
    return code.astype(np.uint8)


def int8_encode(y):
    """float32 value(s) -> INT8: round half to even, clamp to [-127, 127]."""
    y = np.asarray(y, dtype=np.float32)
    r = np.rint(y.astype(np.float64))          # numpy rint rounds half to even
    return np.clip(r, -127, 127).astype(np.int8)


def int4_encode(y):
    """float32 value(s) -> 4-bit codes (held in int8): round half to even,
    clamp to [-7, 7] (symmetric; -8 is not used)."""
    y = np.asarray(y, dtype=np.float32)
    return np.clip(np.rint(y.astype(np.float64)), -7, 7).astype(np.int8)


def pack_int4(codes):
    """[..., D] codes in [-8, 7] -> [..., D/2] bytes: element 2i in the low
    nibble of byte i, element 2i+1 in the high nibble (two's complement)."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed):
    """Inverse of pack_int4: [..., D/2] bytes -> [..., D] int8 codes."""
    b = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo, hi = b & 0xF, b >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def quantize_rows(x, kind):
    """Per-row symmetric absmax quantization.

    x: float32-representable values, shape [..., D]; each row of D values is one
       (token, kv head) of K or V.
    kind: "int8", "int4" (codes unpacked, one per int8), "e5m2" or
    "e5m2_cast" (no scale).
    Returns (codes [..., D] int8|uint8, scales [...] float32).
    """
    x = np.asarray(x, dtype=np.float32)
    if kind == "e5m2_cast":
        # FP8 storage with no scale: each value cast to E5M2 (round to nearest
        # even, saturating), dequantized as the code's value [KV Cache 原理与
        # PagedAttention, §四: FP8 KV stored in FP8 and converted back before
        # use; the vLLM example's fp8_e5m2 KV dtype]. Scales are reported as 1.
        return e5m2_encode(x), np.ones(x.shape[:-1], dtype=np.float32)
    # INT4 KV (the pages' most aggressive row, 1/4 of the memory [KV Cache
    # 原理与 PagedAttention, §四 table]): the same per-token-head absmax form
    # with QMAX 7; the pages' calibration needs data and is not modelled.
    qmax = {"int8": QMAX_INT8, "int4": QMAX_INT4}.get(kind, QMAX_E5M2)
    a = np.max(np.abs(x), axis=-1)                            # exact in fp32
    scale = np.divide(a, qmax, dtype=np.float32)               # fl32(a / QMAX)
    nz = scale > 0
    safe = np.where(nz, scale, np.float32(1.0))
    y = np.divide(x, safe[..., None], dtype=np.float32)        # fl32(x / scale)
    if kind == "int8":
        codes = int8_encode(y)
        codes = np.where(nz[..., None], codes, np.int8(0)).astype(np.int8)
    elif kind == "int4":
        codes = int4_encode(y)
        codes = np.where(nz[..., None], codes, np.int8(0)).astype(np.int8)
    elif kind == "e5m2":
        codes = e5m2_encode(y)
        codes = np.where(nz[..., None], codes, np.uint8(0)).astype(np.uint8)
    else:
        raise ValueError(kind)
    scale = np.where(nz, scale, np.float32(0.0)).astype(np.float32)
    return codes, scale


def dequantize(codes, scales, kind):
    """codes [..., D], scales [...] -> float64 values code * scale (exact in fp64)."""
    if kind in ("int8", "int4"):
        v = np.asarray(codes, dtype=np.int8).astype(np.float64)
    elif kind in ("e5m2", "e5m2_cast"):
        v = e5m2_decode(codes)
    else:
        raise ValueError(kind)
    return v * np.asarray(scales, dtype=np.float32).astype(np.float64)[..., None]


def quantize_k_channels(k, chan_scales):
    """INT8 keys with one scale per (kv head, channel).

    The pages list per-channel granularity (one scale per channel) beside
    per-tensor and per-token-head, and suggest per-channel or per-token for K
    while V may take a coarser one [bjdmk.com.cn/news/6246348, §5.2; KV Cache
    原理与 PagedAttention, §四 table, INT8 row: per-tensor/per-channel].
    Readings (the pages fix none of these): the scales are fixed for a layer
    (calibrated or set by the caller, not derived from the rows being
    written); y = fl32(k / s_c) (IEEE fp32 division); code = clamp(
    round-half-even(y), -127, 127); a zero scale gives code 0.

    k: [..., H, D] float32-representable values; chan_scales: [H, D] float32.
    Returns int8 codes of k's shape.
    """
    k = np.asarray(k, dtype=np.float32)
    s = np.asarray(chan_scales, dtype=np.float32)
    nz = s > 0
    safe = np.where(nz, s, np.float32(1.0))
    y = np.divide(k, safe, dtype=np.float32)                  # fl32(k / s), broadcast [H, D]
    codes = int8_encode(y)
    return np.where(nz, codes, np.int8(0)).astype(np.int8)


def dequantize_k_channels(codes, chan_scales):
    """codes [..., H, D] int8, chan_scales [H, D] -> float64 code * s_c (exact)."""
    return np.asarray(codes, dtype=np.int8).astype(np.float64) * \
        np.asarray(chan_scales, dtype=np.float32).astype(np.float64)
