"""Pins for the quantization oracle.

* E5M2 decode of all 256 codes against torch's float8_e5m2 (an independent
  implementation of the same OCP format);
* E5M2 encode against torch's float8_e5m2 conversion on values below the
  saturation threshold (torch rounds to nearest-even but overflows to Inf where
  this encoder saturates), plus every code round-tripping and every midpoint
  between neighbouring codes going to the even code;
* INT8 rounding against the definition of round-half-even;
* hand-derived rows (tests/golden/quant_hand.json);
* error bounds of the quantizer that follow from its definition.
"""
import json
import os

import numpy as np
import torch

from oracle import quant

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quant_hand.json")


def _torch_e5m2_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e5m2) \
        .view(torch.uint8).numpy()


def test_e5m2_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = quant.e5m2_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e5m2).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    assert quant.e5m2_decode(np.uint8(0x7B)) == 57344.0


def test_e5m2_roundtrip_every_finite_code():
    codes = np.arange(256, dtype=np.uint8)
    vals = quant.e5m2_decode(codes)
    finite = np.isfinite(vals)
    back = quant.e5m2_encode(vals[finite].astype(np.float32))
    assert np.array_equal(back, codes[finite])


def test_e5m2_midpoints_go_to_even_code():
    pos = np.arange(0, 0x7C, dtype=np.uint8)             # +0 .. max finite, then Inf
    v = quant.e5m2_decode(pos)
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (v[:-1] + v[1:]) / 2)  # exact in fp32
    enc = quant.e5m2_encode(mids)
    lo, hi = pos[:-1], pos[1:]
    expect = np.where(lo % 2 == 0, lo, hi)
    assert np.array_equal(enc, expect)
    # one fp32 ulp either side of the midpoint decides by distance
    below = np.nextafter(mids, np.float32(0))
    above = np.nextafter(mids, np.float32(np.inf))
    assert np.array_equal(quant.e5m2_encode(below), lo)
    assert np.array_equal(quant.e5m2_encode(above), hi)
    assert np.array_equal(quant.e5m2_encode(-mids), expect | 0x80)


def test_e5m2_encode_matches_torch_in_range():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(200000) * 10.0 ** rng.uniform(-7, 4.6, 200000),
        rng.uniform(-61439, 61439, 20000),
        rng.standard_normal(20000) * 1e-5,                       # subnormal region
    ]).astype(np.float32)
    x = x[np.abs(x) < 61440]
    assert np.array_equal(quant.e5m2_encode(x), _torch_e5m2_bits(x))


def test_e5m2_saturates():
    x = np.array([61440, 65536, 1e9, np.inf, -61440, -np.inf, 61439.99], dtype=np.float32)
    assert list(quant.e5m2_encode(x)) == [0x7B, 0x7B, 0x7B, 0x7B, 0xFB, 0xFB, 0x7B]


def test_int8_round_half_even_definition():
    rng = np.random.default_rng(12)
    y = np.concatenate([rng.uniform(-130, 130, 100000),
                        np.arange(-1275, 1276) / 10.0,
                        np.arange(-255, 256) / 2.0]).astype(np.float32)
    got = quant.int8_encode(y).astype(np.int64)
    yd = y.astype(np.float64)
    fl = np.floor(yd)
    frac = yd - fl
    rne = np.where(frac > 0.5, fl + 1, np.where(frac < 0.5, fl, np.where(fl % 2 == 0, fl, fl + 1)))
    expect = np.clip(rne, -127, 127).astype(np.int64)
    assert np.array_equal(got, expect)


def test_hand_derived_rows():
    with open(GOLDEN) as f:
        g = json.load(f)
    for kind in ("int8", "e5m2", "int4"):
        for case in g[kind]:
            x = np.array(case["x"], dtype=np.float32)[None, :]
            codes, scale = quant.quantize_rows(x, kind)
            assert scale[0] == np.float32(case["scale"]), case["why"]
            got = codes[0].astype(np.int64)
            assert list(got) == case["codes"], case["why"]
            if kind == "int4":
                assert list(quant.pack_int4(codes)[0]) == case["packed"], case["why"]


def test_quantize_rows_bounds():
    rng = np.random.default_rng(13)
    x = (rng.standard_normal((4096, 128)) * rng.uniform(0.01, 100, (4096, 1))).astype(np.float32)
    for kind in ("int8", "e5m2"):
        codes, scale = quant.quantize_rows(x, kind)
        a = np.abs(x).max(axis=1)
        qmax = 127.0 if kind == "int8" else 57344.0
        assert np.array_equal(scale, (a / np.float32(qmax)).astype(np.float32))
        deq = quant.dequantize(codes, scale, kind)
        err = np.abs(deq - x.astype(np.float64))
        if kind == "int8":
            # half a step, plus the fp32 rounding of x / scale (|y| <= 127)
            assert np.all(err <= scale[:, None].astype(np.float64) * (0.5 + 127 * 2.0 ** -23))
            # the row's largest magnitude maps to +-127
            idx = np.abs(x).argmax(axis=1)
            assert np.all(np.abs(codes[np.arange(4096), idx].astype(int)) == 127)
        else:
            # 2 mantissa bits: relative error <= 2^-3 in the normal range
            y = np.abs(x.astype(np.float64)) / scale[:, None]
            normal = y >= 2.0 ** -14
            rel = err[normal] / np.abs(x.astype(np.float64))[normal]
            assert np.all(rel <= 2.0 ** -3 * (1 + 2.0 ** -20))
            sub = ~normal
            assert np.all(err[sub] <= scale[:, None].repeat(128, 1)[sub] * 2.0 ** -17 * (1 + 2.0 ** -20))


def test_zero_row_and_dequantize_exact():
    x = np.zeros((3, 16), dtype=np.float32)
    x[1, 3] = -2.5
    for kind in ("int8", "e5m2"):
        codes, scale = quant.quantize_rows(x, kind)
        assert scale[0] == 0 and scale[2] == 0 and not codes[0].any() and not codes[2].any()
        deq = quant.dequantize(codes, scale, kind)
        qmax = 127.0 if kind == "int8" else 57344.0
        # the row's absmax maps to -QMAX; its dequantized value is -QMAX * scale
        assert deq[1, 3] == -qmax * float(scale[1])
        assert abs(deq[1, 3] + 2.5) <= 2.5 * 2.0 ** -23


def test_scale_less_e5m2_cast_is_the_plain_encoding():
    """The scale-less FP8 variant stores each value's own E5M2 code: codes of
    exactly representable values decode to themselves, larger values saturate
    to the largest finite code, and the scale is 1."""
    exact = np.array([[1.0, -1.25, 57344.0, 2.0 ** -16, 0.0, -3.0 * 2.0 ** -15, 1.5, -96.0]],
                     dtype=np.float32)
    codes, scales = quant.quantize_rows(exact, "e5m2_cast")
    assert scales.tolist() == [1.0]
    np.testing.assert_array_equal(quant.dequantize(codes, scales, "e5m2_cast"), exact)
    big, _ = quant.quantize_rows(np.array([[1e6, -7e4, 60000.0, 0.1]], np.float32), "e5m2_cast")
    assert big[0, :3].tolist() == [0x7B, 0xFB, 0x7B]
    # 0.1 lies between 0.09375 (0x2E) and 0.109375 (0x2F): 0.00625 above the
    # first, 0.009375 below the second
    assert big[0, 3] == 0x2E


def test_int4_bounds_and_packing():
    rng = np.random.default_rng(14)
    x = (rng.standard_normal((4096, 128)) * rng.uniform(0.01, 100, (4096, 1))).astype(np.float32)
    codes, scale = quant.quantize_rows(x, "int4")
    a = np.abs(x).max(axis=1)
    assert np.array_equal(scale, (a / np.float32(7.0)).astype(np.float32))
    assert codes.min() >= -7 and codes.max() <= 7
    # the row's largest magnitude maps to +-7; everything within half a step
    idx = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(codes[np.arange(4096), idx].astype(int)) == 7)
    err = np.abs(quant.dequantize(codes, scale, "int4") - x.astype(np.float64))
    assert np.all(err <= scale[:, None].astype(np.float64) * (0.5 + 7 * 2.0 ** -23))
    # packing round-trips every code pair, including -8
    allc = np.array([[a, b] for a in range(-8, 8) for b in range(-8, 8)], dtype=np.int8)
    assert np.array_equal(quant.unpack_int4(quant.pack_int4(allc)), allc)
    assert quant.pack_int4(allc).shape == (256, 1) and len(set(quant.pack_int4(allc)[:, 0])) == 256


def test_kchan_hand_rows():
    with open(GOLDEN) as f:
        g = json.load(f)
    for case in g["int8_kchan"]:
        s = np.array(case["scales"], dtype=np.float32)[None, :]      # one kv head
        k = np.array(case["k"], dtype=np.float32)[None, None, :]      # one token
        codes = quant.quantize_k_channels(k, s)
        assert list(codes[0, 0].astype(np.int64)) == case["codes"], case["why"]


def test_kchan_equals_per_token_int8_when_the_scales_agree():
    """With every channel of head h given that head's per-token absmax scale,
    per-channel coding is the per-token INT8 coding of the same row."""
    rng = np.random.default_rng(21)
    k = (rng.standard_normal((1, 8, 128)) * rng.uniform(0.1, 10, (1, 8, 1))).astype(np.float32)
    codes_tok, scale_tok = quant.quantize_rows(k, "int8")
    chan = np.repeat(scale_tok[0][:, None], 128, axis=1)
    codes_ch = quant.quantize_k_channels(k, chan)
    assert np.array_equal(codes_ch, codes_tok)


def test_kchan_error_bound_and_saturation():
    rng = np.random.default_rng(22)
    H, D = 4, 128
    s = rng.uniform(0.001, 0.1, (H, D)).astype(np.float32)
    k = (rng.standard_normal((512, H, D)) * 4.0).astype(np.float32)
    codes = quant.quantize_k_channels(k, s)
    deq = quant.dequantize_k_channels(codes, s)
    sd = s.astype(np.float64)
    kd = k.astype(np.float64)
    inside = np.abs(kd) <= 126.5 * sd
    # round to nearest of an fp32 quotient: within half a step (+ the quotient's rounding)
    assert np.all(np.abs(deq - kd)[inside] <= (0.5 * sd * (1 + 1e-6) + np.abs(kd) * 2.0 ** -23)[inside])
    big = np.abs(kd) >= 127.5 * sd * (1 + 1e-6)
    assert big.any()
    assert np.array_equal(np.abs(codes[big]).astype(np.int64), np.full(big.sum(), 127))
    # integer multiples of a power-of-two scale come back exactly
    s2 = np.full((H, D), 0.125, np.float32)
    m = rng.integers(-127, 128, (64, H, D))
    kk = (m * 0.125).astype(np.float32)
    assert np.array_equal(quant.dequantize_k_channels(quant.quantize_k_channels(kk, s2), s2), kk)


def test_kchan_append_places_codes_and_value_scales():
    from oracle import cache_ops
    rng = np.random.default_rng(23)
    NB, H, bs, D = 5, 2, 16, 64
    kc = np.zeros((NB, H, bs, D), np.int8)
    vc = np.zeros((NB, H, bs, D), np.int8)
    vs = np.zeros((NB, H, bs), np.float32)
    chan = rng.uniform(0.01, 0.05, (H, D)).astype(np.float32)
    k = rng.standard_normal((3, H, D)).astype(np.float32)
    v = rng.standard_normal((3, H, D)).astype(np.float32)
    slots = np.array([2 * bs + 5, -1, 4 * bs + 15])
    cache_ops.append_quantized_kchan(kc, vc, vs, k, v, slots, bs, chan)
    for i, blk, row in ((0, 2, 5), (2, 4, 15)):
        assert np.array_equal(kc[blk, :, row], quant.quantize_k_channels(k[i], chan))
        c, s = quant.quantize_rows(v[i], "int8")
        assert np.array_equal(vc[blk, :, row], c) and np.array_equal(vs[blk, :, row], s)
    assert not kc[[0, 1, 3]].any() and not vc[[0, 1, 3]].any()    # the skipped slot wrote nothing
