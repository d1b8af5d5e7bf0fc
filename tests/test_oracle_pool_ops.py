"""Pins for the KV-bytes formula, block arithmetic, append, block copy and the
pool model.

* the formula against the worked numbers the pages print
  (tests/golden/kv_formula_pages.json);
* internal waste below one block (at most 15 tokens for 16-token blocks);
* append and copy checked at explicit flat byte offsets, computed here from the
  [block][kv_head][row][dim] layout, not through the oracle;
* copy-on-write leaves every other sharer's logical sequence unchanged;
* the scale-bytes product against a count of the scales the oracle's append
  writes.
"""
import json
import os

import numpy as np
import pytest

from oracle import allocator, cache_ops, pool, quant

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_formula_pages.json")


def test_formula_matches_pages_worked_numbers():
    with open(GOLDEN) as f:
        g = json.load(f)
    for c in g["cases"]:
        got = pool.kv_cache_bytes(c["layers"], c["kv_heads"], c["head_dim"],
                                  c["dtype_bytes"], c["seq_len"])
        if "bytes" in c:
            assert got == c["bytes"], c["cite"]
        else:
            assert round(got / c["unit_bytes"], c["decimals"]) == c["approx"], c["cite"]


def test_waste_below_one_block():
    with open(GOLDEN) as f:
        w = json.load(f)["waste"]
    worst = max(pool.internal_waste_tokens(L, w["block_size"]) for L in range(1, 5000))
    assert worst == w["max_waste_tokens"]
    rng = np.random.default_rng(0)
    for bs in (8, 16, 32):
        for L in rng.integers(1, 100000, 1000):
            wst = pool.internal_waste_tokens(L, bs)
            assert 0 <= wst <= bs - 1
            assert pool.blocks_for(L, bs) * bs >= L


def test_append_writes_at_flat_offsets():
    rng = np.random.default_rng(1)
    NB, Hkv, bs, D = 10, 3, 4, 5
    kc = rng.integers(0, 65535, (NB, Hkv, bs, D)).astype(np.uint16)
    vc = rng.integers(0, 65535, (NB, Hkv, bs, D)).astype(np.uint16)
    k0, v0 = kc.copy(), vc.copy()
    T = 6
    kn = rng.integers(0, 65535, (T, Hkv, D)).astype(np.uint16)
    vn = rng.integers(0, 65535, (T, Hkv, D)).astype(np.uint16)
    slots = np.array([7, -1, 39, 0, 22, 7], dtype=np.int64)     # 7 repeats: last wins
    cache_ops.append(kc, vc, kn, vn, slots, bs)
    kflat, vflat = k0.reshape(-1).copy(), v0.reshape(-1).copy()
    for i, s in enumerate(slots):
        if s < 0:
            continue
        blk, row = s // bs, s % bs
        for h in range(Hkv):
            off = ((blk * Hkv + h) * bs + row) * D
            kflat[off:off + D] = kn[i, h]
            vflat[off:off + D] = vn[i, h]
    assert np.array_equal(kc.reshape(-1), kflat)
    assert np.array_equal(vc.reshape(-1), vflat)
    assert np.array_equal(kc[1, :, 3], kn[5])


def test_append_quantized_places_codes_and_scales():
    rng = np.random.default_rng(2)
    NB, Hkv, bs, D = 4, 2, 8, 16
    kc = np.zeros((NB, Hkv, bs, D), np.int8)
    vc = np.zeros((NB, Hkv, bs, D), np.int8)
    ks = np.zeros((NB, Hkv, bs), np.float32)
    vs = np.zeros((NB, Hkv, bs), np.float32)
    kn = rng.standard_normal((3, Hkv, D)).astype(np.float32)
    vn = rng.standard_normal((3, Hkv, D)).astype(np.float32)
    slots = np.array([9, 31, 0])
    cache_ops.append_quantized(kc, vc, ks, vs, kn, vn, slots, bs, "int8")
    codes, sc = quant.quantize_rows(kn, "int8")
    assert np.array_equal(kc[1, :, 1], codes[0]) and np.array_equal(ks[3, :, 7], sc[1])
    assert np.array_equal(kc[0, :, 0], codes[2])


def test_scale_bytes_counts_the_scales_append_writes():
    """scale_bytes against a brute-force count: append T tokens of a quantized
    cache in each of 3 layers through the oracle's own append and count the
    fp32 scale entries it writes (K and V, every head), 4 bytes each."""
    rng = np.random.default_rng(4)
    layers, NB, Hkv, bs, D, T = 3, 6, 2, 8, 16, 29
    written = 0
    for _ in range(layers):
        kc = np.zeros((NB, Hkv, bs, D), np.int8)
        vc = np.zeros((NB, Hkv, bs, D), np.int8)
        ks = np.full((NB, Hkv, bs), np.nan, np.float32)
        vs = np.full((NB, Hkv, bs), np.nan, np.float32)
        kn = rng.standard_normal((T, Hkv, D)).astype(np.float32)
        vn = rng.standard_normal((T, Hkv, D)).astype(np.float32)
        slots = rng.permutation(NB * bs)[:T]
        cache_ops.append_quantized(kc, vc, ks, vs, kn, vn, slots, bs, "int8")
        written += int(np.count_nonzero(~np.isnan(ks)) + np.count_nonzero(~np.isnan(vs)))
    assert written * 4 == pool.scale_bytes(layers, Hkv, 4, T)


def test_block_copy_and_cow_keeps_sharers_intact():
    rng = np.random.default_rng(3)
    NB, Hkv, bs, D = 8, 2, 4, 3
    layers = [rng.integers(0, 255, (NB, Hkv, bs, D)).astype(np.uint8) for _ in range(4)]
    before = [a.copy() for a in layers]
    # two sequences share blocks 2 (full) and 5 (partial, 2 rows used)
    tables = {"A": [2, 5], "B": [2, 5]}
    # B diverges: copy block 5 to fresh block 7, repoint, then write row 2
    cache_ops.block_copy(layers, [(5, 7)])
    tables["B"] = [2, 7]
    for a in layers:
        a[7, :, 2] = 0xEE
    for a, b0 in zip(layers, before):
        assert np.array_equal(a[:7], b0[:7])                 # A's blocks untouched
        assert np.array_equal(a[7, :, :2], b0[5, :, :2])     # B's copy holds the prefix
    for a, b0 in zip(layers, before):
        seq_a = np.concatenate([a[i, :, :] for i in tables["A"]], axis=1)
        seq_a0 = np.concatenate([b0[i, :, :] for i in tables["A"]], axis=1)
        assert np.array_equal(seq_a, seq_a0)


def test_pool_model():
    m = allocator.PoolModel(5)
    ids = m.alloc(3)
    assert ids == [0, 1, 2] and m.used_count() == 3
    assert m.alloc(3) is None and m.used_count() == 3
    m.share([1])
    assert m.shared_count() == 1 and m.cow_needed(1) and not m.cow_needed(0)
    m.free([1])
    assert not m.cow_needed(1)
    with pytest.raises(ValueError):
        m.free([4])
    m.free([0, 1, 2])
    assert m.free_count() == 5
