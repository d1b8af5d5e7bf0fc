"""Host-side checks of the C ABI (no GPU): the library loads and exports every
symbol the header declares; pool layout against the KV-bytes formula; the
refcounted allocator against the reference model; argument validation."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import allocator as ref_alloc
from oracle import pool as ref_pool
from paged_kv_cache_440_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedkv.h")
FAKE_BASE = 1 << 40          # never dereferenced by host-only calls


def _declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:kv_status|const char \*)\s*(\w+)\s*\(", txt, re.M)))


def test_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(B.lib, n), n
    assert B.version().startswith("pagedkv")


def _make_pool(NB=64, layers=2, bs=16, hkv=2, D=64, dt="bf16"):
    d = B.PoolDesc(layers, NB, bs, hkv, D, B.DTYPE_CODES[dt])
    n = ctypes.c_uint64()
    B.check(B.lib.kv_pool_required_bytes(ctypes.byref(d), ctypes.byref(n)))
    h = ctypes.c_void_p()
    B.check(B.lib.kv_pool_create(ctypes.byref(d), ctypes.c_void_p(FAKE_BASE), n.value,
                                 ctypes.byref(h)))
    return h, n.value


def _ptrs(h, layer):
    k, v, ks, vs = (ctypes.c_void_p() for _ in range(4))
    B.check(B.lib.kv_pool_layer_ptrs(h, layer, ctypes.byref(k), ctypes.byref(v),
                                     ctypes.byref(ks), ctypes.byref(vs)))
    return k.value, v.value, ks.value, vs.value


@pytest.mark.parametrize("dt,elt", [("bf16", 2), ("fp16", 2), ("int8", 1), ("e5m2", 1),
                                    ("e5m2_cast", 1)])
@pytest.mark.parametrize("layers,NB,bs,hkv,D", [(80, 37, 16, 8, 128), (1, 5, 32, 3, 64)])
def test_layout_matches_kv_formula(dt, elt, layers, NB, bs, hkv, D):
    h, total = _make_pool(NB, layers, bs, hkv, D, dt)
    try:
        tokens = NB * bs
        kv = ref_pool.kv_cache_bytes(1, hkv, D, elt, tokens)       # one layer, K and V
        prev_end = FAKE_BASE
        for layer in range(layers):
            k, v, ks, vs = _ptrs(h, layer)
            assert k % 256 == 0 and v % 256 == 0 and k >= prev_end
            assert v - k >= kv // 2                        # K region holds half the formula
            if dt in ("int8", "e5m2"):
                sb = ref_pool.scale_bytes(1, hkv, 4, tokens)
                assert ks - v >= kv // 2 and vs - ks >= sb // 2
                prev_end = vs + sb // 2
            else:
                assert ks is None and vs is None
                prev_end = v + kv // 2
        # padding between regions is below 256 bytes each, plus a 256-byte status region
        scales = ref_pool.scale_bytes(layers, hkv, 4, tokens) if dt in ("int8", "e5m2") else 0
        exact = ref_pool.kv_cache_bytes(layers, hkv, D, elt, tokens) + scales
        assert exact + 256 <= total <= exact + 256 + layers * 4 * 255
    finally:
        B.lib.kv_pool_destroy(h)


def test_pool_rejects_bad_descriptions():
    n = ctypes.c_uint64()
    for desc, code in [((1, 8, 8, 1, 64, 0), B.KV_ERR_UNSUPPORTED),
                       ((1, 8, 16, 1, 96, 0), B.KV_ERR_UNSUPPORTED),
                       ((1, 8, 16, 1, 64, 7), B.KV_ERR_UNSUPPORTED),
                       ((0, 8, 16, 1, 64, 0), B.KV_ERR_INVALID),
                       ((1, -1, 16, 1, 64, 0), B.KV_ERR_INVALID)]:
        d = B.PoolDesc(*desc)
        assert B.lib.kv_pool_required_bytes(ctypes.byref(d), ctypes.byref(n)) == code
        assert B.lib.kv_last_error()
    d = B.PoolDesc(1, 8, 16, 1, 64, 0)
    B.check(B.lib.kv_pool_required_bytes(ctypes.byref(d), ctypes.byref(n)))
    h = ctypes.c_void_p()
    assert B.lib.kv_pool_create(ctypes.byref(d), ctypes.c_void_p(FAKE_BASE + 16), n.value,
                                ctypes.byref(h)) == B.KV_ERR_INVALID          # misaligned
    assert B.lib.kv_pool_create(ctypes.byref(d), ctypes.c_void_p(FAKE_BASE), n.value - 1,
                                ctypes.byref(h)) == B.KV_ERR_INVALID          # too small


def _arr(ids):
    return (ctypes.c_int32 * max(len(ids), 1))(*ids)


def _stats(h):
    u, f, s = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    B.check(B.lib.kv_pool_stats(h, ctypes.byref(u), ctypes.byref(f), ctypes.byref(s)))
    return u.value, f.value, s.value


def test_allocator_random_ops_match_model():
    rng = np.random.default_rng(0)
    NB = 40
    h, _ = _make_pool(NB)
    model = ref_alloc.PoolModel(NB)
    held = []                     # references we own (one entry per reference)
    try:
        for step in range(3000):
            op = rng.integers(0, 4)
            if op == 0:
                n = int(rng.integers(0, 6))
                out = (ctypes.c_int32 * max(n, 1))()
                st = B.lib.kv_alloc_blocks(h, n, out)
                if model.free_count() < n:
                    assert st == B.KV_ERR_OOM
                else:
                    assert st == B.KV_OK
                    ids = list(out[:n])
                    assert len(set(ids)) == n
                    model.take(ids)
                    held += ids
            elif op == 1 and held:
                k = int(rng.integers(1, min(4, len(held)) + 1))
                pick = [held.pop(int(rng.integers(0, len(held)))) for _ in range(k)]
                B.check(B.lib.kv_free_blocks(h, len(pick), _arr(pick)))
                model.free(pick)
            elif op == 2 and held:
                i = held[int(rng.integers(0, len(held)))]
                B.check(B.lib.kv_share_blocks(h, 1, _arr([i])))
                model.share([i])
                held.append(i)
            elif op == 3 and held:
                i = held[int(rng.integers(0, len(held)))]
                new = ctypes.c_int32()
                st = B.lib.kv_cow_prepare(h, i, ctypes.byref(new))
                if not model.cow_needed(i):
                    assert st == B.KV_OK and new.value == i
                elif model.free_count() == 0:
                    assert st == B.KV_ERR_OOM
                else:
                    assert st == B.KV_OK and new.value != i
                    model.free([i])
                    model.take([new.value])
                    held.remove(i)
                    held.append(new.value)
            u, f, s = _stats(h)
            assert (u, f, s) == (model.used_count(), model.free_count(), model.shared_count())
            for i in range(NB):
                r = ctypes.c_int32()
                B.check(B.lib.kv_block_refcount(h, i, ctypes.byref(r)))
                assert r.value == model.ref[i]
    finally:
        B.lib.kv_pool_destroy(h)


def test_allocator_errors_change_nothing():
    h, _ = _make_pool(8)
    try:
        out = (ctypes.c_int32 * 8)()
        B.check(B.lib.kv_alloc_blocks(h, 3, out))
        ids = list(out[:3])
        before = _stats(h)
        assert B.lib.kv_alloc_blocks(h, 6, out) == B.KV_ERR_OOM
        assert B.lib.kv_free_blocks(h, 2, _arr([ids[0], 7])) == B.KV_ERR_INVALID   # 7 is free
        assert B.lib.kv_free_blocks(h, 2, _arr([ids[0], ids[0]])) == B.KV_ERR_INVALID
        assert B.lib.kv_share_blocks(h, 1, _arr([9])) == B.KV_ERR_INVALID
        assert B.lib.kv_alloc_blocks(h, -1, out) == B.KV_ERR_INVALID
        assert _stats(h) == before
    finally:
        B.lib.kv_pool_destroy(h)


def test_block_copy_validation_rejects_bad_pairs_before_launch():
    h, _ = _make_pool(16)
    try:
        bad = [[(3, 3)], [(1, 2), (4, 2)], [(1, 2), (2, 5)], [(0, 16)], [(-1, 3)]]
        for pairs in bad:
            flat = [v for p in pairs for v in p]
            assert B.lib.kv_block_copy(h, _arr(flat), len(pairs), None) == B.KV_ERR_INVALID
        assert B.lib.kv_block_copy(h, _arr([]), 0, None) == B.KV_OK
    finally:
        B.lib.kv_pool_destroy(h)


def test_attention_argument_validation_and_workspace_size():
    h, _ = _make_pool(64, 1, 16, 2, 64, "bf16")
    try:
        n = ctypes.c_uint64()
        # Hq must be a multiple of Hkv
        assert B.lib.paged_attn_workspace_bytes(h, 4, 3, 10, ctypes.byref(n)) == B.KV_ERR_INVALID
        assert B.lib.paged_attn_workspace_bytes(h, 4, 8, -1, ctypes.byref(n)) == B.KV_ERR_INVALID
        # 16 B per unit (here one unit per sequence: both kv heads in one group)
        # plus 10 CTAs x 2 sides x 8 slots x 8 heads x (64 + 2) fp32, 256-aligned parts
        B.check(B.lib.paged_attn_workspace_bytes(h, 4, 8, 10, ctypes.byref(n)))
        r256 = lambda x: -(-x // 256) * 256
        recs = 10 * 2 * 8 * 8
        want = r256(4 * 1 * 16) + r256(recs * 2 * 4) + r256(recs * 64 * 4)
        assert n.value == want
        # 16 query heads per kv head (two 8-head chunks): still one unit per sequence
        B.check(B.lib.paged_attn_workspace_bytes(h, 4, 32, 10, ctypes.byref(n)))
        assert n.value == want
        # validation failures return before any device work
        nul = ctypes.c_void_p(0)
        fake = ctypes.c_void_p(FAKE_BASE)
        big = 1 << 20
        args = lambda q, qdt, hq, mb, mc, sc: (h, 0, q, qdt, 4, hq, fake, mb, fake, mc, sc, fake,
                                               10, fake, big, None)
        assert B.lib.paged_attn_decode(*args(nul, 0, 8, 16, 250, 0.125)) == B.KV_ERR_INVALID
        assert B.lib.paged_attn_decode(*args(fake, 1, 8, 16, 250, 0.125)) == B.KV_ERR_UNSUPPORTED
        assert B.lib.paged_attn_decode(*args(fake, 0, 5, 16, 250, 0.125)) == B.KV_ERR_INVALID
        assert B.lib.paged_attn_decode(*args(fake, 0, 8, 0, 250, 0.125)) == B.KV_ERR_INVALID
        assert B.lib.paged_attn_decode(*args(fake, 0, 8, 16, 250, float("nan"))) == B.KV_ERR_INVALID
        assert B.lib.paged_attn_decode(*args(fake, 0, 8, 16, -1, 0.125)) == B.KV_ERR_INVALID
        # too small a workspace
        st = B.lib.paged_attn_decode(h, 0, fake, 0, 4, 8, fake, 16, fake, 250, 0.125, fake, 10,
                                     fake, 16, None)
        assert st == B.KV_ERR_INVALID
        # append / quantize validation
        assert B.lib.kv_append(h, 1, fake, fake, 0, fake, 1, None) == B.KV_ERR_INVALID   # layer
        assert B.lib.kv_append(h, 0, fake, fake, 1, fake, 1, None) == B.KV_ERR_UNSUPPORTED
        assert B.lib.kv_append(h, 0, fake, fake, 0, fake, -1, None) == B.KV_ERR_INVALID
        assert B.lib.kv_append(h, 0, fake, fake, 0, fake, 0, None) == B.KV_OK
        assert B.lib.kv_quantize(fake, 0, 4, 96, 3, fake, fake, None) == B.KV_ERR_UNSUPPORTED
        assert B.lib.kv_quantize(fake, 0, 4, 64, 0, fake, fake, None) == B.KV_ERR_UNSUPPORTED
        assert B.lib.kv_quantize(fake, 0, 0, 64, 3, fake, fake, None) == B.KV_OK
    finally:
        B.lib.kv_pool_destroy(h)


def test_valid_call_without_a_gpu_fails_loudly():
    """On a host with no GPU a well-formed launch reports KV_ERR_CUDA; nothing
    falls back to a CPU path."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h, _ = _make_pool(64, 1, 16, 2, 64, "bf16")
    try:
        fake = ctypes.c_void_p(FAKE_BASE)
        st = B.lib.paged_attn_decode(h, 0, fake, 0, 4, 8, fake, 16, fake, 250, 0.125, fake, 10,
                                     fake, 1 << 20, None)
        assert st == B.KV_ERR_CUDA
        n = ctypes.c_uint64()
        assert B.lib.paged_attn_workspace_bytes(h, 4, 8, 0, ctypes.byref(n)) == B.KV_ERR_CUDA
    finally:
        B.lib.kv_pool_destroy(h)


def test_int4_layout_and_head_dim():
    """INT4 rows are head_dim / 2 bytes (two codes per byte) with fp32 scales;
    head_dim 64 is rejected."""
    NB, layers, bs, hkv, D = 37, 2, 16, 8, 128
    h, total = _make_pool(NB, layers, bs, hkv, D, "int4")
    try:
        tokens = NB * bs
        kv = ref_pool.kv_cache_bytes(1, hkv, D, 0.5, tokens)      # K and V, half a byte per value
        k, v, ks, vs = _ptrs(h, 0)
        assert v - k >= kv // 2 and ks - v >= kv // 2 and vs is not None
        exact = ref_pool.kv_cache_bytes(layers, hkv, D, 0.5, tokens) + \
            ref_pool.scale_bytes(layers, hkv, 4, tokens)
        assert exact + 256 <= total <= exact + 256 + layers * 4 * 255
    finally:
        B.lib.kv_pool_destroy(h)
    d = B.PoolDesc(1, 8, 16, 2, 64, B.DTYPE_CODES["int4"])
    n = ctypes.c_uint64()
    assert B.lib.kv_pool_required_bytes(ctypes.byref(d), ctypes.byref(n)) == B.KV_ERR_UNSUPPORTED


def test_kchan_layout_channel_scales_per_layer():
    """INT8 keys with channel scales: 1-byte K and V rows, a [kv_heads][head_dim]
    fp32 K-scale array per layer and per-token-head V scales."""
    NB, layers, bs, hkv, D = 37, 2, 16, 8, 128
    h, total = _make_pool(NB, layers, bs, hkv, D, "int8_kchan")
    try:
        tokens = NB * bs
        kv = ref_pool.kv_cache_bytes(1, hkv, D, 1, tokens)
        k, v, ks, vs = _ptrs(h, 0)
        k1, _, _, _ = _ptrs(h, 1)
        assert v - k >= kv // 2 and ks - v >= kv // 2
        assert vs - ks == -(-hkv * D * 4 // 256) * 256          # channel scales, 256-aligned
        assert k1 - vs >= tokens * hkv * 4                       # then per-token V scales
        exact = ref_pool.kv_cache_bytes(layers, hkv, D, 1, tokens) + \
            layers * (hkv * D * 4 + tokens * hkv * 4)
        assert exact + 256 <= total <= exact + 256 + layers * 4 * 255
    finally:
        B.lib.kv_pool_destroy(h)


def test_prefill_argument_validation():
    """paged_attn_prefill rejects bad arguments before any device work; on a
    host without a GPU a well-formed call fails loudly (KV_ERR_CUDA)."""
    import torch
    h, _ = _make_pool(64, 1, 16, 2, 64, "bf16")
    hq, _ = _make_pool(64, 1, 16, 2, 64, "int8_kchan")
    try:
        fake = ctypes.c_void_p(FAKE_BASE)
        nul = ctypes.c_void_p(0)

        def call(pool=h, layer=0, q=fake, qdt=0, B_=2, Hq=8, total=10, maxq=5, mb=16, mc=64,
                 scale=0.125, out=fake, cu=fake, tab=fake, lens=fake):
            return B.lib.paged_attn_prefill(pool, layer, q, qdt, B_, Hq, cu, total, maxq, tab, mb,
                                            lens, mc, scale, out, None)

        assert call(layer=1) == B.KV_ERR_INVALID                     # layer out of range
        assert call(pool=hq) == B.KV_ERR_UNSUPPORTED                 # 1-byte caches
        assert call(qdt=1) == B.KV_ERR_UNSUPPORTED                   # q dtype != cache dtype
        assert call(Hq=7) == B.KV_ERR_INVALID                        # not a multiple of Hkv
        assert call(Hq=2 * 129) == B.KV_ERR_UNSUPPORTED              # > 128 heads per kv head
        assert call(total=-1) == B.KV_ERR_INVALID
        assert call(mb=0) == B.KV_ERR_INVALID
        assert call(scale=float("inf")) == B.KV_ERR_INVALID
        assert call(B_=0) == B.KV_OK                                 # nothing to do
        assert call(q=nul) == B.KV_ERR_INVALID
        assert call(q=ctypes.c_void_p(FAKE_BASE + 8)) == B.KV_ERR_INVALID   # misaligned
        assert call(B_=65536) == B.KV_ERR_UNSUPPORTED
        if not torch.cuda.is_available():
            assert call() == B.KV_ERR_CUDA
        # the per-channel key kind has no standalone per-row quantizer
        assert B.lib.kv_quantize(fake, 0, 4, 64, B.KV_INT8_KCHAN, fake, fake, None) == \
            B.KV_ERR_UNSUPPORTED
    finally:
        B.lib.kv_pool_destroy(h)
        B.lib.kv_pool_destroy(hq)


def test_cascade_argument_validation_and_workspace_size():
    """paged_attn_decode_cascade checks its arguments before any launch (the
    prefix pass included); its workspace is the decode workspace plus the
    prefix partials; on a host without a GPU a well-formed call fails loudly."""
    import torch
    h, _ = _make_pool(64, 1, 16, 2, 64, "bf16")
    hq, _ = _make_pool(64, 1, 16, 2, 64, "int8")
    try:
        r256 = lambda x: -(-x // 256) * 256
        n, nd = ctypes.c_uint64(), ctypes.c_uint64()
        B.check(B.lib.paged_attn_cascade_workspace_bytes(h, 4, 8, 10, ctypes.byref(n)))
        B.check(B.lib.paged_attn_workspace_bytes(h, 4, 8, 10, ctypes.byref(nd)))
        assert n.value == r256(nd.value) + r256(4 * 8 * 64 * 4) + r256(4 * 8 * 2 * 4)
        fake = ctypes.c_void_p(FAKE_BASE)
        nul = ctypes.c_void_p(0)

        def call(pool=h, layer=0, q=fake, kn=None, vn=None, qdt=0, B_=4, Hq=8, mb=16, mc=250,
                 pb=4, scale=0.125, out=fake, ctas=10, ws=fake, wsb=1 << 22):
            return B.lib.paged_attn_decode_cascade(pool, layer, q, kn, vn, qdt, B_, Hq, fake, mb,
                                                   fake, mc, pb, scale, out, ctas, ws, wsb, None)

        assert call(layer=1) == B.KV_ERR_INVALID
        assert call(pool=hq) == B.KV_ERR_UNSUPPORTED                 # 16-bit caches only
        assert call(qdt=1) == B.KV_ERR_UNSUPPORTED                   # q dtype != cache dtype
        assert call(pb=0) == B.KV_ERR_INVALID                        # no prefix
        assert call(pb=16) == B.KV_ERR_INVALID                       # no block past the prefix
        assert call(mc=63) == B.KV_ERR_INVALID                       # prefix longer than max
        assert call(Hq=7) == B.KV_ERR_INVALID
        assert call(Hq=2 * 129) == B.KV_ERR_UNSUPPORTED              # > 128 heads per kv head
        assert call(kn=fake) == B.KV_ERR_INVALID                     # k_new without v_new
        assert call(kn=fake, vn=fake, Hq=32) == B.KV_ERR_UNSUPPORTED  # append: <= 8 per kv head
        assert call(wsb=16) == B.KV_ERR_INVALID                      # workspace too small
        assert call(ws=ctypes.c_void_p(FAKE_BASE + 128)) == B.KV_ERR_INVALID   # misaligned
        assert call(q=nul) == B.KV_ERR_INVALID
        assert call(B_=0) == B.KV_OK                                 # nothing to do
        if not torch.cuda.is_available():
            assert call() == B.KV_ERR_CUDA
            assert call(kn=fake, vn=fake) == B.KV_ERR_CUDA
    finally:
        B.lib.kv_pool_destroy(h)
        B.lib.kv_pool_destroy(hq)
