"""GPU parity of append, quantize and copy-on-write block copy: bit-exact
against the oracle on the same generated inputs; plus the device status word
and the bounded-wait self-test."""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_support import bits16, raw_bytes, to_np
from oracle import cache_ops, quant

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_440_b200 as p
    return p


@pytest.mark.parametrize("make", [W.tiny, W.gqa70b, W.mha13b])
def test_append_16bit_bit_exact(pkv, make):
    wl = make(DEV)
    pool = pkv.KVPool(1, wl.num_blocks, wl.block_size, wl.kv_heads, wl.head_dim,
                      wl.cache_dtype, DEV)
    K, V, _, _ = pool.layer_views(0)
    K.copy_(wl.k_fill)
    V.copy_(wl.v_fill)
    slots = wl.slot_new.copy()
    slots[1] = -1                                     # padding token: skipped
    pkv.kv_append(pool, 0, wl.k_new, wl.v_new, torch.from_numpy(slots).to(DEV))
    torch.cuda.synchronize()
    assert pool.status() == 0
    kb, vb = bits16(wl.k_fill), bits16(wl.v_fill)
    cache_ops.append(kb, vb, bits16(wl.k_new), bits16(wl.v_new), slots, wl.block_size)
    touched = np.unique(np.maximum(slots, 0) // wl.block_size)
    if kb.size > 300_000_000:                          # large pool: touched + sampled blocks
        rng = np.random.default_rng(0)
        blocks = np.unique(np.concatenate([touched, rng.choice(wl.num_blocks, 256)]))
        idx = torch.from_numpy(blocks).to(DEV)
        assert np.array_equal(bits16(K[idx]), kb[blocks])
        assert np.array_equal(bits16(V[idx]), vb[blocks])
    else:
        assert np.array_equal(bits16(K), kb)
        assert np.array_equal(bits16(V), vb)


def test_append_out_of_range_slot_is_reported_not_written(pkv):
    pool = pkv.KVPool(1, 8, 16, 2, 64, "bf16", DEV)
    K, V, _, _ = pool.layer_views(0)
    K.zero_()
    V.zero_()
    x = torch.randn(2, 2, 64, device=DEV).to(torch.bfloat16)
    pkv.kv_append(pool, 0, x, x, torch.tensor([3, 8 * 16 + 5], dtype=torch.int64, device=DEV))
    torch.cuda.synchronize()
    assert pool.status() & 4
    assert torch.equal(K[0, :, 3], x[0]) and int((K != 0).sum()) == 2 * 64


def _special_rows(D):
    rows = [np.zeros(D), np.full(D, 1e-30), np.full(D, -3.0), np.linspace(-1, 1, D)]
    r = np.zeros(D)
    r[5] = 1e4
    r[6] = -2.0 ** -20
    rows.append(r)
    r = np.zeros(D)
    r[0] = 57344.0
    r[1:] = np.linspace(-1e-3, 1e-3, D - 1)           # E5M2 subnormal codes
    rows.append(r)
    return np.stack(rows)


@pytest.mark.parametrize("kind", ["int8", "e5m2", "int4"])
@pytest.mark.parametrize("in_dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [64, 128])
def test_quantize_bit_exact(pkv, kind, in_dt, D):
    if kind == "int4" and D != 128:
        pytest.skip("INT4 rows need head_dim 128")
    g = torch.Generator(device=DEV).manual_seed(D)
    x = torch.randn(20000, D, generator=g, device=DEV)
    x = x * torch.exp(torch.randn(20000, 1, generator=g, device=DEV) * 3)   # wide dynamic range
    x = x.clamp(-6e4, 6e4)                                                  # finite in fp16
    x = torch.cat([x, torch.from_numpy(_special_rows(D)).float().to(DEV)]).to(in_dt)
    assert torch.isfinite(x.float()).all()
    codes, scales = pkv.kv_quantize(x, kind)
    torch.cuda.synchronize()
    ref_codes, ref_scales = quant.quantize_rows(to_np(x), kind)
    if kind == "int4":
        ref_codes = quant.pack_int4(ref_codes)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), ref_codes)


@pytest.mark.parametrize("cache", ["bf16", "int8", "e5m2", "e5m2_cast", "int4", "int8_kchan"])
def test_block_copy_bit_exact(pkv, cache):
    """Shared-prefix shapes: 200 copy-on-write pairs, 3 layers, random pool bytes.
    Per-channel key scales belong to the layer, not to a block: left as they are."""
    layers, NB, bs, hkv, D = 3, 1500, 16, 8, 128
    pool = pkv.KVPool(layers, NB, bs, hkv, D, cache, DEV)
    g = torch.Generator(device=DEV).manual_seed(7)
    pool.buffer.copy_(torch.randint(0, 256, pool.buffer.shape, generator=g, device=DEV,
                                    dtype=torch.uint8))
    before = [[raw_bytes(t) if t is not None else None for t in pool.layer_views(l)]
              for l in range(layers)]
    rng = np.random.default_rng(3)
    ids = rng.permutation(NB)[:400]
    pairs = list(zip(ids[:200].tolist(), ids[200:].tolist()))
    pkv.kv_block_copy(pool, pairs)
    torch.cuda.synchronize()
    per_block = [i for i in range(4) if not (cache == "int8_kchan" and i == 2)]
    regions = [lay[i] for lay in before for i in per_block if lay[i] is not None]
    cache_ops.block_copy(regions, pairs)
    views = [pool.layer_views(l) for l in range(layers)]
    after = [raw_bytes(v[i]) for v in views for i in per_block if v[i] is not None]
    for a, r in zip(after, regions):
        assert np.array_equal(a, r)
    if cache == "int8_kchan":
        for l in range(layers):
            assert np.array_equal(raw_bytes(views[l][2]), before[l][2])


def test_bounded_wait_gives_up_and_reports(pkv):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.selftest_wait_timeout(st, limit_us=2000)
    torch.cuda.synchronize()
    assert int(st.item()) & 8
    # the context is still usable afterwards
    y = torch.ones(4, device=DEV) * 2
    assert float(y.sum()) == 8.0


@pytest.mark.parametrize("in_dt", [torch.bfloat16, torch.float16])
def test_append_scale_less_e5m2_bit_exact(pkv, in_dt):
    """FP8 storage without a scale: each value's own E5M2 code (saturating RNE)
    lands in its slot, and the pool has no scale regions."""
    NB, bs, hkv, D, T = 64, 16, 4, 128, 300
    pool = pkv.KVPool(1, NB, bs, hkv, D, "e5m2_cast", DEV)
    K, V, KS, VS = pool.layer_views(0)
    assert KS is None and VS is None
    K.zero_()
    V.zero_()
    g = torch.Generator(device=DEV).manual_seed(5)
    k = (torch.randn(T, hkv, D, generator=g, device=DEV) * 30).clamp(-6e4, 6e4).to(in_dt)
    v = (torch.randn(T, hkv, D, generator=g, device=DEV) * 1e-3).to(in_dt)
    slots = torch.randperm(NB * bs, generator=torch.Generator().manual_seed(6))[:T].to(DEV)
    pkv.kv_append(pool, 0, k, v, slots)
    torch.cuda.synchronize()
    kc = np.zeros((NB, hkv, bs, D), np.uint8)
    vc = np.zeros_like(kc)
    ks = np.zeros((NB, hkv, bs), np.float32)
    vs = np.zeros_like(ks)
    cache_ops.append_quantized(kc, vc, ks, vs, to_np(k), to_np(v), slots.cpu().numpy(), bs,
                               "e5m2_cast")
    assert np.array_equal(K.cpu().numpy(), kc)
    assert np.array_equal(V.cpu().numpy(), vc)


@pytest.mark.parametrize("in_dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D,bs", [(64, 16), (128, 32)])
def test_append_kchan_bit_exact(pkv, in_dt, D, bs):
    """INT8 keys with the layer's channel scales (one zero-scale channel, some
    scales small enough to saturate), INT8 values per row: codes and value
    scales bit-exact with the oracle; the channel scales stay as written."""
    NB, hkv, T = 40, 4, 300
    pool = pkv.KVPool(1, NB, bs, hkv, D, "int8_kchan", DEV)
    K, V, KS, VS = pool.layer_views(0)
    for t in (K, V, VS):
        t.zero_()
    rng = np.random.default_rng(D + bs)
    sigma = rng.uniform(0.25, 4.0, (hkv, D)).astype(np.float32)
    chan = (sigma * 4.0 / 127.0).astype(np.float32)
    chan[1, 3] = 0.0                                    # a dropped channel
    chan[2, :8] = np.float32(1e-4)                      # saturates
    KS.copy_(torch.from_numpy(chan).to(DEV))
    g = torch.Generator(device=DEV).manual_seed(D * bs)
    k = (torch.randn(T, hkv, D, generator=g, device=DEV) * torch.from_numpy(sigma).to(DEV)).to(in_dt)
    v = (torch.randn(T, hkv, D, generator=g, device=DEV) * 3).to(in_dt)
    slots = rng.permutation(NB * bs)[:T].astype(np.int64)
    slots[7] = -1                                       # padding token: skipped
    pkv.kv_append(pool, 0, k, v, torch.from_numpy(slots).to(DEV))
    torch.cuda.synchronize()
    assert pool.status() == 0
    kc = np.zeros((NB, hkv, bs, D), np.int8)
    vc = np.zeros((NB, hkv, bs, D), np.int8)
    vs = np.zeros((NB, hkv, bs), np.float32)
    cache_ops.append_quantized_kchan(kc, vc, vs, to_np(k), to_np(v), slots, bs, chan)
    assert np.array_equal(K.cpu().numpy(), kc)
    assert np.array_equal(V.cpu().numpy(), vc)
    assert np.array_equal(VS.cpu().numpy().view(np.uint32), vs.view(np.uint32))
    assert np.array_equal(KS.cpu().numpy(), chan)
    assert (np.abs(kc[..., 2, :, :8]) == 127).any()     # the saturating channels did saturate
