"""Chunked prefill on the GPU against the oracle (every output row)."""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_support import bits16, build_pool, compare, device_inputs, oracle_cache_16, to_np
from oracle import attention

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_440_b200 as m
    return m


def _cache_16(wl):
    dt = np.float16 if wl.cache_dtype == "fp16" else np.float32
    return to_np(wl.k_fill, dt), to_np(wl.v_fill, dt)


def _run(pkv, pw):
    wl = pw.cache
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    cu = torch.from_numpy(pw.cu_q).to(DEV)
    out = pkv.paged_attn_prefill(pool, 0, pw.q, cu, int(max(pw.chunk_lens.max(), 1)), tables,
                                 lens, int(max(wl.context_lens.max(), 1)), wl.scale)
    torch.cuda.synchronize()
    return pool, out


CASES = [
    # name, Hq, Hkv, D, bs, dtype, lens, chunks
    ("gqa-g8-d128-bs16", 16, 2, 128, 16, "bf16", [37, 300, 129, 64, 5], [37, 100, 1, 64, 2]),
    ("mha-fp16-d64-bs32", 4, 4, 64, 32, "fp16", [50, 200, 33], [50, 17, 33]),
    ("g8-d128-bs32-long", 8, 1, 128, 32, "bf16", [1000, 65], [300, 65]),
    ("g16-d64-bs16", 32, 2, 64, 16, "bf16", [90, 17], [41, 17]),
    ("g3-d128-bs16", 6, 2, 128, 16, "fp16", [70, 140], [70, 60]),
    ("g64-d128-bs16", 64, 1, 128, 16, "bf16", [40, 3], [9, 3]),
    ("g4-fp16-d128-bs32", 8, 2, 128, 32, "fp16", [333, 97, 64], [200, 97, 33]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prefill_matches_oracle(pkv, case):
    name, hq, hkv, D, bs, dt, lens, chunks = case
    pw = W.make_prefill_workload(name, hq, hkv, D, bs, dt, lens, chunks, seed=11, device=DEV)
    pool, out = _run(pkv, pw)
    assert pool.status() == 0
    k, v = _cache_16(pw.cache)
    ref = attention.paged_prefill(to_np(pw.q, np.float64), pw.cu_q, k, v, pw.cache.block_tables,
                                  pw.cache.context_lens, pw.cache.scale)
    compare(out, ref, what=name)


# Several hundred work items (token tile x KV head), more than one per SM: each
# CTA walks 2 to 5 items, so Q buffers, ring stages and S/P buffers carry over
# from one item to the next; prefixes and chunks vary (odd and even stage
# counts, tiles past a short chunk).
MANY = [
    ("many-g8-d128-bs16", 32, 4, 128, 16, "bf16",
     [400, 387, 397, 400, 262, 500, 162, 257, 117, 267],
     [400, 350, 333, 300, 257, 200, 161, 129, 100, 17]),
    ("many-g8-d64-bs32", 32, 4, 64, 32, "fp16",
     [700, 650, 600, 513, 64, 999],
     [640, 533, 500, 457, 64, 450]),
]


@pytest.mark.parametrize("case", MANY, ids=[c[0] for c in MANY])
def test_prefill_many_items_per_cta(pkv, case):
    from concurrent.futures import ThreadPoolExecutor
    name, hq, hkv, D, bs, dt, lens, chunks = case
    pw = W.make_prefill_workload(name, hq, hkv, D, bs, dt, lens, chunks, seed=17, device=DEV)
    pool, out = _run(pkv, pw)
    assert pool.status() == 0
    wl = pw.cache
    k, v = _cache_16(wl)
    q64 = to_np(pw.q, np.float64)

    def one(b):
        lo, hi = int(pw.cu_q[b]), int(pw.cu_q[b + 1])
        return attention.paged_prefill(q64[lo:hi], np.array([0, hi - lo]), k, v,
                                       wl.block_tables[b:b + 1], wl.context_lens[b:b + 1],
                                       wl.scale)

    with ThreadPoolExecutor(8) as ex:
        ref = np.concatenate(list(ex.map(one, range(wl.batch))))
    compare(out, ref, what=name)


@pytest.mark.parametrize("scale", [0.0, -0.3, 0.15])
def test_prefill_any_finite_scale(pkv, scale):
    """The softmax scale may be zero (every attended position weighs the same)
    or negative; the kernel folds its sign into q and keeps its own scale
    positive."""
    pw = W.make_prefill_workload("scale", 16, 2, 128, 16, "bf16", [200, 77, 40], [150, 77, 3],
                                 seed=19, device=DEV)
    wl = pw.cache
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    cu = torch.from_numpy(pw.cu_q).to(DEV)
    out = pkv.paged_attn_prefill(pool, 0, pw.q, cu, 150, tables, lens, 200, scale)
    torch.cuda.synchronize()
    assert pool.status() == 0
    k, v = _cache_16(wl)
    ref = attention.paged_prefill(to_np(pw.q, np.float64), pw.cu_q, k, v, wl.block_tables,
                                  wl.context_lens, scale)
    compare(out, ref, what="scale %g" % scale)


def _random_case(seed):
    """A seeded random prefill shape: group size, head_dim, block size, dtype,
    2 to 5 sequences with prefixes of 0 to 300 and chunks of 1 to 160 tokens."""
    rng = np.random.default_rng(seed)
    hkv = int(rng.choice([1, 2, 4]))
    g = int(rng.choice([1, 2, 4, 8, 16]))
    D = int(rng.choice([64, 128]))
    bs = int(rng.choice([16, 32]))
    dt = str(rng.choice(["bf16", "fp16"]))
    n = int(rng.integers(2, 6))
    chunks = [int(x) for x in rng.integers(1, 161, n)]
    lens = [c + int(rng.integers(0, 301)) for c in chunks]
    return ("rand%d" % seed, g * hkv, hkv, D, bs, dt, lens, chunks)


@pytest.mark.parametrize("seed", range(6))
def test_prefill_random_shapes(pkv, seed):
    name, hq, hkv, D, bs, dt, lens, chunks = _random_case(seed)
    pw = W.make_prefill_workload(name, hq, hkv, D, bs, dt, lens, chunks, seed=100 + seed,
                                 device=DEV)
    pool, out = _run(pkv, pw)
    assert pool.status() == 0
    k, v = _cache_16(pw.cache)
    ref = attention.paged_prefill(to_np(pw.q, np.float64), pw.cu_q, k, v, pw.cache.block_tables,
                                  pw.cache.context_lens, pw.cache.scale)
    compare(out, ref, what=name)


def test_prefill_last_token_agrees_with_decode(pkv):
    """A one-token chunk is a decode step: both paths give the same output
    within the tolerance (different kernels, different orders)."""
    pw = W.make_prefill_workload("one", 16, 2, 128, 16, "bf16", [300, 45, 129], [1, 1, 1],
                                 seed=12, device=DEV)
    pool, out = _run(pkv, pw)
    wl = pw.cache
    tables, lens = device_inputs(wl, DEV)
    dec = pkv.paged_attn_decode(pool, 0, pw.q.contiguous(), tables, lens,
                                int(wl.context_lens.max()), wl.scale)
    torch.cuda.synchronize()
    diff = (out.float() - dec.float()).abs().max().item()
    assert diff <= 1e-2


def test_prefill_70b_shape_sampled(pkv):
    """The 70B-shaped chunked-prefill workload (8 requests, 512 new tokens
    behind a 1536-token prefix): sampled rows against the oracle."""
    pw = W.prefill70b(DEV)
    pool, out = _run(pkv, pw)
    assert pool.status() == 0
    wl = pw.cache
    k, v = _cache_16(wl)
    rows = [(b, i) for b in (0, 5, 7) for i in (0, 1, 15, 16, 255, 511)]
    got = torch.stack([out[pw.cu_q[b] + i] for b, i in rows])
    ref = np.stack([np.stack([attention.prefill_one(to_np(pw.q[pw.cu_q[b] + i, h], np.float64), k, v,
                                                    wl.block_tables[b],
                                                    int(wl.context_lens[b] - pw.chunk_lens[b] + i),
                                                    h // 8, wl.scale)
                              for h in range(64)]) for b, i in rows])
    compare(got, ref, what="prefill70b")


def test_prefill_bad_block_id_is_reported(pkv):
    """A block id outside the pool is reported in the status word and its
    positions are skipped; outputs stay finite and the other sequence's rows
    match the oracle."""
    pw = W.make_prefill_workload("badid", 16, 2, 128, 16, "bf16", [300, 90], [120, 40], seed=21,
                                 device=DEV)
    wl = pw.cache
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    tables[0, 3] = wl.num_blocks + 5              # outside the pool
    cu = torch.from_numpy(pw.cu_q).to(DEV)
    pool.status_clear()
    out = pkv.paged_attn_prefill(pool, 0, pw.q, cu, 120, tables, lens, 300, wl.scale)
    torch.cuda.synchronize()
    assert pool.status() & 1
    assert torch.all(torch.isfinite(out.float()))
    k, v = _cache_16(wl)
    lo = int(pw.cu_q[1])
    ref = attention.paged_prefill(to_np(pw.q[lo:], np.float64), np.array([0, 40]), k, v,
                                  wl.block_tables[1:], wl.context_lens[1:], wl.scale)
    compare(out[lo:], ref, what="good sequence")


def test_prefill_bad_chunk_is_reported(pkv):
    pw = W.make_prefill_workload("bad", 8, 2, 64, 16, "bf16", [40, 30], [10, 12], seed=13,
                                 device=DEV)
    wl = pw.cache
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    lens[1] = 5                                   # fewer positions than new tokens
    cu = torch.from_numpy(pw.cu_q).to(DEV)
    out = torch.full_like(pw.q, 7.0)
    pool.status_clear()
    pkv.paged_attn_prefill(pool, 0, pw.q, cu, 12, tables, lens, 40, wl.scale, out=out)
    torch.cuda.synchronize()
    assert pool.status() & 2
    assert torch.all(out[10:] == 7.0)             # the bad sequence's rows are left alone
    k, v = _cache_16(wl)
    ref = attention.paged_prefill(to_np(pw.q[:10], np.float64), pw.cu_q[:2], k, v,
                                  wl.block_tables[:1], wl.context_lens[:1], wl.scale)
    compare(out[:10], ref, what="good sequence")


@pytest.mark.parametrize("D,bs", [(128, 16), (64, 32)])
def test_prefill_ignores_nan_past_the_context(pkv, D, bs):
    """Cache rows past each sequence's last position (the tail of its last
    block) and blocks no table names hold NaN: they are never attended, so
    the output is finite and matches the oracle."""
    pw = W.make_prefill_workload("nan", 16, 2, D, bs, "bf16", [37, 300, 129, 70], [37, 45, 9, 70],
                                 seed=14, device=DEV)
    wl = pw.cache
    pool = build_pool(pkv, wl, DEV)
    K, V, _, _ = pool.layer_views(0)
    used = set()
    for b, L in enumerate(wl.context_lens):
        nb = (int(L) + bs - 1) // bs
        used.update(int(x) for x in wl.block_tables[b][:nb])
        last = int(wl.block_tables[b][nb - 1])
        if L % bs:
            K[last, :, int(L) % bs:] = float("nan")
            V[last, :, int(L) % bs:] = float("nan")
    for blk in range(wl.num_blocks):
        if blk not in used:
            K[blk] = float("nan")
            V[blk] = float("nan")
    tables, lens = device_inputs(wl, DEV)
    cu = torch.from_numpy(pw.cu_q).to(DEV)
    out = pkv.paged_attn_prefill(pool, 0, pw.q, cu, int(pw.chunk_lens.max()), tables, lens,
                                 int(wl.context_lens.max()), wl.scale)
    torch.cuda.synchronize()
    assert pool.status() == 0
    k, v = _cache_16(wl)
    ref = attention.paged_prefill(to_np(pw.q, np.float64), pw.cu_q, k, v, wl.block_tables,
                                  wl.context_lens, wl.scale)
    compare(out, ref, what="nan tail")
