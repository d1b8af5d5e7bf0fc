"""GPU parity of paged decode attention against the fp64 oracle.

Each test runs one decode step (append of the step's token, then attention)
through the C ABI and compares every output it checks, element by element, with
the oracle on the same generated inputs. Tolerance: max abs 1e-2 and max rel
1e-2 (relative to max(|ref|, 1e-2)). Full-size workloads run in the launch
configuration the benchmark times (default partition size); outputs there are
checked for all heads of every sequence, or of a seeded sample of sequences
where the oracle would be slow.
"""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_support import (bits16, build_pool, check_quant_pool, compare, device_inputs,
                         oracle_cache_16, oracle_cache_quant, oracle_outputs, step, to_np)
from oracle import cache_ops

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_440_b200 as p
    return p


def _all_pairs(wl, seqs=None):
    seqs = range(wl.batch) if seqs is None else seqs
    return [(b, h) for b in seqs for h in range(wl.q_heads)]


def _run_16(pkv, wl, num_ctas=0, seqs=None):
    pool = build_pool(pkv, wl, DEV)
    out = step(pkv, pool, wl, DEV, num_ctas)
    torch.cuda.synchronize()
    assert pool.status() == 0
    k, v = oracle_cache_16(wl)
    pairs = _all_pairs(wl, seqs)
    ref = oracle_outputs(wl, k, v, pairs)
    got = torch.stack([out[b, h] for b, h in pairs])
    return compare(got, ref, what=wl.name)


def test_tiny_default_split(pkv):
    _run_16(pkv, W.tiny(DEV))


@pytest.mark.parametrize("G", [1, 2, 3, 5, 13, 56, 57, 200])
def test_tiny_split_counts_agree(pkv, G):
    """The tiny case has 56 (sequence, kv head) blocks: from one CTA doing
    everything to more CTAs than blocks (idle CTAs), splits fall everywhere."""
    _run_16(pkv, W.tiny(DEV), num_ctas=G)


def test_gqa70b_every_output(pkv):
    """LLaMA-70B-shaped GQA layer, batch 32, lengths U[512, 4096], all 2048 outputs."""
    _run_16(pkv, W.gqa70b(DEV))


@pytest.mark.parametrize("G", [7, 300, 2000])
def test_gqa70b_split_counts(pkv, G):
    _run_16(pkv, W.gqa70b(DEV), num_ctas=G, seqs=[0, 7, 19, 31])


def test_mha13b_every_output(pkv):
    """13B-shaped MHA layer (40/40 heads, fp16), batch 32 x 2048, all 1280 outputs."""
    _run_16(pkv, W.mha13b(DEV))


def test_gqa70b_benchmarked_call(pkv):
    """Exactly the call the benchmark times: paged_attn_decode_append on the
    LLaMA-70B-shaped layer (batch 32, lengths U[512, 4096]) with the default
    CTA count and a workspace from make_workspace. Every pool row is bit-exact
    with the oracle's append (the new token at position L - 1), and all 2048
    outputs match the oracle."""
    wl = W.gqa70b(DEV)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    G = pkv.default_ctas(pool)
    ws = pkv.make_workspace(pool, wl.batch, wl.q_heads, G)
    out = torch.empty_like(wl.q)
    pkv.paged_attn_decode_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens,
                                 int(wl.context_lens.max()), wl.scale, out=out, num_ctas=G,
                                 workspace=ws)
    torch.cuda.synchronize()
    assert pool.status() == 0
    K, V, _, _ = pool.layer_views(0)
    kb, vb = bits16(wl.k_fill), bits16(wl.v_fill)
    cache_ops.append(kb, vb, bits16(wl.k_new), bits16(wl.v_new), wl.slot_new, wl.block_size)
    assert np.array_equal(bits16(K), kb) and np.array_equal(bits16(V), vb)
    k, v = oracle_cache_16(wl)
    pairs = _all_pairs(wl)
    compare(torch.stack([out[b, h] for b, h in pairs]), oracle_outputs(wl, k, v, pairs),
            what="gqa70b benchmarked call")


@pytest.mark.parametrize("kind", ["int8", "e5m2", "int4", "int8_kchan", "e5m2_cast"])
@pytest.mark.parametrize("variant,seqs", [("a", [0, 9, 13, 27, 40, 51, 58, 63]), ("b", [0, 5])])
def test_quantized_long_context(pkv, kind, variant, seqs):
    """Quantized KV, bs 32, (a) 64 x 4096 and (b) 8 x 32768, through the call
    the benchmark times (paged_attn_decode_append: history appended with
    kv_append, the step's token quantized inside the attention kernel). Every
    code and scale of every sequence is bit-exact with the oracle's
    quantization of the same rows; outputs of the sampled sequences match the
    oracle run on the same dequantized values."""
    wl = W.quant_long(kind, variant, DEV)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    out = pkv.paged_attn_decode_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens,
                                       int(wl.context_lens.max()), wl.scale)
    torch.cuda.synchronize()
    assert pool.status() == 0
    rows = check_quant_pool(wl, pool)
    assert rows == int(wl.context_lens.sum()) * wl.kv_heads
    _, (kd, vd, otab) = oracle_cache_quant(wl, seqs)
    pairs = _all_pairs(wl, seqs)
    ref = oracle_outputs(wl, kd, vd, pairs, otab)
    compare(torch.stack([out[b, h] for b, h in pairs]), ref, what=wl.name)


def test_shared_prefix_copy_on_write(pkv):
    """200 requests share a 1500-token prompt (94 blocks of 16, the last holding
    12 tokens). Every request copies the shared partial block before appending
    its private suffix. The oracle builds its own cache with its own allocator
    model and copies; the outputs of all 200 requests agree."""
    from oracle import allocator, cache_ops
    wl = W.shared_prefix(DEV)
    bs, hkv, D = wl.block_size, wl.kv_heads, wl.head_dim
    P = wl.prefix_len
    nprefix = -(-P // bs)

    # ------------------------------------------------ CUDA path (product API)
    pool = pkv.KVPool(1, wl.num_blocks, bs, hkv, D, "bf16", DEV)
    K, V, _, _ = pool.layer_views(0)
    K.zero_()
    V.zero_()
    prefix_ids = pool.alloc(nprefix)
    slots = torch.tensor([prefix_ids[t // bs] * bs + t % bs for t in range(P)],
                         dtype=torch.int64, device=DEV)
    pkv.kv_append(pool, 0, wl.prefix_k, wl.prefix_v, slots)
    tables = []
    for b in range(wl.batch):
        pool.share(prefix_ids)
        tables.append(list(prefix_ids))
    pairs = []
    for b in range(wl.batch):
        last = tables[b][nprefix - 1]
        new = pool.cow_prepare(last)
        assert new != last
        pairs.append((last, new))
        tables[b][nprefix - 1] = new
    assert pool.refcount(prefix_ids[-1]) == 1 and pool.refcount(prefix_ids[0]) == 201
    pkv.kv_block_copy(pool, pairs)
    sl = []
    for b in range(wl.batch):
        L = P + int(wl.suffix_lens[b])
        need = -(-L // bs) - len(tables[b])
        tables[b] += pool.alloc(need)
        sl += [tables[b][t // bs] * bs + t % bs for t in range(P, L)]
    pkv.kv_append(pool, 0, wl.suffix_k, wl.suffix_v, torch.tensor(sl, dtype=torch.int64, device=DEV))
    lens = P + wl.suffix_lens
    mb = max(len(t) for t in tables)
    tbl = np.full((wl.batch, mb), -1, np.int32)
    for b, t in enumerate(tables):
        tbl[b, :len(t)] = t
    out = pkv.paged_attn_decode(pool, 0, wl.q, torch.from_numpy(tbl).to(DEV),
                                torch.from_numpy(lens.astype(np.int32)).to(DEV),
                                int(lens.max()), wl.scale)
    torch.cuda.synchronize()
    assert pool.status() == 0
    st = pool.stats()
    assert st["shared"] == nprefix - 1

    # ------------------------------------------------ oracle (own allocation)
    m = allocator.PoolModel(wl.num_blocks)
    kc = np.zeros((wl.num_blocks, hkv, bs, D), np.float32)
    vc = np.zeros_like(kc)
    o_prefix = m.alloc(nprefix)
    cache_ops.append(kc, vc, to_np(wl.prefix_k), to_np(wl.prefix_v),
                     np.array([o_prefix[t // bs] * bs + t % bs for t in range(P)]), bs)
    o_tables = []
    for b in range(wl.batch):
        m.share(o_prefix)
        o_tables.append(list(o_prefix))
    o_pairs = []
    for b in range(wl.batch):
        fresh = m.alloc(1)[0]
        m.free([o_prefix[-1]])
        o_pairs.append((o_prefix[-1], fresh))
        o_tables[b][-1] = fresh
    cache_ops.block_copy([kc, vc], o_pairs)
    o_sl = []
    for b in range(wl.batch):
        L = P + int(wl.suffix_lens[b])
        o_tables[b] += m.alloc(-(-L // bs) - len(o_tables[b]))
        o_sl += [o_tables[b][t // bs] * bs + t % bs for t in range(P, L)]
    cache_ops.append(kc, vc, to_np(wl.suffix_k), to_np(wl.suffix_v), np.array(o_sl), bs)
    o_tbl = np.full((wl.batch, mb), -1, np.int64)
    for b, t in enumerate(o_tables):
        o_tbl[b, :len(t)] = t
    import concurrent.futures
    from oracle import attention
    q = to_np(wl.q, np.float64)
    pairs = [(b, h) for b in range(wl.batch) for h in range(wl.q_heads)]
    with concurrent.futures.ThreadPoolExecutor(max_workers=8) as ex:
        ref = np.stack(list(ex.map(
            lambda bh: attention.decode_one(q, kc, vc, o_tbl, lens, wl.scale, *bh), pairs)))
    got = torch.stack([out[b, h] for b, h in pairs])
    compare(got, ref, what="shared_prefix")
    # the cascade step on the same pool: the 93 blocks every request still
    # shares once for all requests on the tensor cores, the rest per request
    t_dev = torch.from_numpy(tbl).to(DEV)
    l_dev = torch.from_numpy(lens.astype(np.int32)).to(DEV)
    assert all(t[:nprefix - 1] == tables[0][:nprefix - 1] for t in tables)
    out_c = pkv.paged_attn_decode_cascade(pool, 0, wl.q, t_dev, l_dev, int(lens.max()),
                                          nprefix - 1, wl.scale)
    torch.cuda.synchronize()
    assert pool.status() == 0
    compare(torch.stack([out_c[b, h] for b, h in pairs]), ref, what="shared_prefix cascade")


# --------------------------------------------------------------- edge cases

EDGE_LENS = [0, 1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 300]


@pytest.mark.parametrize("cache", ["bf16", "fp16", "int8", "e5m2", "e5m2_cast", "int4",
                                   "int8_kchan"])
@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("D,bs", [(64, 16), (128, 32)])
def test_edge_lengths_groups_dims(pkv, cache, G, D, bs):
    """Empty, single-token and block-boundary lengths; MHA, GQA groups of 2..16
    heads (16 spans two head units); head_dim 64 / 128; block size 16 / 32; all
    four cache types; 13 CTAs, so units are split at assorted places."""
    if cache == "int4" and D != 128:
        pytest.skip("INT4 rows need head_dim 128")
    qd = "fp16" if cache == "fp16" else "bf16"
    lens = EDGE_LENS
    wl = W.make_decode_workload("edge", len(lens), 2 * G, 2, D, bs, qd, cache, lens,
                                seed=G * 1000 + D + bs, device=DEV)
    pool = build_pool(pkv, wl, DEV)
    out = step(pkv, pool, wl, DEV, num_ctas=13)
    torch.cuda.synchronize()
    assert pool.status() == 0
    pairs = _all_pairs(wl)
    if cache in ("bf16", "fp16"):
        k, v = oracle_cache_16(wl)
        tab = None
    else:
        _, (k, v, tab) = oracle_cache_quant(wl, list(range(wl.batch)))
    ref = oracle_outputs(wl, k, v, pairs, tab)
    compare(torch.stack([out[b, h] for b, h in pairs]), ref, what="edge %s G%d" % (cache, G))
    assert torch.all(out[0] == 0)     # empty sequence


def test_separate_phases_equal_fused_call(pkv):
    wl = W.gqa70b(DEV, batch=8)
    pool = build_pool(pkv, wl, DEV)
    out = step(pkv, pool, wl, DEV, num_ctas=37)
    tables, lens = device_inputs(wl, DEV)
    ws = pkv.make_workspace(pool, wl.batch, wl.q_heads, 37)
    out2 = torch.empty_like(out)
    pkv.paged_attn_partition(pool, 0, wl.q, tables, lens, int(wl.context_lens.max()), wl.scale,
                             out2, ws, num_ctas=37)
    pkv.paged_attn_merge(pool, lens, tables.shape[1], int(wl.context_lens.max()), out2, ws,
                         num_ctas=37)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_bad_block_id_and_length_are_reported(pkv):
    wl = W.make_decode_workload("bad", 3, 8, 2, 64, 16, "bf16", "bf16", [40, 40, 40],
                                seed=5, device=DEV)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    tables[1, 1] = wl.num_blocks + 7          # outside the pool
    lens[2] = 10_000                           # beyond the table width and max_context
    pool.status_clear()
    out = pkv.paged_attn_decode(pool, 0, wl.q, tables, lens, 64, wl.scale)
    torch.cuda.synchronize()
    st = pool.status()
    assert st & 1 and st & 2
    assert torch.all(torch.isfinite(out.float()))
    assert torch.all(out[2] == 0)
    # sequence 0 is untouched by the bad entries
    k, v = to_np(wl.k_fill), to_np(wl.v_fill)
    ref = oracle_outputs(wl, k, v, [(0, h) for h in range(8)])
    compare(out[0], ref, what="good sequence")


# --------------------------------------------------------------- fused append

def _fused_workloads():
    return [
        ("tiny", lambda: W.tiny(DEV)),
        ("gqa70b-8", lambda: W.gqa70b(DEV, batch=8)),
        ("mha-fp16", lambda: W.make_decode_workload("mha", 6, 4, 4, 128, 16, "fp16", "fp16",
                                                    [1, 16, 17, 200, 31, 64], seed=3, device=DEV)),
        ("g4-d64-bs32", lambda: W.make_decode_workload("g4", 5, 8, 2, 64, 32, "bf16", "bf16",
                                                       [0, 1, 32, 33, 150], seed=4, device=DEV)),
        ("int8", lambda: W.make_decode_workload("q8", 4, 16, 2, 128, 32, "bf16", "int8",
                                                [1, 31, 32, 300], seed=5, device=DEV)),
        ("e5m2", lambda: W.make_decode_workload("e5", 4, 16, 2, 128, 16, "bf16", "e5m2",
                                                [2, 17, 64, 129], seed=6, device=DEV)),
        ("e5m2-cast", lambda: W.make_decode_workload("e5c", 4, 16, 2, 64, 32, "fp16", "e5m2_cast",
                                                     [3, 32, 33, 200], seed=8, device=DEV)),
        ("int4", lambda: W.make_decode_workload("i4", 5, 16, 2, 128, 16, "bf16", "int4",
                                                [1, 15, 16, 17, 300], seed=9, device=DEV)),
        ("int8-kchan", lambda: W.make_decode_workload("kc", 4, 16, 2, 128, 32, "bf16", "int8_kchan",
                                                      [1, 31, 32, 300], seed=10, device=DEV)),
        ("int8-kchan-d64", lambda: W.make_decode_workload("kc64", 4, 8, 2, 64, 16, "fp16",
                                                          "int8_kchan", [2, 16, 17, 129],
                                                          seed=11, device=DEV)),
    ]


@pytest.mark.parametrize("name,make", _fused_workloads())
@pytest.mark.parametrize("num_ctas", [0, 7])
def test_fused_append_matches_oracle(pkv, name, make, num_ctas):
    """paged_attn_decode_append writes the step's token at position L - 1 (bit-
    exact with the oracle's append / quantize) and attends over it."""
    wl = make()
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    max_ctx = max(int(wl.context_lens.max()), 1)
    out = pkv.paged_attn_decode_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens, max_ctx,
                                       wl.scale, num_ctas=num_ctas)
    torch.cuda.synchronize()
    assert pool.status() == 0
    pairs = _all_pairs(wl)
    K, V, KS, VS = pool.layer_views(0)
    if wl.cache_dtype in ("bf16", "fp16"):
        k, v = oracle_cache_16(wl)
        tab = None
        kb, vb = bits16(wl.k_fill), bits16(wl.v_fill)
        cache_ops.append(kb, vb, bits16(wl.k_new), bits16(wl.v_new), wl.slot_new, wl.block_size)
        assert np.array_equal(bits16(K), kb) and np.array_equal(bits16(V), vb)
    else:
        (kc, vc, ks, vs), (k, v, tab) = oracle_cache_quant(wl, list(range(wl.batch)))
        used = sorted({int(x) for b in range(wl.batch)
                       for x in wl.block_tables[b, :-(-int(wl.context_lens[b]) // wl.block_size)]})
        assert np.array_equal(K[used].cpu().numpy(), kc[used])
        assert np.array_equal(V[used].cpu().numpy(), vc[used])
        if wl.cache_dtype == "int8_kchan":      # layer channel scales, per-token V scales
            assert np.array_equal(KS.cpu().numpy(), wl.k_chan)
            assert np.array_equal(VS[used].cpu().numpy().view(np.uint32), vs[used].view(np.uint32))
        elif KS is not None:                     # the scale-less cast keeps no scales
            assert np.array_equal(KS[used].cpu().numpy().view(np.uint32), ks[used].view(np.uint32))
            assert np.array_equal(VS[used].cpu().numpy().view(np.uint32), vs[used].view(np.uint32))
    ref = oracle_outputs(wl, k, v, pairs, tab)
    compare(torch.stack([out[b, h] for b, h in pairs]), ref, what="fused append " + name)


def test_fused_append_rejects_more_than_8_heads_per_kv_head(pkv):
    wl = W.make_decode_workload("g16", 2, 32, 2, 64, 16, "bf16", "bf16", [5, 9], seed=7,
                                device=DEV)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attn_decode_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens, 9, wl.scale)
    assert e.value.status == 4


def test_fused_append_phases_equal_one_call(pkv):
    """paged_attn_partition_append + paged_attn_merge gives the bits of
    paged_attn_decode_append."""
    wl = W.gqa70b(DEV, batch=6)
    tables, lens = device_inputs(wl, DEV)
    max_ctx = int(wl.context_lens.max())
    outs = []
    for phases in (False, True):
        pool = build_pool(pkv, wl, DEV)
        if phases:
            ws = pkv.make_workspace(pool, wl.batch, wl.q_heads, 11)
            out = torch.empty_like(wl.q)
            pkv.paged_attn_partition_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens,
                                            max_ctx, wl.scale, out, ws, num_ctas=11)
            pkv.paged_attn_merge(pool, lens, tables.shape[1], max_ctx, out, ws, num_ctas=11)
        else:
            out = pkv.paged_attn_decode_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens,
                                               max_ctx, wl.scale, num_ctas=11)
        torch.cuda.synchronize()
        outs.append((bits16(out), bits16(pool.layer_views(0)[0]), bits16(pool.layer_views(0)[1])))
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("name,make", _fused_workloads())
@pytest.mark.parametrize("G", [3, 37, 0, 300])
def test_decode_whatever_the_workspace_held(pkv, name, make, G):
    """The split-K workspace needs no initialisation: paged_attn_decode gives
    the bits of a first partition + merge whatever the workspace held before
    (zeros, all ones, random bytes), and again on a second call with the same
    workspace."""
    wl = make()
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    pkv.kv_append(pool, 0, wl.k_new, wl.v_new, torch.from_numpy(wl.slot_new).to(DEV))
    max_ctx = max(int(wl.context_lens.max()), 1)
    ws = pkv.make_workspace(pool, wl.batch, wl.q_heads, G)
    ref = torch.empty_like(wl.q)
    pkv.paged_attn_partition(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, ref, ws, num_ctas=G)
    pkv.paged_attn_merge(pool, lens, tables.shape[1], max_ctx, ref, ws, num_ctas=G)
    gen = torch.Generator(device=DEV).manual_seed(G + 1)
    fills = [lambda: ws.zero_(), lambda: ws.fill_(255),
             lambda: ws.copy_(torch.randint(0, 256, ws.shape, generator=gen, device=DEV,
                                            dtype=torch.int32).to(torch.uint8))]
    for fill in fills:
        fill()
        for _ in range(2):
            out = torch.full_like(wl.q, float("nan"))
            pkv.paged_attn_decode(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, out=out,
                                  num_ctas=G, workspace=ws)
            torch.cuda.synchronize()
            assert np.array_equal(bits16(out), bits16(ref)), name
    assert pool.status() == 0


def test_decode_graph_replays_match(pkv):
    """A decode step captured in a CUDA graph (both kernels, launched so that
    the merge may start while the attention kernel drains) gives, replay after
    replay, the bits of the separate partition + merge calls."""
    wl = W.gqa70b(DEV, batch=12)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    pkv.kv_append(pool, 0, wl.k_new, wl.v_new, torch.from_numpy(wl.slot_new).to(DEV))
    max_ctx = int(wl.context_lens.max())
    G = 53
    ws = pkv.make_workspace(pool, wl.batch, wl.q_heads, G)
    ref = torch.empty_like(wl.q)
    pkv.paged_attn_partition(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, ref, ws, num_ctas=G)
    pkv.paged_attn_merge(pool, lens, tables.shape[1], max_ctx, ref, ws, num_ctas=G)
    out = torch.empty_like(wl.q)
    pkv.paged_attn_decode(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, out=out, num_ctas=G,
                          workspace=ws)           # warm-up outside the capture
    torch.cuda.synchronize()
    assert np.array_equal(bits16(out), bits16(ref))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        pkv.paged_attn_decode(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, out=out,
                              num_ctas=G, workspace=ws)
    for _ in range(3):
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bits16(out), bits16(ref))
    del graph
    assert pool.status() == 0


# ------------------------------------------------ cascade (shared prefix) step

def _cascade_case(seed):
    """Sequences whose tables start with the same pb blocks: seeded shapes over
    dtype, head_dim, block size, heads, batch, prefix and suffix lengths (some
    suffixes empty when there is no append)."""
    rng = np.random.default_rng(1000 + seed)
    dtype = ("bf16", "fp16")[seed % 2]
    D = (64, 128)[(seed // 2) % 2]
    bs = (16, 32)[(seed // 4) % 2]
    hkv = int(rng.choice([1, 2, 4, 8]))
    append = seed % 3 != 2
    G = (1, 2, 4, 8)[seed % 4] if append else (16, 64, 8, 1)[(seed // 3) % 4]
    B = int(rng.integers(1, 48))
    pb = int(rng.integers(1, 9))
    suffix = rng.integers(1 if append else 0, 5 * bs, size=B)
    if not append:
        suffix[0] = 0                       # the prefix alone
    lens = pb * bs + suffix
    nblk = -(-lens // bs)
    N = pb + int((nblk - pb).sum()) + 8
    perm = rng.permutation(N).astype(np.int32)
    mb = int(nblk.max()) + 1
    tables = np.full((B, mb), -1, np.int32)
    pos = pb
    for b in range(B):
        tables[b, :pb] = perm[:pb]
        k = int(nblk[b]) - pb
        tables[b, pb:pb + k] = perm[pos:pos + k]
        pos += k
    wl = W.make_decode_workload("cascade%d" % seed, B, G * hkv, hkv, D, bs, dtype, dtype, lens,
                                num_blocks=N, seed=seed, device=DEV, placement=tables)
    return wl, pb, append


@pytest.mark.parametrize("seed", range(10))
def test_cascade_matches_oracle(pkv, seed):
    """paged_attn_decode_cascade: every output against the oracle's decode over
    the whole tables (prefix included); with an append, the new rows are in the
    pool bit for bit."""
    wl, pb, append = _cascade_case(seed)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    kw = dict(k_new=wl.k_new, v_new=wl.v_new) if append else {}
    out = pkv.paged_attn_decode_cascade(pool, 0, wl.q, tables, lens, int(wl.context_lens.max()),
                                        pb, wl.scale, **kw)
    torch.cuda.synchronize()
    assert pool.status() == 0
    if append:
        k, v = oracle_cache_16(wl)
    else:
        dt = np.float16 if wl.cache_dtype == "fp16" else np.float32
        k, v = to_np(wl.k_fill, dt), to_np(wl.v_fill, dt)
    pairs = _all_pairs(wl)
    ref = oracle_outputs(wl, k, v, pairs)
    compare(torch.stack([out[b, h] for b, h in pairs]), ref, what=wl.name)
    if append:
        K, V, _, _ = pool.layer_views(0)
        bs = wl.block_size
        for b in range(wl.batch):
            s_ = int(wl.slot_new[b])
            assert np.array_equal(bits16(K[s_ // bs, :, s_ % bs]), bits16(wl.k_new[b]))
            assert np.array_equal(bits16(V[s_ // bs, :, s_ % bs]), bits16(wl.v_new[b]))


def test_cascade_reports_lengths_inside_the_prefix(pkv):
    """A length shorter than the prefix, or (with an append) equal to it, is
    reported on the device; the other sequences' outputs stay exact."""
    wl, pb, _ = _cascade_case(0)
    assert wl.batch >= 3
    bs = wl.block_size
    pool = build_pool(pkv, wl, DEV)
    pool.status_clear()
    tables, lens = device_inputs(wl, DEV)
    bad = lens.clone()
    bad[1] = pb * bs - 1
    out = pkv.paged_attn_decode_cascade(pool, 0, wl.q, tables, bad, int(wl.context_lens.max()),
                                        pb, wl.scale)
    torch.cuda.synchronize()
    assert pool.status() & 2                 # KV_DEVERR_CONTEXT
    assert torch.count_nonzero(out[1]) == 0
    dt = np.float16 if wl.cache_dtype == "fp16" else np.float32
    k, v = to_np(wl.k_fill, dt), to_np(wl.v_fill, dt)
    pairs = [(b, h) for b in (0, 2) for h in range(wl.q_heads)]
    compare(torch.stack([out[b, h] for b, h in pairs]), oracle_outputs(wl, k, v, pairs))
    pool.status_clear()
    bad = lens.clone()
    bad[2] = pb * bs                      # the new token would land in the shared blocks
    pkv.paged_attn_decode_cascade(pool, 0, wl.q, tables, bad, int(wl.context_lens.max()), pb,
                                  wl.scale, k_new=wl.k_new, v_new=wl.v_new)
    torch.cuda.synchronize()
    assert pool.status() & 2                 # KV_DEVERR_CONTEXT
