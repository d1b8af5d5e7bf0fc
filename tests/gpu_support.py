"""Helpers for the GPU parity tests.

The CUDA path is driven through the package's public API; expected values are
computed only by ``oracle/`` from the generated inputs (never from anything the
GPU produced).
"""
import numpy as np
import torch

from oracle import attention, cache_ops, quant

TOL = 1e-2          # max abs and max rel (floor 1e-2 on |ref|) for attention outputs


def to_np(t, dtype=np.float32):
    return t.detach().float().cpu().numpy().astype(dtype)


def bits16(t):
    return t.detach().contiguous().view(torch.int16).cpu().numpy()


def compare(gpu_out, ref, tol=TOL, what=""):
    """Element-wise check of a bf16/fp16 GPU output against the fp64 oracle."""
    g = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), "%s: non-finite GPU output" % what
    err = np.abs(g - ref)
    max_abs = float(err.max()) if err.size else 0.0
    max_rel = float((err / np.maximum(np.abs(ref), 1e-2)).max()) if err.size else 0.0
    assert max_abs <= tol and max_rel <= tol, \
        "%s: max abs %.3g, max rel %.3g (tolerance %g)" % (what, max_abs, max_rel, tol)
    return max_abs, max_rel


def device_inputs(wl, device):
    tables = torch.from_numpy(wl.block_tables).to(device)
    lens = torch.from_numpy(wl.context_lens.astype(np.int32)).to(device)
    return tables, lens


def build_pool(pkv, wl, device, chunk=65536):
    """A one-layer pool holding the workload's history, filled via the product API
    for quantized caches (kv_append) and by a plain device copy for 16-bit ones."""
    pool = pkv.KVPool(1, wl.num_blocks, wl.block_size, wl.kv_heads, wl.head_dim,
                      wl.cache_dtype, device)
    K, V, KS, VS = pool.layer_views(0)
    if wl.k_fill is not None:
        K.copy_(wl.k_fill)
        V.copy_(wl.v_fill)
    else:
        # rows no append writes compare against the oracle's zeros
        for t in (K, V, KS, VS):
            if t is not None:                     # the scale-less cast has no scales
                t.zero_()
        if wl.cache_dtype == "int8_kchan":        # the layer's key channel scales
            KS.copy_(torch.from_numpy(wl.k_chan).to(device))
        slots = torch.from_numpy(wl.slot_hist).to(device)
        for s in range(0, wl.k_hist.shape[0], chunk):
            pkv.kv_append(pool, 0, wl.k_hist[s:s + chunk].contiguous(),
                          wl.v_hist[s:s + chunk].contiguous(), slots[s:s + chunk].contiguous())
    return pool


def step(pkv, pool, wl, device, num_ctas=0, out=None):
    """One decode step through the product API: append the new token, attend."""
    tables, lens = device_inputs(wl, device)
    slot_new = torch.from_numpy(wl.slot_new).to(device)
    pkv.kv_append(pool, 0, wl.k_new, wl.v_new, slot_new)
    max_ctx = int(wl.context_lens.max()) if wl.batch else 0
    return pkv.paged_attn_decode(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, out=out,
                                 num_ctas=num_ctas)


def oracle_cache_16(wl):
    """Oracle's view of a 16-bit cache after this step's append (exact values:
    float16 for fp16 caches, float32 for bf16, which numpy lacks)."""
    dt = np.float16 if wl.cache_dtype == "fp16" else np.float32
    k = to_np(wl.k_fill, dt)
    v = to_np(wl.v_fill, dt)
    cache_ops.append(k, v, to_np(wl.k_new, dt), to_np(wl.v_new, dt), wl.slot_new, wl.block_size)
    return k, v


def oracle_cache_quant(wl, seqs):
    """Oracle codes/scales for the history and new token of the given sequences.

    Returns the full-size code and scale arrays (other sequences' blocks left
    zero) and, for attention, float64 dequantized caches holding only the
    sampled sequences' blocks, with block tables renumbered to match (the
    result does not depend on physical placement).
    """
    kchan = wl.cache_dtype == "int8_kchan"
    row = wl.head_dim // 2 if wl.cache_dtype == "int4" else wl.head_dim
    shape = (wl.num_blocks, wl.kv_heads, wl.block_size, row)
    cdt = np.int8 if wl.cache_dtype in ("int8", "int8_kchan") else np.uint8
    kc, vc = np.zeros(shape, cdt), np.zeros(shape, cdt)
    ks, vs = np.zeros(shape[:3], np.float32), np.zeros(shape[:3], np.float32)
    if kchan:
        ks = wl.k_chan

    def put(k, v, slots):
        if kchan:
            cache_ops.append_quantized_kchan(kc, vc, vs, k, v, slots, wl.block_size, wl.k_chan)
        else:
            cache_ops.append_quantized(kc, vc, ks, vs, k, v, slots, wl.block_size,
                                       wl.cache_dtype)
    starts = np.concatenate([[0], np.cumsum(np.maximum(wl.context_lens - 1, 0))])
    used = []
    for b in seqs:
        lo, hi = int(starts[b]), int(starts[b + 1])
        put(to_np(wl.k_hist[lo:hi]), to_np(wl.v_hist[lo:hi]), wl.slot_hist[lo:hi])
        put(to_np(wl.k_new[b:b + 1]), to_np(wl.v_new[b:b + 1]), wl.slot_new[b:b + 1])
        nblk = -(-int(wl.context_lens[b]) // wl.block_size)
        used += wl.block_tables[b, :nblk].tolist()
    used = sorted(set(used)) or [0]
    remap = {blk: i for i, blk in enumerate(used)}
    tables = np.full_like(wl.block_tables, -1)
    for b in seqs:
        nblk = -(-int(wl.context_lens[b]) // wl.block_size)
        tables[b, :nblk] = [remap[x] for x in wl.block_tables[b, :nblk]]
    u = np.array(used)
    unpack = quant.unpack_int4 if wl.cache_dtype == "int4" else (lambda c: c)
    if kchan:
        kd = quant.dequantize_k_channels(kc[u].transpose(0, 2, 1, 3), wl.k_chan) \
            .transpose(0, 2, 1, 3)                           # [U, bs, H, D] against [H, D]
        vd = quant.dequantize(vc[u], vs[u], "int8")
    else:
        kd = quant.dequantize(unpack(kc[u]), ks[u], wl.cache_dtype)
        vd = quant.dequantize(unpack(vc[u]), vs[u], wl.cache_dtype)
    return (kc, vc, ks, vs), (kd, vd, tables)


def oracle_outputs(wl, kcache, vcache, pairs, tables=None):
    """Oracle decode output for the listed (b, h) pairs."""
    q = to_np(wl.q, np.float64)
    tables = wl.block_tables if tables is None else tables
    return np.stack([attention.decode_one(q, kcache, vcache, tables,
                                          wl.context_lens, wl.scale, b, h) for b, h in pairs])


def raw_bytes(t):
    """Host copy of a device tensor's bytes, shaped [..., last * itemsize]."""
    return t.detach().contiguous().view(torch.uint8).cpu().numpy()


def host_f32(t):
    """Exact float32 host copy of a bf16 / fp16 device tensor (via its bits)."""
    u = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.bfloat16:
        return (u.astype(np.uint32) << 16).view(np.float32)
    return u.view(np.float16).astype(np.float32)


def check_quant_pool(wl, pool, threads=8):
    """Every code and scale byte a quantized cache holds for every sequence's
    positions 0 .. L-1 (its history, then the step's new token) against the
    oracle's quantization of the same rows. Sequences are checked in parallel
    threads (numpy releases the GIL); returns the number of rows checked."""
    import concurrent.futures
    K, V, KS, VS = pool.layer_views(0)
    kc, vc = K.cpu().numpy(), V.cpu().numpy()
    ks = KS.cpu().numpy() if KS is not None else None
    vs = VS.cpu().numpy() if VS is not None else None
    k_hist, v_hist = host_f32(wl.k_hist), host_f32(wl.v_hist)
    k_new, v_new = host_f32(wl.k_new), host_f32(wl.v_new)
    bs, H = wl.block_size, wl.kv_heads
    starts = np.concatenate([[0], np.cumsum(np.maximum(wl.context_lens - 1, 0))])
    kind = wl.cache_dtype

    def one(b):
        L = int(wl.context_lens[b])
        if L <= 0:
            return 0
        nblk = -(-L // bs)
        ids = wl.block_tables[b, :nblk]
        tok = lambda a: a[ids].transpose(0, 2, 1, 3).reshape(nblk * bs, H, -1)[:L]
        tok_s = lambda a: a[ids].transpose(0, 2, 1).reshape(nblk * bs, H)[:L]
        lo, hi = int(starts[b]), int(starts[b + 1])
        kx = np.concatenate([k_hist[lo:hi], k_new[b:b + 1]])
        vx = np.concatenate([v_hist[lo:hi], v_new[b:b + 1]])
        if kind == "int8_kchan":
            kq, kscale = quant.quantize_k_channels(kx, wl.k_chan), None
            vq, vscale = quant.quantize_rows(vx, "int8")
        else:
            kq, kscale = quant.quantize_rows(kx, kind)
            vq, vscale = quant.quantize_rows(vx, kind)
        if kind == "int4":
            kq, vq = quant.pack_int4(kq), quant.pack_int4(vq)
        assert np.array_equal(tok(kc).view(np.uint8), kq.view(np.uint8)), "K codes, seq %d" % b
        assert np.array_equal(tok(vc).view(np.uint8), vq.view(np.uint8)), "V codes, seq %d" % b
        if kscale is not None and ks is not None:
            assert np.array_equal(tok_s(ks).view(np.uint32), kscale.view(np.uint32)), \
                "K scales, seq %d" % b
        if vs is not None and kind != "e5m2_cast":
            assert np.array_equal(tok_s(vs).view(np.uint32), vscale.view(np.uint32)), \
                "V scales, seq %d" % b
        return L * H

    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        rows = sum(ex.map(one, range(wl.batch)))
    if kind == "int8_kchan":
        assert np.array_equal(ks, wl.k_chan)      # the layer's channel scales, untouched
    return rows
