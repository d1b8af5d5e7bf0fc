"""Append (reshape_and_cache), copy-on-write block copy and quantize-on-append.

Test infrastructure only (see ``oracle/__init__``).

* Append: each decode step computes only the new token's K_t, V_t and puts them at
  the end of the cache [KV Cache 原理与 PagedAttention, §一 "生成第 t 个 token 时";
  bjdmk.com.cn/news/6246348, §2.1]. In a paged cache the end of a sequence is a
  row of some physical block; the caller names it with a slot index
  slot = physical_block * block_size + row (a reading: the pages give no encoding).
  A negative slot means "no token" and is skipped.
* Copy-on-write: before a request writes into a block other requests share, the
  block is copied and the writer's block table repointed to the copy
  [bjdmk.com.cn/news/6246348, §3.2; KV Cache 原理与 PagedAttention, §三 收益 table,
  last row]. The copy is of the whole block: K, V and, for quantized caches, the
  per-token-head scales, in every layer.

All arrays here are raw bit patterns (e.g. uint16 views of bf16/fp16, uint8 codes,
uint32 views of fp32 scales) so that the copies are byte-exact.
"""
import numpy as np

from . import quant


def append(k_cache, v_cache, k_new, v_new, slot_mapping, block_size):
    """In place: cache[slot // bs, :, slot % bs, :] = new[i] for every slot >= 0.

    k_cache, v_cache [NB, Hkv, bs, D]; k_new, v_new [T, Hkv, D]; slot_mapping [T].
    Tokens are written in index order, so for a repeated slot the last one wins.
    """
    for i, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        blk, row = divmod(int(slot), block_size)
        k_cache[blk, :, row, :] = k_new[i]
        v_cache[blk, :, row, :] = v_new[i]


def append_quantized(k_codes, v_codes, k_scales, v_scales, k_new, v_new,
                     slot_mapping, block_size, kind):
    """Quantize each new (token, head) row, then place codes and scales by slot.

    k_codes, v_codes [NB, Hkv, bs, D] ([..., D/2] packed bytes for INT4);
    k_scales, v_scales [NB, Hkv, bs] float32;
    k_new, v_new [T, Hkv, D] float32-representable values.
    """
    kc, ks = quant.quantize_rows(k_new, kind)
    vc, vs = quant.quantize_rows(v_new, kind)
    if kind == "int4":                    # the cache holds two codes per byte
        kc, vc = quant.pack_int4(kc), quant.pack_int4(vc)
    for i, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        blk, row = divmod(int(slot), block_size)
        k_codes[blk, :, row, :] = kc[i]
        v_codes[blk, :, row, :] = vc[i]
        k_scales[blk, :, row] = ks[i]
        v_scales[blk, :, row] = vs[i]


def append_quantized_kchan(k_codes, v_codes, v_scales, k_new, v_new, slot_mapping,
                           block_size, chan_scales):
    """As append_quantized for INT8 keys with per-channel scales: K rows are
    quantized with the layer's fixed [Hkv, D] channel scales
    (quant.quantize_k_channels), V rows per token and head (INT8 absmax).

    k_codes, v_codes [NB, Hkv, bs, D] int8; v_scales [NB, Hkv, bs] float32.
    """
    kc = quant.quantize_k_channels(k_new, chan_scales)
    vc, vs = quant.quantize_rows(v_new, "int8")
    for i, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        blk, row = divmod(int(slot), block_size)
        k_codes[blk, :, row, :] = kc[i]
        v_codes[blk, :, row, :] = vc[i]
        v_scales[blk, :, row] = vs[i]


def block_copy(arrays, pairs):
    """In place: for each (src, dst) pair, every array's block dst := block src.

    arrays: iterable of arrays indexed [block, ...] (one per layer and per K / V /
    K-scale / V-scale region). pairs: [(src, dst), ...], applied in order.
    """
    for src, dst in pairs:
        for a in arrays:
            a[dst] = a[src]
