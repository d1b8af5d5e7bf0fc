"""Paged decode attention reference (float64).

Test infrastructure only (see ``oracle/__init__``).

Definition followed:
* attention output = softmax(Q K^T / sqrt(d)) V [bjdmk.com.cn/news/6246348, §2.1];
  the scale is an argument (1/sqrt(d) by default);
* at decode step t only the new token's query is evaluated against the cached
  K_1..K_t, V_1..V_t, the new K_t, V_t having been appended to the cache end
  [KV Cache 原理与 PagedAttention, §一 "生成第 t 个 token 时"];
* the cache of one sequence is a list of fixed-size logical blocks, logical block i
  stored in physical block block_table[i], and attention gathers the scattered
  physical blocks back into the logical sequence [same page, §三 "工作方式" 1, 2, 4];
* GQA/MQA: several query heads share one KV head [same page, §一 "GQA / MQA"];
  query head h reads KV head h // (Hq / Hkv) (contiguous groups; the pages do
  not state the map, this is the plain reading).

Cache layout (a reading, the pages fix none): [num_blocks][kv_heads][block_size][D].
Position t of a sequence is row t % block_size of physical block
block_table[t // block_size]. A sequence of length 0 yields a zero output.

No partitioning, no online softmax: the whole row of scores is formed, its maximum
subtracted (softmax is invariant to that shift) and normalised once.
"""
import numpy as np


def gather_sequence(cache, block_table_row, context_len, kv_head, block_size):
    """Gather positions 0..context_len-1 of one KV head into a [L, D] float64 array."""
    t = np.arange(context_len)
    blocks = np.asarray(block_table_row)[t // block_size]
    return np.asarray(cache[blocks, kv_head, t % block_size, :], dtype=np.float64)


def attend(q, K, V, scale):
    """softmax(scale * K q) V for one query vector q [D] over K, V [L, D]."""
    q = np.asarray(q, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    s = scale * (K @ q)
    p = np.exp(s - np.max(s))
    return (p @ V) / np.sum(p)


def decode_one(q, k_cache, v_cache, block_tables, context_lens, scale, b, h):
    """Output of query head h of sequence b, float64 [D]."""
    Hq = q.shape[1]
    Hkv = k_cache.shape[1]
    bs = k_cache.shape[2]
    g = h // (Hq // Hkv)
    L = int(context_lens[b])
    K = gather_sequence(k_cache, block_tables[b], L, g, bs)
    V = gather_sequence(v_cache, block_tables[b], L, g, bs)
    return attend(q[b, h], K, V, scale)


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale):
    """Decode attention for every (sequence, query head).

    q [B, Hq, D]; k_cache, v_cache [NB, Hkv, bs, D] (real values, any precision);
    block_tables [B, max_blocks] int; context_lens [B] int; scale float.
    Returns float64 [B, Hq, D].
    """
    B, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("query heads must be a multiple of kv heads")
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            out[b, h] = decode_one(q, k_cache, v_cache, block_tables, context_lens, scale, b, h)
    return out


def prefill_one(q_vec, k_cache, v_cache, table_row, pos, kv_head, scale):
    """Output for one query at position `pos` of a sequence: it attends to
    positions 0..pos, each token seeing every token before it and itself
    [KV Cache 原理与 PagedAttention, §一: token t attends to tokens 1..t]."""
    bs = k_cache.shape[2]
    K = gather_sequence(k_cache, table_row, pos + 1, kv_head, bs)
    V = gather_sequence(v_cache, table_row, pos + 1, kv_head, bs)
    return attend(q_vec, K, V, scale)


def paged_prefill(q, cu_q, k_cache, v_cache, block_tables, context_lens, scale):
    """Chunked prefill over the paged cache: sequence b's new tokens are the
    last c_b = cu_q[b+1] - cu_q[b] of its context_lens[b] positions (their K/V
    already in the cache, behind a prefix that may come from a prefix cache
    [bjdmk.com.cn/news/6246348, §4.1: the cached prefix's prefill is
    skipped]); new token i sits at position context_lens[b] - c_b + i.

    q [T, Hq, D] with T = cu_q[-1] (sequence-major); returns float64 [T, Hq, D].
    """
    T, Hq, D = q.shape
    Hkv = k_cache.shape[1]
    G = Hq // Hkv
    out = np.zeros((T, Hq, D), dtype=np.float64)
    for b in range(len(cu_q) - 1):
        c = int(cu_q[b + 1] - cu_q[b])
        L = int(context_lens[b])
        for i in range(c):
            pos = L - c + i
            for h in range(Hq):
                out[cu_q[b] + i, h] = prefill_one(q[cu_q[b] + i, h], k_cache, v_cache,
                                                  block_tables[b], pos, h // G, scale)
    return out
