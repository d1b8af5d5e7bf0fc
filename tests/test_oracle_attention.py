"""Pins for the attention oracle, against things other than itself.

* brute force: explicit Python loops with math.fsum over a cache laid out by an
  independent writer;
* an independent library routine: torch's scaled_dot_product_attention in fp64
  on the contiguous sequence (softmax(Q K^T * scale) V, the pages' definition);
* closed forms: one token returns its V; constant V returns V; q = 0 or scale = 0
  gives the mean of V; two tokens give a logistic mix;
* invariants: physical placement does not matter (the sequence is logically
  contiguous); heads of one GQA group with equal queries give equal outputs.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention


def _scatter(seqs_k, seqs_v, kv_heads, bs, num_blocks, rng):
    """Lay contiguous per-sequence K/V [L, Hkv, D] into a paged cache.

    Written independently of the oracle: walks blocks, not positions.
    """
    D = seqs_k[0].shape[-1] if seqs_k else 1
    kc = rng.standard_normal((num_blocks, kv_heads, bs, D)) * 100.0   # junk elsewhere
    vc = rng.standard_normal((num_blocks, kv_heads, bs, D)) * 100.0
    need = [-(-k.shape[0] // bs) for k in seqs_k]
    perm = rng.permutation(num_blocks)
    mb = max(1, max(need))
    tables = np.full((len(seqs_k), mb), -1, dtype=np.int64)
    used = 0
    for b, (K, V) in enumerate(zip(seqs_k, seqs_v)):
        for i in range(need[b]):
            blk = perm[used]
            used += 1
            tables[b, i] = blk
            for r in range(bs):
                pos = i * bs + r
                if pos < K.shape[0]:
                    for g in range(kv_heads):
                        kc[blk, g, r] = K[pos, g]
                        vc[blk, g, r] = V[pos, g]
    return kc, vc, tables


def _brute(q, K, V, scale):
    """softmax(scale q.K_t) V with scalar loops and exactly-rounded sums."""
    L = len(K)
    if L == 0:
        return [0.0] * len(V[0]) if V else []
    s = [scale * math.fsum(qi * ki for qi, ki in zip(q, K[t])) for t in range(L)]
    m = max(s)
    p = [math.exp(x - m) for x in s]
    z = math.fsum(p)
    D = len(V[0])
    return [math.fsum(p[t] * V[t][d] for t in range(L)) / z for d in range(D)]


def _random_problem(rng, lens, Hq, Hkv, D, bs, slack=3):
    kseq = [rng.standard_normal((L, Hkv, D)) for L in lens]
    vseq = [rng.standard_normal((L, Hkv, D)) for L in lens]
    nb = sum(-(-L // bs) for L in lens) * slack + 1
    kc, vc, tables = _scatter(kseq, vseq, Hkv, bs, nb, rng)
    q = rng.standard_normal((len(lens), Hq, D))
    return q, kseq, vseq, kc, vc, tables


@pytest.mark.parametrize("lens,Hq,Hkv,bs", [
    ([1, 7, 16, 17, 40], 4, 2, 4),
    ([33, 2], 2, 1, 8),
    ([5, 31], 3, 3, 16),
])
def test_matches_brute_force(lens, Hq, Hkv, bs):
    rng = np.random.default_rng(1)
    D = 8
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, lens, Hq, Hkv, D, bs)
    scale = 0.37
    out = attention.paged_decode(q, kc, vc, tables, np.array(lens), scale)
    G = Hq // Hkv
    for b, L in enumerate(lens):
        for h in range(Hq):
            g = h // G
            K = [list(kseq[b][t, g]) for t in range(L)]
            V = [list(vseq[b][t, g]) for t in range(L)]
            ref = _brute(list(q[b, h]), K, V, scale)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-12)


def test_matches_torch_sdpa_fp64():
    """Independent library path: torch SDPA on the contiguous sequence, GQA by
    repeating each KV head over its group of query heads."""
    rng = np.random.default_rng(2)
    lens = [250, 17, 100, 33]
    Hq, Hkv, D, bs = 8, 2, 64, 16
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, lens, Hq, Hkv, D, bs)
    scale = 0.125
    out = attention.paged_decode(q, kc, vc, tables, np.array(lens), scale)
    for b, L in enumerate(lens):
        Kt = torch.from_numpy(kseq[b]).permute(1, 0, 2)          # [Hkv, L, D]
        Vt = torch.from_numpy(vseq[b]).permute(1, 0, 2)
        Kt = Kt.repeat_interleave(Hq // Hkv, dim=0)               # [Hq, L, D]
        Vt = Vt.repeat_interleave(Hq // Hkv, dim=0)
        qt = torch.from_numpy(q[b])[:, None, :]                   # [Hq, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
        np.testing.assert_allclose(out[b], ref[:, 0, :].numpy(), rtol=1e-12, atol=1e-12)


def test_placement_permutation_is_bit_identical():
    rng = np.random.default_rng(3)
    lens = [40, 9, 64]
    Hq, Hkv, D, bs = 4, 2, 8, 16
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, lens, Hq, Hkv, D, bs)
    out1 = attention.paged_decode(q, kc, vc, tables, np.array(lens), 0.5)
    perm = rng.permutation(kc.shape[0])                 # new physical id of block i
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1)
    out2 = attention.paged_decode(q, kc2, vc2, tables2, np.array(lens), 0.5)
    assert np.array_equal(out1, out2)


def test_single_token_returns_its_value():
    rng = np.random.default_rng(4)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [1, 1], 4, 2, 8, 16)
    out = attention.paged_decode(q, kc, vc, tables, np.array([1, 1]), 3.0)
    for b in range(2):
        for h in range(4):
            assert np.array_equal(out[b, h], vseq[b][0, h // 2])


def test_constant_value_returns_it():
    rng = np.random.default_rng(5)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [37], 2, 1, 8, 16)
    c = rng.standard_normal(8)
    vc[:] = c
    out = attention.paged_decode(q, kc, vc, tables, np.array([37]), 0.9)
    np.testing.assert_allclose(out[0, 0], c, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(out[0, 1], c, rtol=1e-14, atol=1e-15)


@pytest.mark.parametrize("zero", ["q", "scale"])
def test_uniform_softmax_is_mean(zero):
    rng = np.random.default_rng(6)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [50], 2, 2, 8, 16)
    scale = 0.7
    if zero == "q":
        q[:] = 0.0
    else:
        scale = 0.0
    out = attention.paged_decode(q, kc, vc, tables, np.array([50]), scale)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], vseq[0][:, h].mean(axis=0), rtol=1e-13, atol=1e-14)


def test_two_tokens_logistic():
    rng = np.random.default_rng(7)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [2], 1, 1, 8, 16)
    scale = 0.3
    out = attention.paged_decode(q, kc, vc, tables, np.array([2]), scale)
    s0 = scale * float(q[0, 0] @ kseq[0][0, 0])
    s1 = scale * float(q[0, 0] @ kseq[0][1, 0])
    w0 = 1.0 / (1.0 + math.exp(s1 - s0))
    ref = w0 * vseq[0][0, 0] + (1.0 - w0) * vseq[0][1, 0]
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-13, atol=1e-14)


def test_equal_queries_in_a_group_give_equal_outputs():
    rng = np.random.default_rng(8)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [45, 3], 8, 2, 8, 4)
    q[:, 1] = q[:, 0]
    q[:, 6] = q[:, 4]
    out = attention.paged_decode(q, kc, vc, tables, np.array([45, 3]), 0.25)
    assert np.array_equal(out[:, 1], out[:, 0])
    assert np.array_equal(out[:, 6], out[:, 4])
    # and a head of the other group, given the same query, differs
    q2 = q.copy()
    q2[:, 4] = q2[:, 0]
    out2 = attention.paged_decode(q2, kc, vc, tables, np.array([45, 3]), 0.25)
    assert not np.allclose(out2[0, 4], out2[0, 0])


def test_empty_sequence_is_zero():
    rng = np.random.default_rng(9)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [5, 6], 2, 1, 8, 4)
    out = attention.paged_decode(q, kc, vc, tables, np.array([0, 6]), 0.5)
    assert np.array_equal(out[0], np.zeros((2, 8)))


def test_ignores_rows_past_the_context_length():
    """The tail of the last block and unused table entries are never read."""
    rng = np.random.default_rng(10)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [21], 2, 1, 8, 16)
    out1 = attention.paged_decode(q, kc, vc, tables, np.array([21]), 0.5)
    kc[tables[0, 1], :, 5:] = np.nan
    vc[tables[0, 1], :, 5:] = np.nan
    out2 = attention.paged_decode(q, kc, vc, tables, np.array([21]), 0.5)
    assert np.array_equal(out1, out2)


def test_large_scores_stay_finite_and_pick_the_dominant_token():
    """Scores spanning thousands: exp must be taken relative to the row maximum.
    With one score above the rest by > 800 the output is exactly that token's V
    (every other weight underflows to 0 in float64)."""
    rng = np.random.default_rng(11)
    q, kseq, vseq, kc, vc, tables = _random_problem(rng, [30], 1, 1, 8, 16)
    K = kseq[0][:, 0]
    q[0, 0] = K[17] * 1000.0 / float(K[17] @ K[17])     # q.K_17 = 1000
    # every other key is zeroed, so its score is 0 and the margin is 1000
    for t in range(30):
        if t != 17:
            kc[tables[0, t // 16], 0, t % 16] *= 0.0
    out = attention.paged_decode(q, kc, vc, tables, np.array([30]), 1.0)
    assert np.all(np.isfinite(out))
    assert np.array_equal(out[0, 0], vseq[0][17, 0])
