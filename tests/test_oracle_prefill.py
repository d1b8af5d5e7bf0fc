"""Pins for the chunked-prefill oracle (oracle.attention.paged_prefill)."""
import math

import numpy as np
import torch

from oracle import attention


def _case(rng, B=3, Hq=4, Hkv=2, D=8, bs=4, lens=(9, 5, 12), chunks=(4, 5, 1)):
    nb_needed = sum(-(-L // bs) for L in lens)
    NB = nb_needed + 3
    perm = rng.permutation(NB)
    tables = np.full((B, max(-(-L // bs) for L in lens)), -1, np.int64)
    k = 0
    for b, L in enumerate(lens):
        n = -(-L // bs)
        tables[b, :n] = perm[k:k + n]
        k += n
    kc = rng.standard_normal((NB, Hkv, bs, D))
    vc = rng.standard_normal((NB, Hkv, bs, D))
    cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int64)
    q = rng.standard_normal((int(cu[-1]), Hq, D))
    return q, cu, kc, vc, tables, np.array(lens), 0.35


def test_last_chunk_token_is_the_decode_output():
    rng = np.random.default_rng(1)
    q, cu, kc, vc, tables, lens, scale = _case(rng)
    out = attention.paged_prefill(q, cu, kc, vc, tables, lens, scale)
    for b in range(len(lens)):
        qd = q[cu[b + 1] - 1][None].repeat(len(lens), 0)
        for h in range(q.shape[1]):
            ref = attention.decode_one(qd, kc, vc, tables, lens, scale, b, h)
            np.testing.assert_allclose(out[cu[b + 1] - 1, h], ref, rtol=0, atol=1e-15)


def test_first_position_returns_its_value():
    rng = np.random.default_rng(2)
    q, cu, kc, vc, tables, lens, scale = _case(rng, lens=(3,), chunks=(3,), B=1)
    out = attention.paged_prefill(q, cu, kc, vc, tables, lens, scale)
    bs, G = kc.shape[2], q.shape[1] // kc.shape[1]
    for h in range(q.shape[1]):
        np.testing.assert_array_equal(out[0, h], vc[tables[0, 0], h // G, 0])


def test_causality():
    rng = np.random.default_rng(3)
    q, cu, kc, vc, tables, lens, scale = _case(rng)
    out = attention.paged_prefill(q, cu, kc, vc, tables, lens, scale)
    bs = kc.shape[2]
    b, L = 0, int(lens[0])
    c = int(cu[1] - cu[0])
    pos = L - c + 1                              # the chunk's second token
    t = pos + 1                                  # a later position of the same sequence
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[tables[b, t // bs], :, t % bs] += 5.0
    vc2[tables[b, t // bs], :, t % bs] -= 3.0
    out2 = attention.paged_prefill(q, cu, kc2, vc2, tables, lens, scale)
    np.testing.assert_array_equal(out2[cu[0] + 1], out[cu[0] + 1])      # unchanged
    assert np.abs(out2[cu[0] + 2] - out[cu[0] + 2]).max() > 1e-3         # it sees t


def test_brute_force_with_fsum():
    rng = np.random.default_rng(4)
    q, cu, kc, vc, tables, lens, scale = _case(rng, lens=(7, 10), chunks=(3, 10), B=2)
    out = attention.paged_prefill(q, cu, kc, vc, tables, lens, scale)
    bs, Hq, D = kc.shape[2], q.shape[1], q.shape[2]
    G = Hq // kc.shape[1]
    for b in range(2):
        c, L = int(cu[b + 1] - cu[b]), int(lens[b])
        for i in range(c):
            pos = L - c + i
            for h in range(Hq):
                keys = [kc[tables[b, t // bs], h // G, t % bs] for t in range(pos + 1)]
                vals = [vc[tables[b, t // bs], h // G, t % bs] for t in range(pos + 1)]
                s = [scale * math.fsum(q[cu[b] + i, h, d] * kk[d] for d in range(D)) for kk in keys]
                m = max(s)
                w = [math.exp(x - m) for x in s]
                tot = math.fsum(w)
                ref = [math.fsum(w[t] * vals[t][d] for t in range(pos + 1)) / tot for d in range(D)]
                np.testing.assert_allclose(out[cu[b] + i, h], ref, rtol=1e-12, atol=1e-12)


def test_against_torch_sdpa_with_a_causal_mask():
    rng = np.random.default_rng(5)
    q, cu, kc, vc, tables, lens, scale = _case(rng, B=1, lens=(13,), chunks=(6,), Hq=8, Hkv=2)
    out = attention.paged_prefill(q, cu, kc, vc, tables, lens, scale)
    bs, G = kc.shape[2], 4
    L, c = 13, 6
    K = np.stack([attention.gather_sequence(kc, tables[0], L, g, bs) for g in range(2)])
    V = np.stack([attention.gather_sequence(vc, tables[0], L, g, bs) for g in range(2)])
    Kt = torch.from_numpy(K).repeat_interleave(G, 0)           # [Hq, L, D]
    Vt = torch.from_numpy(V).repeat_interleave(G, 0)
    Qt = torch.from_numpy(q.transpose(1, 0, 2).copy())         # [Hq, c, D]
    mask = torch.arange(L)[None, :] <= (L - c + torch.arange(c))[:, None]
    ref = torch.nn.functional.scaled_dot_product_attention(Qt, Kt, Vt, attn_mask=mask, scale=scale)
    np.testing.assert_allclose(out, ref.numpy().transpose(1, 0, 2), rtol=1e-12, atol=1e-12)
