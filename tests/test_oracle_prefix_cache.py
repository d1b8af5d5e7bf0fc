"""Pins for the prefix-cache oracle (oracle/prefix_cache.py): the pages'
worked example, hand-derived LRU orders, and an independent brute force."""
import json
import os
import random

import pytest

from oracle.allocator import PoolModel
from oracle.prefix_cache import PrefixCacheModel

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "prefix_cache_pages.json")


def _cache(bs, nblocks=64):
    pool = PoolModel(nblocks)
    return pool, PrefixCacheModel(pool, bs)


def _store(pool, cache, tokens, bs):
    """A request computes the KV of `tokens` into fresh blocks, caches them and
    finishes (drops its own references)."""
    ids = pool.alloc(-(-len(tokens) // bs))
    cache.insert(tokens, ids)
    pool.free(ids)
    return ids


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: "bs%d" % c["bs"])
def test_pages_radix_example(case):
    g = json.load(open(GOLDEN))
    bs = case["bs"]
    a, b = list(g["a"]), list(g["b"])
    pool, cache = _cache(bs)
    ids = _store(pool, cache, a, bs)
    got, matched = cache.match(b)
    assert matched == g["shared_tokens"] == case["full_blocks"] * bs + case["partial_tokens"]
    nret = case["full_blocks"] + (1 if case["partial_tokens"] else 0)
    assert got == ids[:nret]


def test_only_exact_prefixes_count():
    # a token that changes at the start (a timestamp, a random id) defeats the cache
    bs = 4
    pool, cache = _cache(bs)
    prompt = list(range(100, 140))
    _store(pool, cache, prompt, bs)
    assert cache.match(prompt[:32])[1] == 32
    assert cache.match([7] + prompt[1:])[1] == 0
    # the same tokens further along still match up to the first difference
    changed = prompt[:13] + [999] + prompt[14:]
    assert cache.match(changed)[1] == 13


def test_lru_leaves_go_first_and_shared_prefix_survives():
    bs = 2
    pool, cache = _cache(bs)
    a = _store(pool, cache, [1, 2, 3, 4], bs)        # clock 1: a0 (1,2), a1 (3,4)
    b = pool.alloc(2)
    cache.insert([1, 2, 5, 6], b)                    # clock 2: (1,2) touched, b1 = (5,6) new
    pool.free(b)
    assert cache.cached_blocks() == 3 and pool.ref[b[0]] == 0   # b0 duplicated a0: not kept
    cache.match([1, 2, 3, 4])                        # clock 3: a0, a1 touched
    pool.free(a)                                     # the request that matched finishes
    # leaves: a1 (time 3) and b1 (time 2): b1 goes first, then a1, then the
    # shared block a0 once it has become a leaf
    assert cache.evict(1) == [b[1]]
    assert cache.evict(5) == [a[1], a[0]]
    assert cache.cached_blocks() == 0 and pool.free_count() == 64


def test_blocks_in_use_are_not_evicted():
    bs = 2
    pool, cache = _cache(bs)
    a = _store(pool, cache, [1, 2, 3, 4], bs)
    ids, n = cache.match([1, 2, 3, 4])               # a request holds both blocks
    assert n == 4 and ids == a
    assert cache.evict(10) == []                     # the leaf a1 has refcount 2
    pool.free([ids[1]])                              # the request lets go of a1 only
    assert cache.evict(10) == [a[1]]                 # a0 is in use: it stays
    assert pool.ref[a[0]] == 2


def test_clear_drops_only_the_cache_references():
    bs = 2
    pool, cache = _cache(bs)
    a = _store(pool, cache, [1, 2, 3, 4, 5, 6], bs)
    ids, _ = cache.match([1, 2, 3])                  # holds a0 and (partial) a1
    cache.clear()
    assert cache.cached_blocks() == 0
    assert [pool.ref[x] for x in a] == [1, 1, 0]


def test_partial_match_ties_go_to_the_smallest_block():
    bs = 4
    pool, cache = _cache(bs)
    x = _store(pool, cache, [1, 2, 3, 4, 9, 9, 7, 7], bs)
    y = _store(pool, cache, [1, 2, 3, 4, 9, 9, 8, 8], bs)
    ids, n = cache.match([1, 2, 3, 4, 9, 9, 5, 5])
    assert n == 6 and ids == [x[0], min(x[1], y[1])]


def test_against_brute_force_over_inserted_prompts():
    """With nothing evicted, the full-block part of a match is the longest
    common prefix (in whole blocks) with any inserted prompt's full blocks, and
    the partial part the longest common run into the next block of one of
    them: computed here from the list of prompts, not from the cache."""
    rng = random.Random(3)
    for bs in (1, 2, 3, 4):
        pool, cache = _cache(bs, nblocks=4000)
        prompts = []
        for _ in range(60):
            base = rng.choice(prompts) if prompts and rng.random() < 0.7 else []
            cut = rng.randint(0, len(base))
            p = base[:cut] + [rng.randint(0, 3) for _ in range(rng.randint(0, 12))]
            if rng.random() < 0.5:
                _store(pool, cache, p, bs)
                prompts.append(p)
            else:
                ids, n = cache.match(p)
                full = 0
                for q in prompts:
                    qf = len(q) // bs * bs
                    k = 0
                    while k < min(len(p), qf) and p[k] == q[k]:
                        k += 1
                    full = max(full, k // bs * bs)
                part = 0
                for q in prompts:
                    if len(q) // bs * bs >= full + bs and q[:full] == p[:full]:
                        j = 0
                        while j < bs and full + j < len(p) and q[full + j] == p[full + j]:
                            j += 1
                        part = max(part, j)
                assert n == full + part, (bs, p)
                pool.free(ids)
        # every cached key is a prefix of some inserted prompt
        for key in cache.entries:
            assert any(list(key) == q[:len(key)] for q in prompts)
