"""The library's prefix cache (C ABI kv_prefix_*, host only) against the
oracle's model, operation by operation: the same prompts stored, matched and
evicted on both, with the oracle pool mirroring the library's block choices."""
import ctypes
import random

import pytest

import paged_kv_cache_440_b200 as pkv
from paged_kv_cache_440_b200 import binding
from oracle.allocator import PoolModel
from oracle.prefix_cache import PrefixCacheModel


FAKE_BASE = 1 << 40  # the pool's memory is never touched by host-only calls


class HostPool(binding.KVPool):
    """A pool descriptor over an address no call dereferences: only its
    allocator is used here, so no GPU is needed."""

    def __init__(self, nblocks, bs):
        self.desc = binding.PoolDesc(1, nblocks, bs, 1, 64, binding.DTYPE_CODES["bf16"])
        n = ctypes.c_uint64()
        binding.check(binding.lib.kv_pool_required_bytes(ctypes.byref(self.desc), ctypes.byref(n)))
        h = ctypes.c_void_p()
        binding.check(binding.lib.kv_pool_create(ctypes.byref(self.desc), ctypes.c_void_p(FAKE_BASE),
                                                 n.value, ctypes.byref(h)))
        self.handle = h


def _pair(nblocks, bs):
    pool = HostPool(nblocks, bs)
    return pool, pkv.PrefixCache(pool), PoolModel(nblocks)


def _refs_equal(pool, model):
    return all(pool.refcount(i) == model.ref[i] for i in range(model.num_blocks))


def test_pages_example_through_the_library():
    """The pages' example behind a 16-token common opening and a tail, so that
    request A fills two whole blocks of 16: B matches the opening and the 6
    shared characters of A's second block (that block comes back as a partial
    match, to be copied before B writes into it)."""
    opening = list(range(1000, 1016))
    a = opening + [ord(c) for c in "你是助手，请回答"] + [7] * 8
    b = opening + [ord(c) for c in "你是助手，请总结"] + [9] * 8
    pool, pc, _ = _pair(16, 16)
    ids = pool.alloc(2)
    assert pc.insert(a, ids) == 2
    pool.free(ids)
    got, n = pc.match(b)
    assert n == 16 + 6 and got == ids
    st = pc.stats()
    assert st["lookups"] == 1 and st["hits"] == 1 and st["hit_tokens"] == 22
    pc.close()
    assert pool.stats()["used"] == 2                 # only the lookup's references remain


@pytest.mark.parametrize("bs", [16, 32])
def test_random_operations_match_the_oracle(bs):
    rng = random.Random(100 + bs)
    nblocks = 400
    pool, pc, mpool = _pair(nblocks, bs)
    model = PrefixCacheModel(mpool, bs)
    prompts, live = [], []
    seen = {"partial": 0, "whole": 0, "evicted": 0}
    for step in range(600):
        op = rng.random()
        if op < 0.4:                                     # a request prefills and caches
            base = rng.choice(prompts) if prompts and rng.random() < 0.8 else []
            p = base[:rng.randint(0, len(base))] + [rng.randint(0, 2) for _ in range(rng.randint(0, 3 * bs))]
            need = -(-len(p) // bs)
            if need > pool.stats()["free"]:
                freed = pc.evict(need)
                assert freed == model.evict(need)
                if need > pool.stats()["free"]:
                    continue
            ids = pool.alloc(need)
            mpool.take(ids)
            assert pc.insert(p, ids) == model.insert(p, ids)
            pool.free(ids)
            mpool.free(ids)
            prompts.append(p)
        elif op < 0.75 and prompts:                      # a lookup, sometimes held a while
            p = rng.choice(prompts)
            p = p[:rng.randint(0, len(p))] + [rng.randint(0, 2) for _ in range(rng.randint(0, bs))]
            got = pc.match(p)
            assert got == model.match(p), (step, p)
            seen["partial" if got[1] % bs else "whole"] += got[1] > 0
            if rng.random() < 0.5:
                live.append(got[0])
            else:
                pool.free(got[0])
                mpool.free(got[0])
        elif op < 0.9:                                   # memory pressure
            k = rng.randint(1, 8)
            freed = pc.evict(k)
            assert freed == model.evict(k)
            seen["evicted"] += len(freed)
        elif live:                                       # a held request finishes
            ids = live.pop(rng.randrange(len(live)))
            pool.free(ids)
            mpool.free(ids)
        if step % 50 == 0:
            assert _refs_equal(pool, mpool)
            st = pc.stats()
            assert st["cached_blocks"] == model.cached_blocks()
            assert (st["lookups"], st["hits"], st["hit_tokens"]) == \
                (model.lookups, model.hits, model.hit_tokens)
        if step == 400:                                  # weights changed: forget everything
            pc.clear()
            model.clear()
    assert _refs_equal(pool, mpool)
    assert min(seen.values()) > 10, seen     # the run exercised every path
    for ids in live:
        pool.free(ids)
        mpool.free(ids)
    pc.close()
    model.clear()
    assert _refs_equal(pool, mpool) and pool.stats()["used"] == 0


def test_validation():
    pool, pc, _ = _pair(8, 16)
    t16, t33 = list(range(16)), list(range(33))
    with pytest.raises(pkv.PagedKVError):
        pc.insert(t16, [5])                             # block 5 is not allocated
    assert pc.stats()["cached_blocks"] == 0
    ids = pool.alloc(1)
    with pytest.raises(pkv.PagedKVError):
        pc.insert(t33, ids)                             # two full blocks, one id
    assert pc.insert(t16 + [99], ids) == 1              # the partial tail is not cached
    assert pc.match(t16 + [99]) == (ids, 16)
