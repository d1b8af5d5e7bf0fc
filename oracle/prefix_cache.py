"""Reference model of a prefix cache over the paged KV pool.

Test infrastructure only (see ``oracle/__init__``).

What it models [bjdmk.com.cn/news/6246348, §4.1, §4.2; KV Cache 原理与
PagedAttention, §五]:

* Requests whose prompts start with the same tokens can reuse the KV blocks
  already computed for that prefix instead of recomputing it. KV depends on
  the token and its position, so only an exact prefix counts (§4.3).
* The cached prefixes form a tree: a new prompt takes the longest cached
  prefix, including a partial match inside a block, and the blocks it adds
  extend the tree.
* Under memory pressure the least recently used leaves go first, so a hot
  shared prefix outlives the private tails hanging off it.
* A change of model weights invalidates everything (``clear``).

This model is the plain definition, not a tree: the cache is a dict from
every cached full-block prefix ``tuple(tokens[:k * bs])`` to the block holding
its k-th block and that block's last access time. The set is prefix-closed.
A "leaf" is a key that no other key extends by one block.

Readings (the pages give none of these details):

* One clock tick per operation; every block a match or insert touches gets
  that tick.
* A partial match is the block, among the one-block extensions of the matched
  full-block prefix, sharing the most leading tokens (at least one) with the
  rest of the prompt; ties go to the smallest block id.
* The cache holds one pool reference per cached block; a match takes one more
  per returned block on the caller's behalf.
* Eviction picks the leaf with the smallest (last access, block id) among
  leaves whose block is held by the cache alone (pool refcount 1), drops the
  cache's reference (freeing the block) and repeats.
"""


class PrefixCacheModel:
    def __init__(self, pool, block_size):
        self.pool = pool            # oracle.allocator.PoolModel
        self.bs = block_size
        self.entries = {}           # prefix tuple -> [block id, last access]
        self.clock = 0
        self.lookups = 0
        self.hits = 0
        self.hit_tokens = 0

    def cached_blocks(self):
        return len(self.entries)

    def _extensions(self, prefix):
        n = len(prefix) + self.bs
        return [k for k in self.entries if len(k) == n and k[:len(prefix)] == prefix]

    def match(self, tokens):
        """Longest cached prefix of ``tokens``: (block ids, matched tokens).
        The last id may be a block matched only in part; the caller copies it
        before writing. One reference per returned id goes to the caller."""
        tokens = tuple(tokens)
        self.clock += 1
        bs, n = self.bs, len(tokens)
        ids, k = [], 0
        while (k + 1) * bs <= n and tokens[:(k + 1) * bs] in self.entries:
            e = self.entries[tokens[:(k + 1) * bs]]
            e[1] = self.clock
            ids.append(e[0])
            k += 1
        matched = k * bs
        if matched < n:
            best = None
            for key in self._extensions(tokens[:matched]):
                j = 0
                while j < bs and matched + j < n and key[matched + j] == tokens[matched + j]:
                    j += 1
                blk = self.entries[key][0]
                if j >= 1 and (best is None or j > best[0] or (j == best[0] and blk < best[1])):
                    best = (j, blk, key)
            if best is not None:
                self.entries[best[2]][1] = self.clock
                ids.append(best[1])
                matched += best[0]
        self.pool.share(ids)
        self.lookups += 1
        self.hits += matched > 0
        self.hit_tokens += matched
        return ids, matched

    def insert(self, tokens, block_ids):
        """Record that the full blocks of ``tokens`` are held in ``block_ids``
        (one id per full block; a trailing partial block is not cached).
        Returns how many blocks became newly cached."""
        tokens = tuple(tokens)
        nfull = len(tokens) // self.bs
        for i in range(nfull):
            if self.pool.ref[block_ids[i]] < 1:
                raise ValueError("block %d is not allocated" % block_ids[i])
        self.clock += 1
        new = 0
        for i in range(nfull):
            key = tokens[:(i + 1) * self.bs]
            if key in self.entries:
                self.entries[key][1] = self.clock
            else:
                self.entries[key] = [block_ids[i], self.clock]
                self.pool.share([block_ids[i]])
                new += 1
        return new

    def evict(self, want):
        """Free up to ``want`` blocks held by the cache alone, least recently
        used leaves first. Returns the freed ids in eviction order."""
        freed = []
        while len(freed) < want:
            leaves = [k for k in self.entries if not self._extensions(k)]
            cands = [k for k in leaves if self.pool.ref[self.entries[k][0]] == 1]
            if not cands:
                break
            key = min(cands, key=lambda k: (self.entries[k][1], self.entries[k][0]))
            blk = self.entries.pop(key)[0]
            self.pool.free([blk])
            freed.append(blk)
        return freed

    def clear(self):
        """Drop every cached prefix (e.g. after a model weight update)."""
        for blk, _ in self.entries.values():
            self.pool.free([blk])
        self.entries = {}
