"""Reference model of the KV block pool with reference counts.

Test infrastructure only (see ``oracle/__init__``).

* The pool preallocates fixed-size physical blocks, hands them to sequences on
  demand and takes them back when done, like RAM pages
  [KV Cache 原理与 PagedAttention, §三 "工作方式" 3; aiworkagent.org q17,
  "KV Memory Pool"].
* Sequences with a common prefix point their block tables at the same physical
  blocks; a write to a shared block first copies it (copy-on-write), as fork()
  shares pages [bjdmk.com.cn/news/6246348, §3.1, §3.2].

The model tracks a refcount per block: alloc sets it to 1, share adds 1, free
subtracts 1 (returning the block to the pool at 0). ``cow`` on a block with
refcount > 1 takes a fresh block for the writer and drops one reference from the
shared block; on an exclusively owned block it is the block itself. Which free
id is handed out is not part of the contract; ``alloc`` here takes the lowest.
"""


class PoolModel:
    def __init__(self, num_blocks):
        self.num_blocks = num_blocks
        self.ref = [0] * num_blocks

    def free_count(self):
        return sum(1 for r in self.ref if r == 0)

    def used_count(self):
        return self.num_blocks - self.free_count()

    def shared_count(self):
        return sum(1 for r in self.ref if r > 1)

    def alloc(self, n):
        """Return n fresh block ids or None (out of memory, nothing taken)."""
        if n < 0:
            raise ValueError("negative count")
        free = [i for i, r in enumerate(self.ref) if r == 0]
        if len(free) < n:
            return None
        ids = free[:n]
        for i in ids:
            self.ref[i] = 1
        return ids

    def take(self, ids):
        """Mark specific fresh ids as allocated (mirrors another allocator's choice)."""
        for i in ids:
            if self.ref[i] != 0:
                raise ValueError("block %d is not free" % i)
            self.ref[i] = 1

    def free(self, ids):
        for i in ids:
            if not (0 <= i < self.num_blocks) or self.ref[i] == 0:
                raise ValueError("block %d is not allocated" % i)
        for i in ids:
            self.ref[i] -= 1

    def share(self, ids):
        for i in ids:
            if not (0 <= i < self.num_blocks) or self.ref[i] == 0:
                raise ValueError("block %d is not allocated" % i)
        for i in ids:
            self.ref[i] += 1

    def cow_needed(self, block):
        return self.ref[block] > 1
