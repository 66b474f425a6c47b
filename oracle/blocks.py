"""Reference model of shared cache blocks: block copies and a reference-counted
block pool.

TEST INFRASTRUCTURE (same rules as the rest of ``oracle/``): only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it.

The Tiny-Infer page ("从零构建CUDA推理引擎：Tiny-Infer项目的技术深度解析",
section "分页KV缓存：借鉴操作系统的内存管理") plans vLLM-style block copying so
that sequences sampled in parallel from one prompt can share the prompt's
physical blocks; the vLLM page's section 1 names the block manager beside the
paged cache.  Neither page fixes an interface, so this module states the plain
reading:

* a block copy is a bytewise copy of one whole physical block (all kv heads,
  all rows) to another, in every pool (K and V; INT8 codes and scales);
* a block is free (count 0) or held by ``count`` sequences; allocation takes
  free blocks and gives them count 1, sharing adds a holder, releasing drops
  one and frees the block at 0;
* before a holder writes into a block it calls copy-on-write: a block with one
  holder is written in place; a shared block is copied to a fresh block for the
  writer, which drops its hold on the shared one.

Every operation is all-or-nothing: one that cannot complete changes nothing.
Which free block an allocation returns is a policy, not part of the method; the
model keeps a stack (a fresh pool hands out the lowest ids first, a freed block
is reused first) so that a run of operations has one expected result.
"""
from __future__ import annotations

import numpy as np


def copy_blocks(pools, pairs) -> int:
    """For each (src, dst) row of ``pairs`` copy block ``src`` to block ``dst``
    in every pool of ``pools`` (NumPy arrays indexed by block on axis 0).  Rows
    with an id outside the pool are skipped; the count of skipped rows is
    returned so a caller can check the error report."""
    pairs = np.asarray(pairs, dtype=np.int64).reshape(-1, 2)
    skipped = 0
    nb = pools[0].shape[0]
    for src, dst in pairs:
        if not (0 <= src < nb and 0 <= dst < nb):
            skipped += 1
            continue
        for pool in pools:
            pool[dst] = pool[src]
    return skipped


class BlockPool:
    """Pure-Python reference-counted pool of ``num_blocks`` physical blocks."""

    def __init__(self, num_blocks: int):
        if num_blocks < 0:
            raise ValueError("num_blocks must be >= 0")
        self.count = [0] * num_blocks
        self.free = list(range(num_blocks - 1, -1, -1))   # top of the stack = last element

    def _live(self, b: int) -> bool:
        return 0 <= b < len(self.count) and self.count[b] > 0

    def num_free(self) -> int:
        return len(self.free)

    def refcount(self, b: int) -> int:
        return self.count[b] if 0 <= b < len(self.count) else -1

    def alloc(self, n: int):
        """n fresh blocks with count 1, or None (nothing taken) if fewer are free."""
        if n < 0 or n > len(self.free):
            return None
        out = []
        for _ in range(n):
            b = self.free.pop()
            self.count[b] = 1
            out.append(b)
        return out

    def share(self, ids) -> bool:
        if not all(self._live(b) for b in ids):
            return False
        for b in ids:
            self.count[b] += 1
        return True

    def release(self, ids) -> bool:
        need = {}
        for b in ids:
            need[b] = need.get(b, 0) + 1
        if not all(0 <= b < len(self.count) and self.count[b] >= k for b, k in need.items()):
            return False
        for b in ids:
            self.count[b] -= 1
            if self.count[b] == 0:
                self.free.append(b)
        return True

    def cow(self, b: int):
        """(block to write into, must_copy) or None (nothing changed)."""
        if not self._live(b):
            return None
        if self.count[b] == 1:
            return b, False
        if not self.free:
            return None
        nb = self.free.pop()
        self.count[nb] = 1
        self.count[b] -= 1
        return nb, True

    def check(self) -> None:
        """Invariants: counts are >= 0, the free blocks are exactly those with
        count 0, each listed once."""
        assert all(c >= 0 for c in self.count)
        assert len(set(self.free)) == len(self.free)
        assert set(self.free) == {b for b, c in enumerate(self.count) if c == 0}
