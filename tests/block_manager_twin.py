"""A Python restatement of the host block allocator, for the tests only.

The library's own allocator is the C ABI's pa_alloc_* (the workload builders
in paged_kv_cache_458_b200.gen drive it).  This twin is written from the same
description (a stack free list, reference counts, copy-on-write of a shared
last block; zingnex.cn, "vLLM与PagedAttention深度剖析", section 3.2 items 1-4)
and the tests run random operation sequences through both and compare every
table, slot, copy pair and reference count.
"""
import numpy as np


class BlockManager:
    """Free list + reference counts + per-sequence block tables.

    The free list is a stack: it starts as ``order`` with ``order[0]`` on top,
    and a block whose reference count drops to zero is pushed back on top, so
    the next allocation reuses it (the pool reuse of zingnex.cn section 3.2,
    item 4).  ``append_slot`` allocates only when a token crosses into a new
    block (item 1) and copies a shared last block before writing to it
    (item 3, copy-on-write).
    """

    def __init__(self, num_blocks: int, block_size: int, order=None):
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = np.arange(num_blocks) if order is None else np.asarray(order)
        assert sorted(order.tolist()) == list(range(num_blocks))
        self.free = [int(b) for b in order[::-1]]
        self.ref = np.zeros(num_blocks, dtype=np.int64)
        self.tables: dict[int, list[int]] = {}
        self.lens: dict[int, int] = {}
        self.peak_used = 0

    # -- primitives
    def used(self) -> int:
        return self.num_blocks - len(self.free)

    def alloc(self) -> int:
        if not self.free:
            raise MemoryError("block pool exhausted")
        b = self.free.pop()
        assert self.ref[b] == 0
        self.ref[b] = 1
        self.peak_used = max(self.peak_used, self.used())
        return b

    def release(self, b: int) -> None:
        assert self.ref[b] > 0
        self.ref[b] -= 1
        if self.ref[b] == 0:
            self.free.append(b)

    # -- sequence operations
    def add_seq(self, seq: int, n_tokens: int) -> None:
        assert seq not in self.tables
        self.tables[seq] = []
        self.lens[seq] = 0
        self.extend(seq, n_tokens)

    def extend(self, seq: int, n_tokens: int) -> None:
        """Grow a sequence by ``n_tokens`` (prefill): blocks on demand, no CoW."""
        tab = self.tables[seq]
        L = self.lens[seq] + n_tokens
        while len(tab) * self.block_size < L:
            tab.append(self.alloc())
        self.lens[seq] = L

    def fork(self, parent: int, child: int) -> None:
        """``child`` shares every block of ``parent`` (refcount + 1 each)."""
        assert child not in self.tables
        tab = list(self.tables[parent])
        for b in tab:
            self.ref[b] += 1
        self.tables[child] = tab
        self.lens[child] = self.lens[parent]

    def free_seq(self, seq: int) -> None:
        # last block first, so the sequence's first block ends on top of the stack
        for b in reversed(self.tables.pop(seq)):
            self.release(b)
        del self.lens[seq]

    def append_slot(self, seq: int):
        """Reserve the slot of the next token of ``seq``.

        Returns ``(slot, pair)`` where ``pair`` is ``(src, dst)`` when the last
        block was shared and had to be copied first, else ``None``.
        """
        tab = self.tables[seq]
        L = self.lens[seq]
        off = L % self.block_size
        pair = None
        if off == 0:
            b = self.alloc()
            tab.append(b)
        else:
            b = tab[-1]
            if self.ref[b] > 1:
                nb = self.alloc()
                pair = (b, nb)
                self.release(b)
                tab[-1] = nb
                b = nb
        self.lens[seq] = L + 1
        return b * self.block_size + off, pair

    def table_array(self, seqs, max_blocks: int) -> np.ndarray:
        t = np.full((len(seqs), max_blocks), -1, dtype=np.int32)
        for i, s in enumerate(seqs):
            tab = self.tables[s]
            assert len(tab) <= max_blocks
            t[i, :len(tab)] = tab
        return t

    def lens_array(self, seqs) -> np.ndarray:
        return np.array([self.lens[s] for s in seqs], dtype=np.int32)
