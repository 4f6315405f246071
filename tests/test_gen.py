"""The seeded input generator: shapes, block structure, poisoning (no GPU)."""
import numpy as np
import pytest

import block_manager_twin
from paged_kv_cache_458_b200 import gen, pa


def test_tiny_workload_matches_its_statement():
    c = gen.make_case("tiny", n_steps=1)
    assert (c.num_seqs, c.num_q_heads, c.num_kv_heads, c.head_dim, c.block_size) == (4, 4, 4, 64, 16)
    assert c.num_blocks == 32 and c.dtype == gen.F16
    assert c.context_lens.tolist() == [1, 15, 16, 37]
    assert c.steps[0].context_lens.tolist() == [2, 16, 17, 38]
    assert c.scale == pytest.approx(1 / 8)
    # every sequence owns distinct blocks, allocated in the seeded permutation's order
    order = c.structure["pool_order"]
    used = [b for s in range(4) for b in c.block_tables[s] if b >= 0]
    assert used == list(order[:len(used)])
    assert len(set(used)) == len(used) == 1 + 1 + 1 + 3
    # 16 -> 17 crosses a block boundary: one new block, no copy
    assert len(c.steps[0].pairs) == 0
    assert (c.steps[0].block_tables[2] >= 0).sum() == 2


def test_generation_is_reproducible():
    a = gen.make_case("tiny", n_steps=2)
    b = gen.make_case("tiny", n_steps=2)
    for x, y in ((a.k_cache, b.k_cache), (a.q, b.q), (a.steps[1].k_new, b.steps[1].k_new)):
        assert np.array_equal(x, y)
    c = gen.make_case("tiny", n_steps=1)
    assert np.array_equal(a.k_cache, c.k_cache), "step count must not change the pool"


def test_poison_marks_exactly_the_empty_slots():
    c = gen.make_case("tiny", n_steps=0)
    valid = gen.valid_slot_mask(c.block_tables, c.context_lens, c.num_blocks, c.block_size)
    rows = c.k_cache.reshape(c.num_blocks * c.block_size, -1)
    nan_rows = np.all(rows == gen.NAN_BITS[gen.F16], axis=1)
    assert np.array_equal(nan_rows, ~valid)
    assert valid.sum() == 1 + 15 + 16 + 37


@pytest.mark.parametrize("name", ["llama2_7b", "mistral_7b_gqa"])
def test_private_workloads(name):
    c = gen.make_case(name, n_steps=3, with_pool=False)
    w = gen.WORKLOADS[name]
    lo, hi = (64, 1024) if name == "llama2_7b" else (1024, 4096)
    ctx0 = c.structure["initial_context_lens"]
    assert ctx0.min() >= lo and ctx0.max() <= hi and len(ctx0) == w.num_seqs
    used = c.block_tables[c.block_tables >= 0]
    assert len(np.unique(used)) == len(used), "no sharing in these workloads"
    need = sum(-(-(int(L) + 3) // 16) for L in ctx0)
    assert c.num_blocks == int(np.ceil(1.25 * need))
    for st in c.steps:
        assert len(st.pairs) == 0
    assert np.array_equal(c.steps[-1].context_lens, ctx0 + 3)


def test_prefix_workload_shares_two_blocks():
    c = gen.make_case("qwen_7b_prefix", n_steps=2, with_pool=False)
    bt = c.block_tables
    assert c.block_size == 256
    assert np.all(bt[:, 0] == bt[0, 0]) and np.all(bt[:, 1] == bt[0, 1])
    gen_tokens = c.structure["generated"]
    assert gen_tokens.min() >= 1 and gen_tokens.max() <= 512
    assert np.array_equal(c.context_lens, 512 + gen_tokens)
    private = bt[:, 2:][bt[:, 2:] >= 0]
    assert len(np.unique(private)) == len(private)
    assert not np.isin([bt[0, 0], bt[0, 1]], private).any()
    for st in c.steps:
        assert len(st.pairs) == 0
        blocks = st.slot_mapping // 256
        assert not np.isin(blocks, [bt[0, 0], bt[0, 1]]).any(), "appends go to private blocks"


def test_beam_workload_shares_all_but_last_block():
    c = gen.make_case("llama2_70b_beam", n_steps=3, with_pool=False)
    S, bs = c.num_seqs, c.block_size
    assert S == 256 and c.num_q_heads == 64 and c.num_kv_heads == 8
    short = c.structure["short_group"]
    assert short.sum() == round(0.7 * 64)
    ctx0 = c.structure["initial_context_lens"]
    for g in range(64):
        L = int(ctx0[4 * g])
        assert np.all(ctx0[4 * g:4 * g + 4] == L)
        assert (1 <= L <= 500) if short[g] else (1024 <= L <= 4096)
        nb = -(-L // bs)
        tabs = c.block_tables[4 * g:4 * g + 4, :nb]
        assert np.all(tabs[:, :nb - 1] == tabs[0, :nb - 1])
        assert len(set(tabs[:, nb - 1].tolist())) == 4
    for st in c.steps:
        assert len(st.pairs) <= 192
        # three copies per group whose last block is partially filled before the append
        partial = sum(1 for g in range(64) if (int(st.context_lens[4 * g]) - 1) % bs != 0)
        assert len(st.pairs) == 3 * partial
        dst = st.pairs[:, 1]
        assert len(np.unique(dst)) == len(dst)
        assert not np.isin(dst, st.pairs[:, 0]).any()


# The allocator's behaviour, derived by hand from its rules, on the library's
# C allocator (through gen.PoolAllocator) and on the tests' Python twin.


class _Twin:
    def __init__(self, nb, bs, order=None):
        self.m = block_manager_twin.BlockManager(nb, bs, order)

    def add(self, s, n):
        self.m.add_seq(s, n)

    def fork(self, p, c):
        self.m.fork(p, c)

    def free(self, s):
        self.m.free_seq(s)

    def table(self, s):
        return list(self.m.tables[s])

    def append(self, seqs):
        out = [self.m.append_slot(s) for s in seqs]
        return [o[0] for o in out], [o[1] for o in out if o[1] is not None]

    def ref(self, b):
        return int(self.m.ref[b])

    def used(self):
        return self.m.used()


class _C:
    def __init__(self, nb, bs, order=None):
        self.m = gen.PoolAllocator(nb, bs, order)

    def add(self, s, n):
        self.m.add_seq(s, n)

    def fork(self, p, c):
        self.m.fork(p, c)

    def free(self, s):
        self.m.free_seq(s)

    def table(self, s):
        t = self.m.table_array([s], self.m.num_blocks)[0]
        return [int(b) for b in t if b >= 0]

    def append(self, seqs):
        slots, pairs = self.m.append_slots(seqs)
        return slots.tolist(), [tuple(p) for p in pairs.tolist()]

    def ref(self, b):
        return self.m._a.refcount(b)

    def used(self):
        return self.m.used()


IMPLS = pytest.mark.parametrize("impl", [_C, _Twin], ids=["c_allocator", "python_twin"])


@IMPLS
def test_allocator_reuses_freed_blocks_lifo(impl):
    m = impl(8, 16, order=[5, 2, 7, 0, 1, 3, 4, 6])
    m.add(0, 40)
    assert m.table(0) == [5, 2, 7]
    m.add(1, 1)
    assert m.table(1) == [0]
    m.free(0)
    assert m.used() == 1
    m.add(2, 20)
    assert m.table(2) == [5, 2], "most recently freed blocks are reused first"


@IMPLS
def test_allocator_cow_and_refcounts(impl):
    m = impl(6, 4)
    m.add(0, 6)                      # blocks 0, 1 (second block half full)
    m.fork(0, 1)
    assert [m.ref(b) for b in range(2)] == [2, 2]
    slots, pairs = m.append([1])     # shared partially-filled block -> copy
    assert pairs == [(1, 2)] and slots == [2 * 4 + 2]
    assert [m.ref(b) for b in range(3)] == [2, 1, 1]
    slots, pairs = m.append([0])     # now private again -> in place
    assert pairs == [] and slots == [1 * 4 + 2]
    slots, pairs = m.append([0, 1])  # both fill their blocks: no allocation
    assert slots == [1 * 4 + 3, 2 * 4 + 3] and pairs == []
    slots, pairs = m.append([1])     # block full: a fresh block, no copy
    assert slots == [3 * 4 + 0] and pairs == []
    m.free(0)
    m.free(1)
    assert m.used() == 0 and all(m.ref(b) == 0 for b in range(6))


def test_allocator_out_of_blocks():
    m = block_manager_twin.BlockManager(2, 16)
    m.add_seq(0, 32)
    with pytest.raises(MemoryError):
        m.append_slot(0)
    c = gen.PoolAllocator(2, 16)
    c.add_seq(0, 32)
    with pytest.raises(pa.PaError):
        c.append_slots([0])

