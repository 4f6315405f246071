"""The C ABI without a GPU: symbols, host-side validation, host allocator."""
import ctypes

import numpy as np
import pytest

import block_manager_twin
from paged_kv_cache_458_b200 import gen, pa


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_458_b200 import build

    build.build()
    return pa.lib()


def test_library_exports_every_declared_symbol(lib):
    names = pa.header_functions()
    assert {"pa_decode", "pa_cache_append", "pa_copy_blocks", "pa_decode_workspace_bytes"} <= set(names)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, f"declared in include/pa.h but not exported: {missing}"


def test_status_strings(lib):
    for st in range(6):
        assert pa.status_string(st) and pa.status_string(st) != "unknown status"
    assert lib.pa_status_string(99) == b"unknown status"
    assert "sm_100a" in pa.pa_build_info()
    assert pa.pa_last_cuda_error()  # a static string, set by the last PA_ERR_CUDA


def _shape(**kw):
    base = dict(num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                num_blocks=64, max_blocks_per_seq=8, partition_tokens=0, dtype=pa.PA_F16)
    base.update(kw)
    return pa.make_shape(**base)


FAKE = 1 << 20  # a 16-byte-aligned non-null address; validation fails before any use


@pytest.mark.parametrize("kw,expect", [
    (dict(head_dim=96), pa.PA_ERR_UNSUPPORTED),
    (dict(head_dim=0), pa.PA_ERR_INVALID_ARG),
    (dict(num_q_heads=8, num_kv_heads=3), pa.PA_ERR_INVALID_ARG),
    (dict(num_q_heads=64, num_kv_heads=2), pa.PA_ERR_UNSUPPORTED),  # group 32
    (dict(block_size=12), pa.PA_ERR_UNSUPPORTED),       # blocks are multiples of 8 tokens
    (dict(dtype=7), pa.PA_ERR_UNSUPPORTED),
    (dict(partition_tokens=24), pa.PA_ERR_UNSUPPORTED),
    (dict(partition_tokens=4096), pa.PA_ERR_UNSUPPORTED),
    (dict(num_blocks=1 << 27), pa.PA_ERR_UNSUPPORTED),      # num_blocks * block_size >= 2^31
    (dict(num_seqs=-1), pa.PA_ERR_INVALID_ARG),
    (dict(variant=3), pa.PA_ERR_INVALID_ARG),
    (dict(variant=2, head_dim=64), pa.PA_ERR_UNSUPPORTED),
    (dict(variant=2, partition_tokens=64), pa.PA_ERR_UNSUPPORTED),
    (dict(variant=2, partition_tokens=1024), pa.PA_ERR_UNSUPPORTED),
    (dict(shared_prefix=2), pa.PA_ERR_INVALID_ARG),
    (dict(shared_prefix=1, variant=1), pa.PA_ERR_UNSUPPORTED),
    (dict(shared_prefix=1, variant=2), pa.PA_ERR_UNSUPPORTED),
    (dict(shared_prefix=1, head_dim=64), pa.PA_ERR_UNSUPPORTED),
    (dict(shared_prefix=1, partition_tokens=1024), pa.PA_ERR_UNSUPPORTED),
    (dict(shared_prefix=1, partition_tokens=192), pa.PA_ERR_UNSUPPORTED),
])
def test_decode_rejects_bad_shapes(lib, kw, expect):
    s = _shape(**kw)
    st = lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s), 100, FAKE, 1 << 20, None)
    assert st == expect


def test_shared_prefix_workspace(lib):
    """Counter, two plan records (16 B per sequence each, 256-aligned), split-K
    space for P + 2 partitions (a member's shared tokens and its own run may
    each end in a partial partition and start the next one part-way)."""
    s = _shape(shared_prefix=1)
    rows = 4 * 8 * 3                       # S * Hq * (1 partition + 2)
    acc = rows * 128 * 4
    assert lib.pa_decode_workspace_bytes(ctypes.byref(s), 100) == 256 + 2 * 256 + acc + rows * 8
    s20 = _shape(shared_prefix=1, num_seqs=20, max_blocks_per_seq=64)
    rows = 20 * 8 * 4                      # 1000 tokens: 2 partitions + 2
    assert lib.pa_decode_workspace_bytes(ctypes.byref(s20), 1000) == \
        256 + 2 * 512 + rows * 128 * 4 + rows * 8
    assert pa.pa_decode_resolved_variant(s) == pa.PA_DECODE_RESOLVED_SHARED_PREFIX


def test_fp8_cache_validation(lib):
    s8 = _shape(cache_format=pa.PA_CACHE_FP8_E4M3)
    s16 = _shape()
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE)
    # each entry point takes its own cache format
    assert lib.pa_decode(*args, ctypes.byref(s8), 100, FAKE, 1 << 20, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s16),
                             100, FAKE, 1 << 20, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s8),
                             100, FAKE, 1 << 20, None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, FAKE + 2, FAKE, FAKE, FAKE, 0.1, FAKE,
                             ctypes.byref(s8), 100, FAKE, 1 << 20, None) == pa.PA_ERR_INVALID_ARG
    for bad, st in ((dict(cache_format=2), pa.PA_ERR_UNSUPPORTED),
                    (dict(cache_format=pa.PA_CACHE_FP8_E4M3, variant=2, head_dim=64),
                     pa.PA_ERR_UNSUPPORTED),
                    (dict(cache_format=pa.PA_CACHE_FP8_E4M3, shared_prefix=1, variant=1),
                     pa.PA_ERR_UNSUPPORTED)):
        s = _shape(**bad)
        assert lib.pa_decode_fp8(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE,
                                 ctypes.byref(s), 100, FAKE, 1 << 20, None) == st
    # an E4M3 cache takes the tensor-core kernels by the same rule as a 16-bit one
    assert pa.pa_decode_resolved_variant(_shape(cache_format=1, num_q_heads=16)) == \
        pa.PA_DECODE_TENSOR_CORES
    assert pa.pa_decode_resolved_variant(_shape(cache_format=1, num_q_heads=4)) == \
        pa.PA_DECODE_CUDA_CORES
    assert pa.pa_decode_resolved_variant(_shape(cache_format=1, shared_prefix=1)) == \
        pa.PA_DECODE_RESOLVED_SHARED_PREFIX
    # appends
    assert lib.pa_cache_append(FAKE, FAKE, FAKE, 3, FAKE, FAKE, ctypes.byref(s8), None) == \
        pa.PA_ERR_INVALID_ARG
    assert lib.pa_cache_append_fp8(FAKE, FAKE, FAKE, 3, FAKE, FAKE, FAKE, FAKE, ctypes.byref(s16),
                                   None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_cache_append_fp8(FAKE, FAKE, FAKE, 3, FAKE, FAKE, None, FAKE, ctypes.byref(s8),
                                   None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_cache_append_fp8(FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE, FAKE, ctypes.byref(s8),
                                   None) == pa.PA_OK
    # the workspace does not depend on the cache format
    for kw in (dict(), dict(variant=1), dict(num_q_heads=4), dict(shared_prefix=1)):
        assert lib.pa_decode_workspace_bytes(ctypes.byref(_shape(cache_format=1, **kw)), 1000) == \
            lib.pa_decode_workspace_bytes(ctypes.byref(_shape(**kw)), 1000)


def test_multi_query_workspace_and_validation(lib):
    s = _shape(max_blocks_per_seq=64)
    one = lib.pa_decode_workspace_bytes(ctypes.byref(s), 700)
    assert lib.pa_decode_multi_workspace_bytes(ctypes.byref(s), 1, 700) == one
    assert lib.pa_decode_multi_workspace_bytes(ctypes.byref(s), 0, 700) == 0
    w4 = lib.pa_decode_multi_workspace_bytes(ctypes.byref(s), 4, 700)
    # 4 tokens x g 4 = 16 columns: one tensor-core item per (sequence, kv
    # head, partition) for all four queries, 512-token partitions: counter,
    # then 4 sequences x 4 queries x 8 heads x 2 partitions of (128 + 2) floats
    rows = 4 * 4 * 8 * 2
    assert w4 == 256 + rows * 128 * 4 + rows * 8
    # 1 query head per kv head, 2 tokens: the same path, 2 partitions
    s1 = _shape(num_q_heads=2, max_blocks_per_seq=64)
    rows = 4 * 2 * 2 * 2
    assert lib.pa_decode_multi_workspace_bytes(ctypes.byref(s1), 2, 700) == \
        256 + rows * 128 * 4 + rows * 8
    # forced onto CUDA cores: virtual tables and contexts, then a one-token
    # decode of 8 virtual sequences (one 1024-token partition: the counter only)
    s1c = _shape(num_q_heads=2, max_blocks_per_seq=64, variant=1)
    assert lib.pa_decode_multi_workspace_bytes(ctypes.byref(s1c), 2, 700) == 4 * 8 * 64 + 256 + 256
    # 8 tokens x g 8 = 64 columns > 32: the virtual sequences, grouped
    s88 = _shape(num_q_heads=16, max_blocks_per_seq=64)
    assert lib.pa_decode_multi_workspace_bytes(ctypes.byref(s88), 8, 700) > 4 * 8 * 16 * 2 * 520
    st = lib.pa_decode_multi(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s), 0, 700, FAKE,
                             1 << 24, None)
    assert st == pa.PA_ERR_INVALID_ARG
    st = lib.pa_decode_multi(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s), 4, 700, FAKE,
                             w4 - 1, None)
    assert st == pa.PA_ERR_INVALID_ARG
    s8 = _shape(max_blocks_per_seq=64, cache_format=pa.PA_CACHE_FP8_E4M3)
    st = lib.pa_decode_multi(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s8), 4, 700,
                             FAKE, 1 << 24, None)
    assert st == pa.PA_ERR_INVALID_ARG


def test_swap_validation(lib):
    s = _shape()
    call = lambda pairs=FAKE, n=2, sk=FAKE, sv=FAKE + (1 << 24), snb=8, dk=FAKE + (2 << 24), \
        dv=FAKE + (3 << 24), dnb=8: lib.pa_swap_blocks(pairs, n, sk, sv, snb, dk, dv, dnb,  # noqa: E731
                                                      ctypes.byref(s), None)
    n0 = pa.pa_kernel_launches()
    assert call(n=0) == pa.PA_OK
    assert call(n=-1) == pa.PA_ERR_INVALID_ARG
    assert call(pairs=None) == pa.PA_ERR_INVALID_ARG
    assert call(dk=None) == pa.PA_ERR_INVALID_ARG
    assert call(sk=FAKE + 8) == pa.PA_ERR_INVALID_ARG            # misaligned
    assert call(dk=FAKE + 4096) == pa.PA_ERR_INVALID_ARG         # pools overlap
    assert call(n=70000) == pa.PA_ERR_UNSUPPORTED
    # FAKE addresses are no memory the device knows: refused before any launch
    assert call() == pa.PA_ERR_INVALID_ARG
    assert pa.pa_kernel_launches() == n0


def test_default_partition(lib):
    assert pa.pa_decode_partition_tokens(_shape()) == 512                      # tensor cores (group 4)
    assert pa.pa_decode_partition_tokens(_shape(num_q_heads=4)) == 1024        # CUDA cores (group 2)
    assert pa.pa_decode_partition_tokens(_shape(num_q_heads=16)) == 512        # tensor cores
    assert pa.pa_decode_partition_tokens(_shape(shared_prefix=1)) == 512
    assert pa.pa_decode_partition_tokens(_shape(partition_tokens=48)) == 48
    assert pa.pa_decode_partition_tokens(_shape(num_q_heads=16, variant=1)) == 1024


def test_resolved_variant(lib):
    assert pa.pa_decode_resolved_variant(_shape()) == pa.PA_DECODE_TENSOR_CORES        # group 4
    assert pa.pa_decode_resolved_variant(_shape(num_q_heads=4)) == pa.PA_DECODE_CUDA_CORES  # group 2
    # 8-token blocks: tensor cores from group 8 only
    assert pa.pa_decode_resolved_variant(_shape(block_size=8)) == pa.PA_DECODE_CUDA_CORES
    assert pa.pa_decode_resolved_variant(_shape(block_size=8, num_q_heads=16)) == pa.PA_DECODE_TENSOR_CORES
    assert pa.pa_decode_resolved_variant(_shape(num_q_heads=16)) == pa.PA_DECODE_TENSOR_CORES
    assert pa.pa_decode_resolved_variant(_shape(num_q_heads=16, head_dim=64)) == pa.PA_DECODE_CUDA_CORES
    assert pa.pa_decode_resolved_variant(_shape(num_q_heads=16, partition_tokens=1024)) == pa.PA_DECODE_CUDA_CORES
    assert pa.pa_decode_resolved_variant(_shape(variant=2)) == pa.PA_DECODE_TENSOR_CORES
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_resolved_variant(_shape(head_dim=96))
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


def test_decode_rejects_bad_pointers_and_sizes(lib):
    s = _shape()
    call = lambda **o: lib.pa_decode(  # noqa: E731
        o.get("q", FAKE), FAKE, FAKE, o.get("bt", FAKE), FAKE, o.get("scale", 0.1), FAKE,
        ctypes.byref(s), o.get("maxlen", 100), o.get("ws", FAKE), o.get("wsb", 1 << 20), None)
    assert call(q=None) == pa.PA_ERR_INVALID_ARG
    assert call(q=FAKE + 8) == pa.PA_ERR_INVALID_ARG            # misaligned
    assert call(bt=FAKE + 2) == pa.PA_ERR_INVALID_ARG
    assert call(scale=float("nan")) == pa.PA_ERR_INVALID_ARG
    assert call(maxlen=8 * 16 + 1) == pa.PA_ERR_INVALID_ARG     # beyond max_blocks_per_seq * bs
    assert call(maxlen=-1) == pa.PA_ERR_INVALID_ARG
    # 100 tokens fit one partition: only the work counter ...
    assert lib.pa_decode_workspace_bytes(ctypes.byref(s), 100) == 256
    st = lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s), 100, None, 0, None)
    assert st == pa.PA_ERR_INVALID_ARG
    # ... 2000 tokens need two default (1024-token, CUDA-core) partitions and split-K space
    s2 = _shape(max_blocks_per_seq=128, num_q_heads=4)  # group 2
    assert lib.pa_decode_workspace_bytes(ctypes.byref(s2), 1024) == 256
    need = lib.pa_decode_workspace_bytes(ctypes.byref(s2), 2000)
    rows = 4 * 4 * 2
    assert need == 256 + rows * 128 * 4 + rows * 2 * 4
    st = lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s2), 2000, FAKE, need - 1, None)
    assert st == pa.PA_ERR_INVALID_ARG
    st = lib.pa_decode(FAKE, FAKE, FAKE, FAKE, FAKE, 0.1, FAKE, ctypes.byref(s2), 2000, None, 0, None)
    assert st == pa.PA_ERR_INVALID_ARG
    # the tensor-core kernel's default partition is 512 tokens
    s3 = _shape(num_q_heads=16, max_blocks_per_seq=128)
    assert lib.pa_decode_workspace_bytes(ctypes.byref(s3), 1000) == 256 + 4 * 16 * 2 * 130 * 4


def test_empty_batches_launch_nothing(lib):
    before = pa.pa_kernel_launches()
    s = _shape(num_seqs=0)
    assert lib.pa_decode(None, None, None, None, None, 0.1, None, ctypes.byref(s), 0, None, 0, None) == 0
    assert lib.pa_cache_append(None, None, None, 0, None, None, ctypes.byref(_shape()), None) == 0
    assert lib.pa_copy_blocks(None, 0, None, None, ctypes.byref(_shape()), None) == 0
    assert pa.pa_kernel_launches() == before


def test_append_and_copy_reject_bad_arguments(lib):
    s = _shape()
    assert lib.pa_cache_append(FAKE, FAKE, FAKE, -1, FAKE, FAKE, ctypes.byref(s), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_cache_append(None, FAKE, FAKE, 3, FAKE, FAKE, ctypes.byref(s), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_cache_append(FAKE, FAKE, FAKE, 3, FAKE + 4, FAKE, ctypes.byref(s), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, -2, FAKE, FAKE, ctypes.byref(s), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(None, 2, FAKE, FAKE, ctypes.byref(s), None) == pa.PA_ERR_INVALID_ARG
    assert lib.pa_copy_blocks(FAKE, 70000, FAKE, FAKE, ctypes.byref(s), None) == pa.PA_ERR_UNSUPPORTED
    bad = _shape(head_dim=80)
    assert lib.pa_copy_blocks(FAKE, 1, FAKE, FAKE, ctypes.byref(bad), None) == pa.PA_ERR_UNSUPPORTED


# ---------------------------------------------------------------- allocator


def _apply(ops, mgr_py, mgr_c, max_blocks):
    """Run the same operation list on both managers and compare state."""
    for op in ops:
        kind = op[0]
        if kind == "add":
            mgr_py.add_seq(op[1], op[2])
            mgr_c.add_seq(op[1], op[2])
        elif kind == "fork":
            mgr_py.fork(op[1], op[2])
            mgr_c.fork(op[1], op[2])
        elif kind == "free":
            mgr_py.free_seq(op[1])
            mgr_c.free_seq(op[1])
        elif kind == "append":
            seqs = op[1]
            exp_slots, exp_pairs = [], []
            for s in seqs:
                slot, pair = mgr_py.append_slot(s)
                exp_slots.append(slot)
                if pair is not None:
                    exp_pairs.append(pair)
            slots, pairs = mgr_c.append_slots(seqs)
            assert slots.tolist() == exp_slots
            assert [tuple(p) for p in pairs.tolist()] == exp_pairs
        seqs = sorted(mgr_py.tables)
        if seqs:
            t, lens = mgr_c.block_tables(seqs, max_blocks)
            assert np.array_equal(t, mgr_py.table_array(seqs, max_blocks))
            assert lens.tolist() == [mgr_py.lens[s] for s in seqs]
        assert mgr_c.num_free() == len(mgr_py.free)
        for b in range(mgr_py.num_blocks):
            assert mgr_c.refcount(b) == mgr_py.ref[b]


def test_allocator_matches_python_twin(lib):
    rng = np.random.default_rng(7)
    NB, bs = 96, 16
    order = rng.permutation(NB)
    py = block_manager_twin.BlockManager(NB, bs, order)
    c = pa.Allocator(NB, bs, order)
    ops, live, nxt = [], [], 0
    for _ in range(300):
        r = rng.random()
        if r < 0.25 or not live:
            ops.append(("add", nxt, int(rng.integers(0, 40))))
            live.append(nxt)
            nxt += 1
        elif r < 0.4:
            ops.append(("fork", int(rng.choice(live)), nxt))
            live.append(nxt)
            nxt += 1
        elif r < 0.5 and len(live) > 1:
            s = int(rng.choice(live))
            ops.append(("free", s))
            live.remove(s)
        else:
            k = int(rng.integers(1, min(6, len(live)) + 1))
            ops.append(("append", [int(x) for x in rng.choice(live, size=k, replace=False)]))
        try:
            _apply(ops[-1:], py, c, 64)
        except MemoryError:
            break  # the Python side ran out first; the C side is checked below
    c.close()


def test_beam_workload_copies_come_from_the_allocator(lib):
    """The beam workload's per-step tables, slots and copy-on-write pairs are
    the C allocator's: replay the same host operations on the Python twin and
    check the recorded case against it, and against the copy rule itself."""
    case = gen.make_case("llama2_70b_beam", n_steps=3, with_pool=False, num_seqs=32)
    py = block_manager_twin.BlockManager(case.num_blocks, case.block_size,
                                         case.structure["pool_order"])
    ctx = case.structure["initial_context_lens"]
    bs = case.block_size
    for g in range(8):
        L = int(ctx[4 * g])
        shared = ((L - 1) // bs) * bs
        py.add_seq(4 * g, shared)
        for k in range(1, 4):
            py.fork(4 * g, 4 * g + k)
        for k in range(4):
            py.extend(4 * g + k, L - shared)
    seqs = list(range(32))
    assert np.array_equal(py.table_array(seqs, case.max_blocks_per_seq), case.block_tables)
    for st in case.steps:
        for g in range(8):
            for k in range(1, 4):
                py.free_seq(4 * g + k)
                py.fork(4 * g, 4 * g + k)
        before = py.table_array(seqs, case.max_blocks_per_seq)
        lens = [py.lens[s] for s in seqs]
        res = [py.append_slot(s) for s in seqs]
        assert np.array_equal(st.slot_mapping, [r[0] for r in res])
        assert [tuple(p) for p in st.pairs.tolist()] == [r[1] for r in res if r[1] is not None]
        assert np.array_equal(py.table_array(seqs, case.max_blocks_per_seq), st.block_tables)
        # the rule: a pair exactly where a sequence appends into a partly
        # filled last block that another sequence still holds
        for s, (slot, pair) in zip(seqs, res):
            last = int(before[s, (lens[s] - 1) // bs]) if lens[s] else -1
            partial = lens[s] % bs != 0
            if pair is not None:
                assert partial and pair[0] == last and slot // bs == pair[1]


def test_allocator_out_of_blocks_changes_nothing(lib):
    c = pa.Allocator(3, 16)
    c.add_seq(0, 16)
    c.add_seq(1, 16)
    c.add_seq(2, 5)
    before = c.block_tables([0, 1, 2], 4)
    with pytest.raises(pa.PaError) as e:
        c.append_slots([2, 0, 1])       # 0 and 1 each need a new block; only 0 free
    assert e.value.status == pa.PA_ERR_OOM
    after = c.block_tables([0, 1, 2], 4)
    assert all(np.array_equal(x, y) for x, y in zip(before, after))
    assert c.num_free() == 0
    with pytest.raises(pa.PaError):
        c.add_seq(3, 1)
    c.close()


def test_allocator_rejects_bad_input(lib):
    assert not lib.pa_alloc_create(4, 16, (ctypes.c_int32 * 4)(0, 1, 1, 3))
    assert not lib.pa_alloc_create(0, 16, None)
    c = pa.Allocator(4, 16)
    with pytest.raises(pa.PaError):
        c.fork(5, 6)
    c.add_seq(1, 3)
    with pytest.raises(pa.PaError):
        c.add_seq(1, 3)
    with pytest.raises(pa.PaError):
        c.append_slots([1, 1])
    with pytest.raises(pa.PaError):
        c.block_tables([1, 9], 4)
    assert c.refcount(-1) == -1 and c.refcount(4) == -1
    c.close()
