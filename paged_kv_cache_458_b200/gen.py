"""Seeded synthetic inputs for paged decode attention.

This module builds the inputs that both the CUDA path and the CPU oracle
consume: query rows, the paged K/V pool, block tables, context lengths, slot
mappings for the per-step append and copy-on-write pairs.  It holds none of
the attention arithmetic; it only draws random numbers and lays out block
structure.

Block structure follows the PagedAttention description on the pages:

* fixed-size physical blocks of ``block_size`` tokens in one pool tensor of
  shape ``[num_blocks, block_size, num_heads, head_dim]`` (zingnex.cn,
  "vLLM与PagedAttention深度剖析", section 3.2, second code block);
* a per-sequence block table from logical to physical blocks, e.g. logical
  block 0 -> physical block 7 (5688vip.com notes, section 2.2);
* blocks allocated only when a token crosses into a new block, and freed
  blocks reused from a pool (zingnex.cn section 3.2, items 1 and 4;
  jsqmd.com "vLLM-v0.11.0性能实测", section 4.2);
* shared blocks with copy-on-write for beam candidates (zingnex.cn section
  3.2, item 3) and a shared prefix across requests (jsqmd.com section 4.2).

Values are drawn as float32 N(0, 1) from NumPy's PCG64 and rounded to
nearest-even into fp16 or bf16.  Each workload has its own seed
(458000 + its number); independent sub-streams are spawned for structure,
pool contents and per-step values so that changing the number of steps does
not change the pool.

Element arrays are returned as ``uint16`` bit patterns.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

F16 = 0
BF16 = 1
DTYPE_NAMES = {F16: "f16", BF16: "bf16"}

# Quiet-NaN bit patterns used to poison every cache slot that holds no token.
NAN_BITS = {F16: 0x7E00, BF16: 0x7FC0}

SEED_BASE = 458000


@dataclass(frozen=True)
class Workload:
    """One of the five decode workloads the build is measured on."""

    name: str
    number: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: int
    description: str
    partition_tokens: int = 0   # split-K partition the workload states (0: the library's default)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 4, 4, 4, 64, 16, F16,
                 "4 seqs, ctx {1,15,16,37}, 4/4 heads, D 64, bs 16, pool of 32 "
                 "blocks in seeded random order, fp16, +1 appended token"),
        Workload("llama2_7b", 2, 64, 32, 32, 128, 16, F16,
                 "batch 64, 32/32 heads, D 128, bs 16, fp16, ctx U[64,1024], "
                 "shuffled pool 1.25x need, +1 token per seq per step"),
        Workload("mistral_7b_gqa", 3, 128, 32, 8, 128, 16, BF16,
                 "batch 128, 32/8 heads (group 4), D 128, bs 16, bf16, "
                 "ctx U[1024,4096], shuffled pool 1.25x need, 512-token partitions", 512),
        Workload("qwen_7b_prefix", 4, 64, 32, 32, 128, 256, F16,
                 "batch 64, 32/32 heads, D 128, bs 256, fp16, all tables share 2 "
                 "prefix blocks (512 tokens) + private U[1,512] tokens"),
        Workload("llama2_70b_beam", 5, 256, 64, 8, 128, 16, BF16,
                 "batch 256 = 64 beam groups x 4, 64/8 heads (group 8), D 128, bs 16, "
                 "bf16, ctx 70% lognormal(median 300, sigma 0.5) clipped [1,500], "
                 "30% U[1024,4096], beams share all but the last block, CoW before append"),
    ]
}
WORKLOAD_BY_NUMBER = {w.number: w for w in WORKLOADS.values()}


# ----------------------------------------------------------------------------
# value generation


def f32_to_f16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to fp16 (nearest-even) and return the bit patterns."""
    return np.asarray(x, dtype=np.float32).astype(np.float16).view(np.uint16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even) and return the bit patterns.

    Inputs are finite normal draws, so no NaN/Inf handling is needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    return f32_to_f16_bits(x) if dtype == F16 else f32_to_bf16_bits(x)


def normal_bits(rng: np.random.Generator, shape, dtype: int, chunk: int = 1 << 24) -> np.ndarray:
    """N(0,1) float32 draws rounded into ``dtype``; drawn in chunks to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        out[i:i + m] = to_bits(rng.standard_normal(m, dtype=np.float32), dtype)
    return out.reshape(shape)


def bits_to_f32(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Widen fp16/bf16 bit patterns to float32 (exact)."""
    bits = np.asarray(bits, dtype=np.uint16)
    if dtype == F16:
        return bits.view(np.float16).astype(np.float32)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# block manager (input construction)


class PoolAllocator:
    """The library's host block allocator (the C ABI's pa_alloc_*: free list,
    reference counts, block tables) behind the calls the workload builders
    make, plus the peak number of blocks in use.

    The free list is a stack that starts as ``order`` with ``order[0]`` on
    top; a block whose reference count drops to zero goes back on top, so the
    next allocation reuses it (the pool reuse of zingnex.cn section 3.2, item
    4).  ``append_slots`` allocates only when a token crosses into a new block
    (item 1) and copies a shared last block before writing to it (item 3,
    copy-on-write), returning the copy pairs.
    """

    def __init__(self, num_blocks: int, block_size: int, order=None):
        from . import build, pa

        try:
            pa.lib()
        except pa.LibraryMissing:
            build.build()  # host code only: the allocator needs no GPU
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        self._a = pa.Allocator(self.num_blocks, self.block_size, order)
        self.lens: dict[int, int] = {}  # tokens per live sequence
        self.peak_used = 0

    def _track(self):
        self.peak_used = max(self.peak_used, self.used())

    def used(self) -> int:
        return self.num_blocks - self._a.num_free()

    def add_seq(self, seq: int, n_tokens: int) -> None:
        self._a.add_seq(seq, n_tokens)
        self.lens[seq] = int(n_tokens)
        self._track()

    def extend(self, seq: int, n_tokens: int) -> None:
        """Grow a sequence by ``n_tokens`` (prefill): blocks on demand, no copy."""
        self._a.extend(seq, n_tokens)
        self.lens[seq] += int(n_tokens)
        self._track()

    def fork(self, parent: int, child: int) -> None:
        """``child`` shares every block of ``parent`` (reference count + 1 each)."""
        self._a.fork(parent, child)
        self.lens[child] = self.lens[parent]

    def free_seq(self, seq: int) -> None:
        self._a.free_seq(seq)
        del self.lens[seq]

    def append_slots(self, seqs):
        """Slots of the next token of each of ``seqs`` (in order) and the
        copy-on-write pairs (src, dst), int32 [n][2]."""
        slots, pairs = self._a.append_slots(seqs)
        for s in seqs:
            self.lens[int(s)] += 1
        self._track()
        return slots, pairs

    def table_array(self, seqs, max_blocks: int) -> np.ndarray:
        """Block tables [len(seqs)][max_blocks], padded with -1."""
        return self._a.block_tables(list(seqs), max_blocks)[0]

    def lens_array(self, seqs) -> np.ndarray:
        return np.array([self.lens[int(s)] for s in seqs], dtype=np.int32)

    def close(self) -> None:
        self._a.close()


# ----------------------------------------------------------------------------
# workload construction


@dataclass
class Step:
    """Host inputs of one decode step: CoW copies, append, then decode."""

    pairs: np.ndarray          # int32 [n][2] (src, dst), possibly n == 0
    slot_mapping: np.ndarray   # int32 [S]
    k_new: np.ndarray          # uint16 [S][Hkv][D]
    v_new: np.ndarray          # uint16 [S][Hkv][D]
    q: np.ndarray              # uint16 [S][Hq][D]
    block_tables: np.ndarray   # int32 [S][MBS], after the step's allocation
    context_lens: np.ndarray   # int32 [S], including the appended token


@dataclass
class Case:
    workload: Workload
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    max_blocks_per_seq: int
    dtype: int
    scale: float
    k_cache: np.ndarray        # uint16 [NB][bs][Hkv][D], state before step 0
    v_cache: np.ndarray
    q: np.ndarray              # uint16 [S][Hq][D], query for a decode of the initial state
    block_tables: np.ndarray   # int32 [S][MBS], initial state
    context_lens: np.ndarray   # int32 [S], initial state
    steps: list = field(default_factory=list)
    structure: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def pool_shape(self):
        return (self.num_blocks, self.block_size, self.num_kv_heads, self.head_dim)


def _rng(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, sub])))


_STREAM_STRUCT, _STREAM_POOL, _STREAM_QUERY, _STREAM_STEP = 1, 2, 3, 4


def _context_lengths(w: Workload, rng: np.random.Generator):
    """Initial context lengths (before any appended token) and extra structure."""
    S = w.num_seqs
    info = {}
    if w.name == "tiny":
        ctx = np.array([1, 15, 16, 37], dtype=np.int64)
    elif w.name == "llama2_7b":
        ctx = rng.integers(64, 1024, size=S, endpoint=True)
    elif w.name == "mistral_7b_gqa":
        ctx = rng.integers(1024, 4096, size=S, endpoint=True)
    elif w.name == "qwen_7b_prefix":
        gen = rng.integers(1, 512, size=S, endpoint=True)
        info["prefix_tokens"] = 512
        info["generated"] = gen
        ctx = 512 + gen
    elif w.name == "llama2_70b_beam":
        G = S // 4
        n_short = int(round(0.7 * G))
        short = np.zeros(G, dtype=bool)
        short[rng.permutation(G)[:n_short]] = True
        lg = np.clip(np.rint(rng.lognormal(math.log(300.0), 0.5, size=G)), 1, 500)
        un = rng.integers(1024, 4096, size=G, endpoint=True)
        per_group = np.where(short, lg, un).astype(np.int64)
        info["short_group"] = short
        ctx = np.repeat(per_group, 4)
    else:  # pragma: no cover
        raise KeyError(w.name)
    return ctx.astype(np.int64), info


def _build_initial(w: Workload, mgr: PoolAllocator, ctx: np.ndarray, info: dict) -> None:
    S, bs = w.num_seqs, w.block_size
    if w.name == "qwen_7b_prefix":
        P = info["prefix_tokens"]
        mgr.add_seq(0, P)
        for s in range(1, S):
            mgr.fork(0, s)
        for s in range(S):
            mgr.extend(s, int(ctx[s]) - P)
    elif w.name == "llama2_70b_beam":
        for g in range(S // 4):
            b0 = 4 * g
            L = int(ctx[b0])
            shared = ((L - 1) // bs) * bs  # all full blocks but the last one
            mgr.add_seq(b0, shared)
            for k in range(1, 4):
                mgr.fork(b0, b0 + k)
            for k in range(4):
                mgr.extend(b0 + k, L - shared)
    else:
        for s in range(S):
            mgr.add_seq(s, int(ctx[s]))


def _run_steps(w: Workload, mgr: PoolAllocator, n_steps: int):
    """Host block operations of each step: beam re-fork, then one appended
    slot per sequence (with the copy-on-write pairs the allocator returns)."""
    S = w.num_seqs
    out = []
    for _ in range(n_steps):
        if w.name == "llama2_70b_beam":
            # Stand-in for beam re-selection: beams 1..3 take beam 0 as parent.
            for g in range(S // 4):
                for k in range(1, 4):
                    mgr.free_seq(4 * g + k)
                    mgr.fork(4 * g, 4 * g + k)
        slots, pairs = mgr.append_slots(list(range(S)))
        out.append((slots, np.asarray(pairs, dtype=np.int32).reshape(-1, 2)))
    return out


def _pool_blocks(w: Workload, ctx, info, n_steps: int) -> int:
    if w.name == "tiny":
        return 32
    probe = PoolAllocator(1 << 22, w.block_size)
    _build_initial(w, probe, ctx, info)
    _run_steps(w, probe, n_steps)
    probe.close()
    return int(math.ceil(1.25 * probe.peak_used))


def make_case(name: str, n_steps: int = 1, poison: bool = True, seed: int | None = None,
              num_seqs: int | None = None, with_pool: bool = True) -> Case:
    """Build a workload's initial state and ``n_steps`` decode steps.

    ``poison`` fills every pool slot that holds no token with NaN, so that a
    read of a slot past a sequence's context shows up in the output.
    ``num_seqs`` truncates the batch (beam workloads keep whole groups).
    ``with_pool=False`` skips drawing pool values (structure only).
    """
    w = WORKLOADS[name]
    if num_seqs is not None:
        assert num_seqs <= w.num_seqs
        if w.name == "llama2_70b_beam":
            assert num_seqs % 4 == 0
        w = Workload(w.name, w.number, num_seqs, w.num_q_heads, w.num_kv_heads,
                     w.head_dim, w.block_size, w.dtype, w.description, w.partition_tokens)
    seed = SEED_BASE + w.number if seed is None else int(seed)
    rs = _rng(seed, _STREAM_STRUCT)
    ctx0, info = _context_lengths(w, rs)
    if num_seqs is not None and w.name != "tiny":
        ctx0 = ctx0[:num_seqs]
    NB = _pool_blocks(w, ctx0, info, n_steps)
    order = rs.permutation(NB)
    mgr = PoolAllocator(NB, w.block_size, order)
    _build_initial(w, mgr, ctx0, info)
    seqs = list(range(w.num_seqs))
    max_len = int(ctx0.max()) + n_steps
    MBS = -(-max_len // w.block_size)
    bt0 = mgr.table_array(seqs, MBS)
    cl0 = mgr.lens_array(seqs)
    step_ops = _run_steps(w, mgr, n_steps)

    # Replay the operations to record the per-step tables (cheap; keeps the
    # structure pass above free of per-step bookkeeping).
    mgr2 = PoolAllocator(NB, w.block_size, order)
    _build_initial(w, mgr2, ctx0, info)
    steps_tables = []
    for _ in range(n_steps):
        _run_steps(w, mgr2, 1)
        steps_tables.append((mgr2.table_array(seqs, MBS), mgr2.lens_array(seqs)))

    S, Hq, Hkv, D, bs = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size
    scale = float(np.float32(1.0 / math.sqrt(D)))
    rq = _rng(seed, _STREAM_QUERY)
    q0 = normal_bits(rq, (S, Hq, D), w.dtype)

    if with_pool:
        rp = _rng(seed, _STREAM_POOL)
        kc = normal_bits(rp, (NB, bs, Hkv, D), w.dtype)
        vc = normal_bits(rp, (NB, bs, Hkv, D), w.dtype)
        if poison:
            valid = valid_slot_mask(bt0, cl0, NB, bs)
            nan = np.uint16(NAN_BITS[w.dtype])
            kc.reshape(NB * bs, Hkv * D)[~valid] = nan
            vc.reshape(NB * bs, Hkv * D)[~valid] = nan
    else:
        kc = vc = np.zeros((0,), dtype=np.uint16)

    steps = []
    for i, ((slots, pairs), (bt, cl)) in enumerate(zip(step_ops, steps_tables)):
        r = _rng(seed, _STREAM_STEP, i)
        steps.append(Step(
            pairs=pairs, slot_mapping=slots,
            k_new=normal_bits(r, (S, Hkv, D), w.dtype),
            v_new=normal_bits(r, (S, Hkv, D), w.dtype),
            q=normal_bits(r, (S, Hq, D), w.dtype),
            block_tables=bt, context_lens=cl))

    structure = dict(info)
    structure["initial_context_lens"] = ctx0
    structure["pool_order"] = order
    return Case(workload=w, seed=seed, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv,
                head_dim=D, block_size=bs, num_blocks=NB, max_blocks_per_seq=MBS,
                dtype=w.dtype, scale=scale, k_cache=kc, v_cache=vc, q=q0,
                block_tables=bt0, context_lens=cl0, steps=steps, structure=structure)


def valid_slot_mask(block_tables: np.ndarray, context_lens: np.ndarray, num_blocks: int,
                    block_size: int) -> np.ndarray:
    """Boolean [NB * bs]: True where some sequence stores a token."""
    valid = np.zeros(num_blocks * block_size, dtype=bool)
    ar = np.arange(block_size)
    for s in range(block_tables.shape[0]):
        L = int(context_lens[s])
        if L == 0:
            continue
        nb = -(-L // block_size)
        slots = (block_tables[s, :nb].astype(np.int64)[:, None] * block_size + ar).reshape(-1)[:L]
        valid[slots] = True
    return valid


def grouped_decode_case(rng: np.random.Generator, *, groups, num_q_heads: int,
                        num_kv_heads: int, head_dim: int, block_size: int, dtype: int,
                        poison: bool = True):
    """A decode input whose consecutive sequences come in groups sharing a prefix.

    ``groups`` is a list of ``(shared_tokens, [context of each member])``.
    The members' tables start with the blocks of a parent that holds
    ``shared_tokens`` tokens (its last block may be partly filled, and the
    members then continue in it, as forks of one prompt do before they
    diverge) and go on with private blocks; a member shorter than the shared
    part keeps only its own prefix of it.  Blocks come from a random
    permutation of the pool.  Returns a dict like ``random_decode_case``.
    """
    bs = block_size
    ctx = [int(c) for _, members in groups for c in members]
    need = sum(-(-int(sh) // bs) for sh, _ in groups) + sum(-(-c // bs) for c in ctx) + 2
    NB = max(need, 4)
    mgr = PoolAllocator(NB, bs, rng.permutation(NB))
    s = 0
    for gi, (shared, members) in enumerate(groups):
        # The parent grows to the shared length; a member shorter than that
        # forks when the parent holds exactly its tokens, the others fork at
        # the shared length and then grow on their own.
        parent = -1 - gi
        mgr.add_seq(parent, 0)
        ids = list(range(s, s + len(members)))
        for L in sorted({int(c) for c in members if c < shared}):
            mgr.extend(parent, L - mgr.lens[parent])
            for sid, c in zip(ids, members):
                if c == L:
                    mgr.fork(parent, sid)
        mgr.extend(parent, int(shared) - mgr.lens[parent])
        for sid, c in zip(ids, members):
            if c >= shared:
                mgr.fork(parent, sid)
                mgr.extend(sid, int(c) - int(shared))
        s += len(members)
    S = s
    MBS = max(1, -(-max(ctx, default=0) // bs))
    bt = mgr.table_array(list(range(S)), MBS)
    cl = mgr.lens_array(list(range(S)))
    q = normal_bits(rng, (S, num_q_heads, head_dim), dtype)
    kc = normal_bits(rng, (NB, bs, num_kv_heads, head_dim), dtype)
    vc = normal_bits(rng, (NB, bs, num_kv_heads, head_dim), dtype)
    if poison:
        valid = valid_slot_mask(bt, cl, NB, bs)
        nan = np.uint16(NAN_BITS[dtype])
        kc.reshape(NB * bs, -1)[~valid] = nan
        vc.reshape(NB * bs, -1)[~valid] = nan
    return dict(q=q, k_cache=kc, v_cache=vc, block_tables=bt, context_lens=cl,
                num_blocks=NB, max_blocks_per_seq=MBS,
                scale=float(np.float32(1.0 / math.sqrt(head_dim))))


def random_decode_case(rng: np.random.Generator, *, num_seqs: int, num_q_heads: int,
                       num_kv_heads: int, head_dim: int, block_size: int, dtype: int,
                       context_lens, num_blocks: int | None = None, poison: bool = True,
                       shared_prefix_blocks: int = 0):
    """A small decode input of arbitrary shape for edge-case tests.

    Blocks are allocated from a random permutation of the pool; with
    ``shared_prefix_blocks`` > 0 every sequence long enough starts with the
    same physical blocks.  Returns a dict of host arrays.
    """
    ctx = np.asarray(context_lens, dtype=np.int64)
    S = num_seqs
    assert ctx.shape == (S,)
    need = int(sum(-(-int(L) // block_size) for L in ctx)) + 1
    NB = max(need + 2, 4) if num_blocks is None else int(num_blocks)
    order = rng.permutation(NB)
    mgr = PoolAllocator(NB, block_size, order)
    if shared_prefix_blocks:
        P = shared_prefix_blocks * block_size
        mgr.add_seq(-1, P)
    for s in range(S):
        L = int(ctx[s])
        if shared_prefix_blocks and L > shared_prefix_blocks * block_size:
            mgr.fork(-1, s)
            mgr.extend(s, L - shared_prefix_blocks * block_size)
        else:
            mgr.add_seq(s, L)
    MBS = max(1, -(-int(ctx.max(initial=0)) // block_size))
    bt = mgr.table_array(list(range(S)), MBS)
    cl = mgr.lens_array(list(range(S)))
    q = normal_bits(rng, (S, num_q_heads, head_dim), dtype)
    kc = normal_bits(rng, (NB, block_size, num_kv_heads, head_dim), dtype)
    vc = normal_bits(rng, (NB, block_size, num_kv_heads, head_dim), dtype)
    if poison:
        valid = valid_slot_mask(bt, cl, NB, block_size)
        nan = np.uint16(NAN_BITS[dtype])
        kc.reshape(NB * block_size, -1)[~valid] = nan
        vc.reshape(NB * block_size, -1)[~valid] = nan
    return dict(q=q, k_cache=kc, v_cache=vc, block_tables=bt, context_lens=cl,
                num_blocks=NB, max_blocks_per_seq=MBS,
                scale=float(np.float32(1.0 / math.sqrt(head_dim))))
