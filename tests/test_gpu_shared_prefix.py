"""Shared-prefix decode (pa_shape.shared_prefix = 1) against the CPU oracle.

Sequences whose block tables start with the same physical blocks are decoded
in groups: their shared tokens once for all members, then each member's own
tokens, then a merge.  The result must match the oracle like any decode, and
the group plan the first kernel leaves in the workspace must match the rule
in include/pa.h, recomputed here on the host (bit-exact: it is index work).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from paged_kv_cache_458_b200 import gen, pa  # noqa: E402
from gpu_util import SHARED, dev, dev_i32, gpu_decode, host_bits, shape_of  # noqa: E402
from tolerance import assert_decode_close  # noqa: E402

pytestmark = pytest.mark.gpu

CHUNK = 256        # groups stay inside aligned windows of this many sequences
MIN_SHARED = 128   # fewer shared tokens: no group


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_458_b200 import build

    build.build()
    pa.pa_last_device_error()
    yield
    torch.cuda.empty_cache()


def expected_plan(bt, cl, block_size, group, partition_tokens):
    """The grouping rule of pa_decode's shared-prefix mode, written out."""
    S = len(cl)
    max_members = 32 // group

    def first(s):
        if cl[s] <= 0:
            return -1
        return int(bt[s, 0])

    plan = np.zeros((S, 4), dtype=np.int32)
    plan[:, 1] = 1
    s = 0
    while s < S:
        f = first(s)
        end = min(S, (s // CHUNK + 1) * CHUNK)
        b = s + 1
        while f >= 0 and b < end and first(b) == f:
            b += 1
        if f >= 0:
            for lead in range(s, b, max_members):
                members = list(range(lead, min(b, lead + max_members)))
                if len(members) < 2:
                    continue
                min_ctx = min(int(cl[m]) for m in members)
                nb = min(-(-int(cl[m]) // block_size) for m in members)
                common = nb
                for m in members[1:]:
                    j = 0
                    while j < common and bt[m, j] == bt[lead, j]:
                        j += 1
                    common = j
                shared = min(common * block_size, min_ctx) // 16 * 16
                if shared < MIN_SHARED:
                    continue
                gp = -(-shared // partition_tokens)
                for m in members:
                    plan[m] = (m - lead, len(members), shared, gp)
        s = b
    return plan


def expected_plan2(plan, cl, partition_tokens, own_partition_tokens):
    """Second plan record: {own-row offset in the group's row list (-1: read
    on their own), partial count, rows of the own tokens read on their own
    (-1: none, or in the list), rows of the list the sequence leads (-1: it
    leads no group of two or more)}.  A group folds its members' own tokens
    into its list when, each run rounded up to 16 rows, they total at most
    max(T, 64 x members) rows."""
    PT = partition_tokens
    S = len(cl)
    out = np.zeros((S, 4), dtype=np.int32)
    s = 0
    while s < S:
        rank, n, T, p_sh = (int(x) for x in plan[s])
        assert rank == 0
        members = list(range(s, s + n))
        runs = [-(-(int(cl[m]) - T) // 16) * 16 for m in members]
        fold = n >= 2 and sum(runs) <= max(T, 64 * n)
        off = T
        offs = []
        for r in runs:
            offs.append(off)
            off += r
        rows = off if fold else T
        for i, m in enumerate(members):
            own = int(cl[m]) - T
            slots = p_sh
            if own > 0:
                if fold:
                    first, last = max(offs[i] // PT, p_sh), (offs[i] + own - 1) // PT
                    slots += max(0, last - first + 1)
                else:
                    slots += -(-own // own_partition_tokens)
            own_rows = own if not fold and (n == 1 or own > 0) else -1
            out[m] = (offs[i] if fold else -1, slots, own_rows, rows if i == 0 and n >= 2 else -1)
        s += n
    return out


def run_shared(c, dtype, partition_tokens=0, poison_ws=True):
    """pa_decode with shared_prefix; returns (out bits, plan left in the workspace)."""
    shape = shape_of(dtype, c["q"], c["k_cache"], c["block_tables"], partition_tokens, SHARED)
    maxlen = int(np.max(c["context_lens"], initial=0))
    wsb = pa.pa_decode_workspace_bytes(shape, maxlen)
    assert wsb > 0
    if poison_ws:
        # the workspace needs no initialisation: start from arbitrary bytes
        ws = torch.randint(0, 256, (wsb,), dtype=torch.uint8, device="cuda")
    else:
        ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    out = torch.full(c["q"].shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    pa.pa_decode(dev(c["q"], dtype), dev(c["k_cache"], dtype), dev(c["v_cache"], dtype),
                 dev_i32(c["block_tables"]), dev_i32(c["context_lens"]), c["scale"], out, shape,
                 maxlen, ws, wsb)
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_OK, f"device check fired: {bits:#x}"
    S = c["q"].shape[0]
    rec = -(-16 * S // 256) * 256
    plan = ws[256:256 + 16 * S].cpu().numpy().view(np.int32).reshape(S, 4)
    plan2 = ws[256 + rec:256 + rec + 16 * S].cpu().numpy().view(np.int32).reshape(S, 4)
    pt = pa.pa_decode_partition_tokens(shape)
    # own tokens read on their own: the kernel the shape gets without shared
    # prefixes, the tensor-core one in partitions of pt, the CUDA-core one in
    # its largest partitions (2048 tokens)
    plain = shape_of(dtype, c["q"], c["k_cache"], c["block_tables"], partition_tokens)
    own_pt = pt if pa.pa_decode_resolved_variant(plain) == pa.PA_DECODE_TENSOR_CORES else 2048
    exp2 = expected_plan2(plan, c["context_lens"], pt, own_pt)
    assert np.array_equal(plan2, exp2), f"second plan record differs:\n{plan2}\nexpected\n{exp2}"
    return host_bits(out), plan


def groups_for(rng, group):
    """Groups that reach every branch of the plan and of the shared kernel."""
    mm = 32 // group
    g = []
    g.append((700, [700 + int(x) for x in rng.integers(1, 40, size=mm + 3)]))  # run > max members
    g.append((256, [256, 256 + 5]))            # a member with no own tokens
    g.append((100, [110, 120]))                # too short to share
    g.append((128, [128, 129, 200][:max(2, min(3, mm))]))  # exactly one tile
    g.append((0, [0]))                         # empty context breaks a run
    g.append((129, [150, 170]))
    g.append((1000, [1030, 500]))              # a member shorter than the shared part
    g.append((2049, [2100, 2060]))             # several shared partitions
    g.append((0, [37]))                        # alone
    g.append((300, [310, 305, 301, 300][:max(2, min(4, mm))]))  # beam-like
    g.append((200, [800, 700]))                # long own tokens: read on their own
    g.append((512, [1000, 600, 530][:max(2, min(3, mm))]))  # a long shared prompt, long continuations
    return g


@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("block_size", [8, 16, 256])
def test_shared_prefix_groups(orc, dtype, group, block_size):
    rng = np.random.default_rng(9000 + 10 * group + block_size + dtype)
    c = gen.grouped_decode_case(rng, groups=groups_for(rng, group), num_q_heads=2 * group,
                                num_kv_heads=2, head_dim=128, block_size=block_size, dtype=dtype)
    out, plan = run_shared(c, dtype)
    exp = expected_plan(c["block_tables"], c["context_lens"], block_size, group, 512)
    assert np.array_equal(plan, exp), f"plan differs:\n{plan}\nexpected\n{exp}"
    assert (exp[:, 1] >= 2).any(), "the case must form groups"
    ref = orc.decode(dtype, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, dtype, f"shared g{group} bs{block_size}")


@pytest.mark.parametrize("partition_tokens", [128, 256, 384, 512])
def test_shared_prefix_partitions(orc, partition_tokens):
    rng = np.random.default_rng(9100 + partition_tokens)
    groups = [(1500, [1500 + int(x) for x in rng.integers(0, 700, size=4)]),
              (400, [401, 402, 900, 403]), (130, [130, 131])]
    c = gen.grouped_decode_case(rng, groups=groups, num_q_heads=16, num_kv_heads=2, head_dim=128,
                                block_size=16, dtype=gen.BF16)
    out, plan = run_shared(c, gen.BF16, partition_tokens)
    exp = expected_plan(c["block_tables"], c["context_lens"], 16, 8, partition_tokens)
    assert np.array_equal(plan, exp)
    ref = orc.decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.BF16, f"shared pt{partition_tokens}")


def test_shared_prefix_groups_stay_inside_launch_windows(orc):
    """A run that crosses sequence 256 is cut there (two launches of the shared kernel)."""
    rng = np.random.default_rng(9200)
    groups = [(0, [int(x) for x in rng.integers(1, 40, size=250)]),
              (300, [300 + int(x) for x in rng.integers(0, 30, size=12)]),
              (200, [220, 230, 240])]
    c = gen.grouped_decode_case(rng, groups=groups, num_q_heads=2, num_kv_heads=2, head_dim=128,
                                block_size=16, dtype=gen.F16)
    # the first group of singles shares nothing; give them distinct first blocks
    assert len(np.unique(c["block_tables"][:250, 0])) == 250
    out, plan = run_shared(c, gen.F16)
    exp = expected_plan(c["block_tables"], c["context_lens"], 16, 1, 512)
    assert np.array_equal(plan, exp)
    assert exp[255, 1] == 6 and exp[256, 1] == 6 and exp[256, 0] == 0
    ref = orc.decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.F16, "shared across launch windows")


def test_shared_prefix_deterministic_and_layout_free(orc):
    """Bit-identical on a rerun and under any relabelling of physical blocks."""
    rng = np.random.default_rng(9300)
    c = gen.grouped_decode_case(rng, groups=groups_for(rng, 8), num_q_heads=16, num_kv_heads=2,
                                head_dim=128, block_size=16, dtype=gen.BF16)
    a, _ = run_shared(c, gen.BF16)
    b, _ = run_shared(c, gen.BF16, poison_ws=False)
    assert np.array_equal(a, b)
    pi = rng.permutation(c["num_blocks"])
    kc, vc = np.empty_like(c["k_cache"]), np.empty_like(c["v_cache"])
    kc[pi], vc[pi] = c["k_cache"], c["v_cache"]
    bt = c["block_tables"].copy()
    bt[bt >= 0] = pi[bt[bt >= 0]]
    p, _ = run_shared(dict(c, k_cache=kc, v_cache=vc, block_tables=bt), gen.BF16)
    assert np.array_equal(a, p)


def test_shared_prefix_matches_plain_decode(orc):
    """Same inputs without shared_prefix: both within tolerance of the oracle."""
    rng = np.random.default_rng(9400)
    c = gen.grouped_decode_case(rng, groups=[(600, [610, 620, 630, 640])] * 3, num_q_heads=64,
                                num_kv_heads=8, head_dim=128, block_size=16, dtype=gen.BF16)
    shared, _ = run_shared(c, gen.BF16)
    plain, _, _ = gpu_decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                             c["context_lens"], c["scale"])
    ref = orc.decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(shared, ref, gen.BF16, "shared")
    assert_decode_close(plain, ref, gen.BF16, "plain")


def test_shared_prefix_bad_block_ids_reported():
    """An out-of-pool entry in a shared prefix is reported, not followed."""
    rng = np.random.default_rng(9500)
    c = gen.grouped_decode_case(rng, groups=[(400, [420, 430, 440, 450])], num_q_heads=8,
                                num_kv_heads=1, head_dim=128, block_size=16, dtype=gen.BF16)
    bt = c["block_tables"].copy()
    bt[:, 3] = c["num_blocks"] + 5   # all members: still one shared prefix
    _, status, bits = gpu_decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], bt,
                                 c["context_lens"], c["scale"], expect_ok=False, variant=SHARED)
    assert status == pa.PA_ERR_DEVICE_CHECK and bits & 0x1


@pytest.mark.parametrize("group,launches", [(8, 3), (1, 4)])
def test_shared_prefix_launches(group, launches):
    """plan + the row lists of the groups + merge; where the own tokens read
    on their own go to the tensor cores (group 8) they are items of the list
    launch, else (group 1) the CUDA-core kernel reads them in a launch of its
    own."""
    rng = np.random.default_rng(9600)
    c = gen.grouped_decode_case(rng, groups=[(300, [310, 320]), (0, [45])], num_q_heads=group,
                                num_kv_heads=1, head_dim=128, block_size=16, dtype=gen.BF16)
    before = pa.pa_kernel_launches()
    out, _ = run_shared(c, gen.BF16)
    assert pa.pa_kernel_launches() - before == launches


@pytest.mark.parametrize("group", [1, 8])
def test_shared_prefix_tables_without_entries(group):
    """A batch of empty contexts whose tables hold no entries at all
    (max_blocks_per_seq = 0; the table pointer is valid but names nothing):
    the plan reads no table entry, every output row is zero, and no device
    check fires."""
    rng = np.random.default_rng(9700 + group)
    S, Hkv, D, bs, NB = 5, 1, 128, 16, 4
    dtype = gen.BF16
    q = gen.normal_bits(rng, (S, Hkv * group, D), dtype)
    k = gen.normal_bits(rng, (NB, bs, Hkv, D), dtype)
    v = gen.normal_bits(rng, (NB, bs, Hkv, D), dtype)
    shape = pa.make_shape(num_seqs=S, num_q_heads=Hkv * group, num_kv_heads=Hkv, head_dim=D,
                          block_size=bs, num_blocks=NB, max_blocks_per_seq=0, dtype=dtype,
                          shared_prefix=1)
    wsb = pa.pa_decode_workspace_bytes(shape, 0)
    ws = torch.randint(0, 256, (max(16, wsb),), dtype=torch.uint8, device="cuda")
    out = torch.full(q.shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    no_entries = dev_i32(np.zeros(4, dtype=np.int32))  # a valid pointer, nothing in it is read
    pa.pa_decode(dev(q, dtype), dev(k, dtype), dev(v, dtype), no_entries,
                 dev_i32(np.zeros(S, dtype=np.int32)), 0.088, out, shape, 0, ws, wsb)
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_OK, f"device check fired: {bits:#x}"
    assert np.all(host_bits(out) == 0)
