"""CUDA path against the CPU oracle, through the C ABI (needs a B200).

Decode outputs must meet the tolerance in tests/tolerance.py element by
element; append and copy-on-write must leave the whole pool byte-identical
to the oracle's.  Every pool slot that holds no token is NaN, so a read past
a context or through a stale table entry shows up as NaN.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from paged_kv_cache_458_b200 import gen, pa  # noqa: E402
import golden_cases  # noqa: E402
from gpu_util import MODES, SHARED, dev, dev_i32, gpu_decode, host_bits, shape_of  # noqa: E402
from tolerance import assert_decode_close  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_458_b200 import build

    build.build()
    pa.pa_last_device_error()  # start from a clean error word
    yield
    torch.cuda.empty_cache()


def _oracle_decode(orc, dtype, q, kc, vc, bt, cl, scale):
    return orc.decode(dtype, q, kc, vc, bt, cl, scale)


# ---------------------------------------------------------------- golden


@pytest.mark.parametrize("case", golden_cases.load_cases(), ids=lambda c: c["name"])
def test_golden_block_mapping(case):
    c = golden_cases.build(case)
    out, _, _ = gpu_decode(c["dtype"], c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"])
    assert_decode_close(out, c["expected"], c["dtype"], case["name"])


# ---------------------------------------------------------------- full workloads


VARIANTS = MODES


@pytest.fixture(scope="module")
def workload_refs(orc):
    """Each workload's inputs and oracle results, built once per module."""
    cache = {}

    def get(name):
        if name not in cache:
            case = gen.make_case(name, n_steps=1, poison=True)
            st = case.steps[0]
            ref0 = orc.decode(case.dtype, case.q, case.k_cache, case.v_cache, case.block_tables,
                              case.context_lens, case.scale)
            hk, hv = case.k_cache.copy(), case.v_cache.copy()
            orc.copy_blocks(st.pairs, hk, hv)
            orc.cache_append(st.k_new, st.v_new, st.slot_mapping, hk, hv)
            ref1 = orc.decode(case.dtype, st.q, hk, hv, st.block_tables, st.context_lens, case.scale)
            cache.clear()  # keep one workload's pools in host memory at a time
            cache[name] = (case, ref0, hk, hv, ref1)
        return cache[name]

    return get


def _run_workload(workload_refs, name, variant=0):
    case, ref0, hk, hv, ref1 = workload_refs(name)
    dtype, S = case.dtype, case.num_seqs
    st = case.steps[0]
    maxlen = int(st.context_lens.max())
    shape = shape_of(dtype, case.q, case.k_cache, case.block_tables, variant=variant)
    kc, vc = dev(case.k_cache, dtype), dev(case.v_cache, dtype)
    ws = torch.empty(max(16, pa.pa_decode_workspace_bytes(shape, maxlen)), dtype=torch.uint8,
                     device="cuda")
    out0 = torch.empty(case.q.shape, dtype=pa.torch_dtype(dtype), device="cuda")
    out1 = torch.empty_like(out0)
    # decode of the initial state
    pa.pa_decode(dev(case.q, dtype), kc, vc, dev_i32(case.block_tables), dev_i32(case.context_lens),
                 case.scale, out0, shape, int(case.context_lens.max()), ws)
    # one step: copy-on-write, append, decode
    pa.pa_copy_blocks(dev_i32(st.pairs), len(st.pairs), kc, vc, shape)
    pa.pa_cache_append(dev(st.k_new, dtype), dev(st.v_new, dtype), dev_i32(st.slot_mapping), S,
                       kc, vc, shape)
    pa.pa_decode(dev(st.q, dtype), kc, vc, dev_i32(st.block_tables), dev_i32(st.context_lens),
                 case.scale, out1, shape, maxlen, ws)
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_OK, f"device check fired: {bits:#x}"
    assert np.array_equal(host_bits(kc).reshape(hk.shape), hk), "K pool differs after copy+append"
    assert np.array_equal(host_bits(vc).reshape(hv.shape), hv), "V pool differs after copy+append"
    s0 = assert_decode_close(host_bits(out0), ref0, dtype, f"{name} initial decode")
    s1 = assert_decode_close(host_bits(out1), ref1, dtype, f"{name} step decode")
    return case, s0, s1


def test_tiny_workload(workload_refs):
    case, s0, s1 = _run_workload(workload_refs, "tiny")
    assert case.steps[0].context_lens.tolist() == [2, 16, 17, 38]


@pytest.mark.parametrize("name", ["llama2_7b", "mistral_7b_gqa", "qwen_7b_prefix", "llama2_70b_beam"])
@pytest.mark.parametrize("variant", [0, 1, 2, SHARED], ids=lambda v: VARIANTS[v])
def test_full_workload(workload_refs, name, variant):
    case, s0, s1 = _run_workload(workload_refs, name, variant)
    if name == "llama2_70b_beam":
        assert len(case.steps[0].pairs) > 0, "the beam step must exercise copy-on-write"
    print(f"{name} [{VARIANTS[variant]}]: initial {s0}  step {s1}")


# ---------------------------------------------------------------- edge cases

EDGE_CTX = [0, 1, 15, 16, 17, 31, 33, 511, 512, 513, 1023, 1024, 1025, 2047, 2049]


@pytest.mark.parametrize("variant", [1, 2, SHARED], ids=lambda v: VARIANTS[v])
@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("group", [1, 2, 4, 8, 16])
def test_edge_contexts(orc, dtype, head_dim, group, variant):
    if variant in (2, SHARED) and head_dim != 128:
        pytest.skip("the tensor-core kernels are built for head_dim 128")
    rng = np.random.default_rng(1000 * group + head_dim + dtype)
    Hkv = 2
    c = gen.random_decode_case(rng, num_seqs=len(EDGE_CTX), num_q_heads=Hkv * group,
                               num_kv_heads=Hkv, head_dim=head_dim, block_size=16, dtype=dtype,
                               context_lens=EDGE_CTX)
    out, _, _ = gpu_decode(dtype, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"], variant=variant)
    ref = orc.decode(dtype, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, dtype, f"g{group} D{head_dim} {VARIANTS[variant]}")
    assert np.all(out[0] == 0), "an empty context must give a zero row"


@pytest.mark.parametrize("variant", [1, 2, SHARED], ids=lambda v: VARIANTS[v])
@pytest.mark.parametrize("block_size", [8, 16, 32, 256])
@pytest.mark.parametrize("partition_tokens", [16, 48, 128, 256, 512, 2048])
def test_block_and_partition_sizes(orc, block_size, partition_tokens, variant):
    if variant in (2, SHARED) and (partition_tokens % 128 or partition_tokens > 512):
        pytest.skip("the tensor-core kernels take partitions of 128, 256, 384 or 512 tokens")
    rng = np.random.default_rng(block_size * 7 + partition_tokens)
    ctx = [1, 47, 48, 49, 255, 256, 257, 700, 2048, 2100]
    c = gen.random_decode_case(rng, num_seqs=len(ctx), num_q_heads=8, num_kv_heads=2,
                               head_dim=128, block_size=block_size, dtype=gen.BF16,
                               context_lens=ctx, shared_prefix_blocks=1)
    out, _, _ = gpu_decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"], partition_tokens=partition_tokens,
                           variant=variant)
    ref = orc.decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.BF16, f"bs{block_size} pt{partition_tokens}")


@pytest.mark.parametrize("variant", [1, 2, SHARED], ids=lambda v: VARIANTS[v])
def test_last_physical_block_and_stale_entries(orc, variant):
    rng = np.random.default_rng(3)
    c = gen.random_decode_case(rng, num_seqs=3, num_q_heads=4, num_kv_heads=4, head_dim=128,
                               block_size=16, dtype=gen.F16, context_lens=[20, 5, 33])
    NB = c["num_blocks"]
    bt = np.full((3, 8), -1, dtype=np.int32)
    bt[:, :c["block_tables"].shape[1]] = c["block_tables"]
    # move sequence 0's second block to the last physical block of the pool
    old = bt[0, 1]
    last = NB - 1
    other = np.argwhere(bt == last)
    kc, vc = c["k_cache"], c["v_cache"]
    kc[[old, last]] = kc[[last, old]]
    vc[[old, last]] = vc[[last, old]]
    if len(other):
        bt[tuple(other[0])] = old
    bt[0, 1] = last
    bt[1, 1:] = 1 << 30      # stale entries past the context: never read
    bt[2, 3:] = -7
    out, _, _ = gpu_decode(gen.F16, c["q"], kc, vc, bt, c["context_lens"], c["scale"],
                           max_context_len=64, variant=variant)
    ref = orc.decode(gen.F16, c["q"], kc, vc, bt, c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.F16, "last block / stale entries")


def test_all_contexts_empty():
    c = gen.random_decode_case(np.random.default_rng(4), num_seqs=5, num_q_heads=8, num_kv_heads=1,
                               head_dim=128, block_size=16, dtype=gen.BF16, context_lens=[0] * 5)
    out, _, _ = gpu_decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"], max_context_len=0)
    assert np.all(out == 0)


@pytest.mark.parametrize("variant", [1, 2, SHARED], ids=lambda v: VARIANTS[v])
def test_permutation_invariance_and_determinism(variant):
    rng = np.random.default_rng(5)
    c = gen.random_decode_case(rng, num_seqs=6, num_q_heads=16, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=gen.BF16, context_lens=[3, 100, 513, 1500, 64, 900])
    args = (c["q"], c["k_cache"], c["v_cache"], c["block_tables"], c["context_lens"], c["scale"])
    a, _, _ = gpu_decode(gen.BF16, *args, variant=variant)
    b, _, _ = gpu_decode(gen.BF16, *args, variant=variant)
    assert np.array_equal(a, b), "decode is not deterministic"
    pi = rng.permutation(c["num_blocks"])
    kc = np.empty_like(c["k_cache"])
    vc = np.empty_like(c["v_cache"])
    kc[pi], vc[pi] = c["k_cache"], c["v_cache"]
    bt = c["block_tables"].copy()
    bt[bt >= 0] = pi[bt[bt >= 0]]
    p, _, _ = gpu_decode(gen.BF16, c["q"], kc, vc, bt, c["context_lens"], c["scale"],
                         variant=variant)
    assert np.array_equal(a, p), "output depends on where the blocks sit"


# ---------------------------------------------------------------- append / copy


def test_append_and_copy_bit_exact(orc):
    rng = np.random.default_rng(6)
    NB, bs, Hkv, D = 40, 16, 8, 128
    kc = rng.integers(0, 1 << 16, size=(NB, bs, Hkv, D), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, size=(NB, bs, Hkv, D), dtype=np.uint16)
    T = 33
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int32)
    slots[[3, 10]] = -1
    k = rng.integers(0, 1 << 16, size=(T, Hkv, D), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(T, Hkv, D), dtype=np.uint16)
    srcs = rng.choice(NB, size=12, replace=False)
    pairs = np.stack([srcs[:6], srcs[6:]], axis=1).astype(np.int32)
    shape = pa.make_shape(num_seqs=1, num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                          num_blocks=NB, max_blocks_per_seq=1, dtype=pa.PA_F16)
    dk, dv = dev(kc, gen.F16), dev(vc, gen.F16)
    pa.pa_copy_blocks(dev_i32(pairs), len(pairs), dk, dv, shape)
    pa.pa_cache_append(dev(k, gen.F16), dev(v, gen.F16), dev_i32(slots), T, dk, dv, shape)
    assert pa.pa_last_device_error()[0] == pa.PA_OK
    orc.copy_blocks(pairs, kc, vc)
    orc.cache_append(k, v, slots, kc, vc)
    assert np.array_equal(host_bits(dk).reshape(kc.shape), kc)
    assert np.array_equal(host_bits(dv).reshape(vc.shape), vc)


# ---------------------------------------------------------------- device checks


def test_device_checks_report_and_skip():
    rng = np.random.default_rng(8)
    c = gen.random_decode_case(rng, num_seqs=2, num_q_heads=2, num_kv_heads=2, head_dim=64,
                               block_size=16, dtype=gen.F16, context_lens=[40, 10], poison=False)
    NB = c["num_blocks"]
    bt = c["block_tables"].copy()
    bt[0, 1] = NB + 3
    out, st, bits = gpu_decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], bt, c["context_lens"],
                               c["scale"], expect_ok=False)
    assert st == pa.PA_ERR_DEVICE_CHECK and bits & pa.PA_DEVERR_BLOCK_ID
    assert np.all(np.isfinite(gen.bits_to_f32(out, gen.F16)))
    bt[0, 1] = -1
    _, st, bits = gpu_decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], bt, c["context_lens"],
                             c["scale"], expect_ok=False)
    assert st == pa.PA_ERR_DEVICE_CHECK and bits & pa.PA_DEVERR_BLOCK_ID
    # context above the host's bound: clamped and reported
    _, st, bits = gpu_decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                             c["context_lens"], c["scale"], max_context_len=20, expect_ok=False)
    assert st == pa.PA_ERR_DEVICE_CHECK and bits & pa.PA_DEVERR_CONTEXT_LEN
    # the word was cleared by the read
    _, st, _ = gpu_decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                          c["context_lens"], c["scale"])
    assert st == pa.PA_OK

    shape = shape_of(gen.F16, c["q"], c["k_cache"], c["block_tables"])
    dk, dv = dev(c["k_cache"], gen.F16), dev(c["v_cache"], gen.F16)
    before = host_bits(dk)
    pa.pa_cache_append(dev(c["k_cache"][0, :2], gen.F16), dev(c["v_cache"][0, :2], gen.F16),
                       dev_i32([NB * 16, -5]), 2, dk, dv, shape)
    st, bits = pa.pa_last_device_error()
    assert st == pa.PA_ERR_DEVICE_CHECK and bits == pa.PA_DEVERR_SLOT
    assert np.array_equal(host_bits(dk), before)
    pa.pa_copy_blocks(dev_i32([[0, NB], [-1, 2]]), 2, dk, dv, shape)
    st, bits = pa.pa_last_device_error()
    assert st == pa.PA_ERR_DEVICE_CHECK and bits == pa.PA_DEVERR_PAIR
    assert np.array_equal(host_bits(dk), before)


def test_launch_counter_counts_kernels():
    rng = np.random.default_rng(9)
    for ctx, pt, kernels in (([600, 10], 256, 2), ([200, 10], 256, 1)):
        c = gen.random_decode_case(rng, num_seqs=2, num_q_heads=2, num_kv_heads=2, head_dim=64,
                                   block_size=16, dtype=gen.F16, context_lens=ctx)
        n0 = pa.pa_kernel_launches()
        gpu_decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                   c["context_lens"], c["scale"], partition_tokens=pt)
        # partition kernel, plus the split-K merge kernel when a context spans partitions
        assert pa.pa_kernel_launches() - n0 == kernels


def test_workspace_needs_no_initialisation(orc):
    """Split-K counters carry a per-call tag: garbage or a previous call's
    values in the workspace must not change the result."""
    rng = np.random.default_rng(10)
    ws = torch.full((8 << 20,), 0xFF, dtype=torch.uint8, device="cuda")
    for trial, (ctx, g) in enumerate((([1500, 700, 33, 2600], 4), ([513, 1024, 4000], 8),
                                      ([1500, 700, 33, 2600], 4))):
        c = gen.random_decode_case(rng, num_seqs=len(ctx), num_q_heads=2 * g, num_kv_heads=2,
                                   head_dim=128, block_size=16, dtype=gen.BF16, context_lens=ctx)
        shape = shape_of(gen.BF16, c["q"], c["k_cache"], c["block_tables"])
        maxlen = int(max(ctx))
        wsb = pa.pa_decode_workspace_bytes(shape, maxlen)
        assert 0 < wsb <= ws.numel()
        if trial == 2:
            ws[:wsb].random_(0, 256)
        out = torch.empty(c["q"].shape, dtype=torch.bfloat16, device="cuda")
        pa.pa_decode(dev(c["q"], gen.BF16), dev(c["k_cache"], gen.BF16), dev(c["v_cache"], gen.BF16),
                     dev_i32(c["block_tables"]), dev_i32(c["context_lens"]), c["scale"], out, shape,
                     maxlen, ws, wsb)
        assert pa.pa_last_device_error()[0] == pa.PA_OK
        ref = orc.decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                         c["context_lens"], c["scale"])
        assert_decode_close(host_bits(out), ref, gen.BF16, f"trial {trial}")


def test_tensor_core_device_checks_and_launches():
    """Bad block ids read as zeros on the tensor-core path too, with the error
    word set; one persistent launch (+ merge) per decode."""
    rng = np.random.default_rng(11)
    c = gen.random_decode_case(rng, num_seqs=3, num_q_heads=16, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=gen.BF16, context_lens=[700, 40, 300],
                               poison=False)
    bt = c["block_tables"].copy()
    bt[0, 3] = c["num_blocks"] + 1
    n0 = pa.pa_kernel_launches()
    out, st, bits = gpu_decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], bt, c["context_lens"],
                               c["scale"], variant=2, expect_ok=False)
    assert pa.pa_kernel_launches() - n0 == 2
    assert st == pa.PA_ERR_DEVICE_CHECK and bits & pa.PA_DEVERR_BLOCK_ID
    assert np.all(np.isfinite(gen.bits_to_f32(out, gen.BF16)))


def test_tensor_core_batches_beyond_one_launch(orc):
    """More than 256 sequences run as several persistent launches (256 each)."""
    rng = np.random.default_rng(12)
    ctx = rng.integers(0, 300, size=600)
    c = gen.random_decode_case(rng, num_seqs=600, num_q_heads=8, num_kv_heads=1, head_dim=128,
                               block_size=16, dtype=gen.F16, context_lens=ctx)
    n0 = pa.pa_kernel_launches()
    out, _, _ = gpu_decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"], variant=2)
    # 600 = 256 + 256 + 88; every context fits one partition (no merge)
    assert pa.pa_kernel_launches() - n0 == 3
    ref = orc.decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.F16, "600 sequences")
