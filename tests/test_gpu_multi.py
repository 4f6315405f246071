"""Several query tokens per sequence (pa_decode_multi) against the CPU oracle.

Query token t of a sequence with Tq new tokens attends causally to tokens
0 .. ctx - Tq + t.  Tokens beyond each query's range are NaN in these pools,
so a read past the causal limit shows up as NaN.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from paged_kv_cache_458_b200 import gen, pa  # noqa: E402
from gpu_util import dev, dev_i32, host_bits  # noqa: E402
from tolerance import assert_decode_close  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_cache_458_b200 import build

    build.build()
    pa.pa_last_device_error()
    yield
    torch.cuda.empty_cache()


def _case(seed, Tq, ctx, group, head_dim, dtype, block_size=16, shared_prefix_blocks=0, Hkv=2):
    rng = np.random.default_rng(seed)
    c = gen.random_decode_case(rng, num_seqs=len(ctx), num_q_heads=Hkv * group, num_kv_heads=Hkv,
                               head_dim=head_dim, block_size=block_size, dtype=dtype,
                               context_lens=ctx, shared_prefix_blocks=shared_prefix_blocks)
    q = gen.normal_bits(rng, (len(ctx), Tq, Hkv * group, head_dim), dtype)
    return dict(c, q=q)


def _gpu_multi(c, dtype, Tq, partition_tokens=0, variant=0):
    S, _, Hq, D = c["q"].shape
    NB, bs, Hkv, _ = c["k_cache"].shape
    shape = pa.make_shape(num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                          num_blocks=NB, max_blocks_per_seq=c["block_tables"].shape[1],
                          partition_tokens=partition_tokens, dtype=dtype, variant=variant)
    maxlen = int(np.max(c["context_lens"], initial=0))
    wsb = pa.pa_decode_multi_workspace_bytes(shape, Tq, maxlen)
    assert wsb > 0
    ws = torch.randint(0, 256, (wsb,), dtype=torch.uint8, device="cuda")  # no initialisation needed
    out = torch.full(c["q"].shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    pa.pa_decode_multi(dev(c["q"], dtype), dev(c["k_cache"], dtype), dev(c["v_cache"], dtype),
                       dev_i32(c["block_tables"]), dev_i32(c["context_lens"]), c["scale"], out,
                       shape, Tq, maxlen, ws, wsb)
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_OK, f"device check fired: {bits:#x}"
    return host_bits(out)


CTX = [1, 2, 4, 7, 16, 17, 130, 511, 512, 600, 1500, 2100]


@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("group", [1, 4, 8])
@pytest.mark.parametrize("Tq", [2, 4, 8])
def test_multi_query_tokens(orc, dtype, head_dim, group, Tq):
    c = _case(1200 + 31 * Tq + 7 * group + head_dim + dtype, Tq, CTX, group, head_dim, dtype)
    out = _gpu_multi(c, dtype, Tq)
    ref = orc.decode_multi(dtype, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"])
    assert_decode_close(out, ref, dtype, f"Tq{Tq} g{group} D{head_dim}")
    # contexts shorter than Tq leave the first queries empty
    assert np.all(out[0, :Tq - 1] == 0) and np.any(out[0, Tq - 1] != 0)


@pytest.mark.parametrize("partition_tokens", [128, 512, 1024])
@pytest.mark.parametrize("variant", [0, 1, 2])
def test_multi_partitions_and_variants(orc, partition_tokens, variant):
    if variant == 2 and partition_tokens > 512:
        pytest.skip("the tensor-core kernel takes partitions up to 512 tokens")
    Tq = 4
    c = _case(1300 + partition_tokens + variant, Tq, [5, 300, 1100, 2050], 8, 128, gen.BF16,
              block_size=256)
    out = _gpu_multi(c, gen.BF16, Tq, partition_tokens, variant)
    ref = orc.decode_multi(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.BF16, f"pt{partition_tokens} v{variant}")


def test_multi_with_shared_prefixes_across_sequences(orc):
    """Sequences that also share a prompt: one run of virtual sequences, several groups."""
    Tq = 3
    c = _case(1400, Tq, [700, 710, 720, 730, 40], 1, 128, gen.F16, shared_prefix_blocks=40)
    out = _gpu_multi(c, gen.F16, Tq)
    ref = orc.decode_multi(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.F16, "multi + shared prompt")


def test_multi_verification_step(orc):
    """A speculative step: append Tq tokens per sequence, then decode them all."""
    Tq, S, D, Hkv, g, bs = 4, 6, 128, 2, 4, 16
    rng = np.random.default_rng(1500)
    ctx0 = rng.integers(20, 400, size=S).astype(np.int32)
    c = gen.random_decode_case(rng, num_seqs=S, num_q_heads=Hkv * g, num_kv_heads=Hkv, head_dim=D,
                               block_size=bs, dtype=gen.BF16, context_lens=ctx0 + Tq, poison=False)
    bt, ctx = c["block_tables"], c["context_lens"]
    slots = np.array([int(bt[s, j // bs]) * bs + j % bs
                      for s in range(S) for j in range(ctx[s] - Tq, ctx[s])], dtype=np.int32)
    k_new = gen.normal_bits(rng, (S * Tq, Hkv, D), gen.BF16)
    v_new = gen.normal_bits(rng, (S * Tq, Hkv, D), gen.BF16)
    q = gen.normal_bits(rng, (S, Tq, Hkv * g, D), gen.BF16)
    NB = c["num_blocks"]
    shape = pa.make_shape(num_seqs=S, num_q_heads=Hkv * g, num_kv_heads=Hkv, head_dim=D,
                          block_size=bs, num_blocks=NB, max_blocks_per_seq=bt.shape[1],
                          dtype=gen.BF16)
    kc, vc = dev(c["k_cache"], gen.BF16), dev(c["v_cache"], gen.BF16)
    pa.pa_cache_append(dev(k_new, gen.BF16), dev(v_new, gen.BF16), dev_i32(slots), S * Tq, kc, vc,
                       shape)
    maxlen = int(ctx.max())
    wsb = pa.pa_decode_multi_workspace_bytes(shape, Tq, maxlen)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    n0 = pa.pa_kernel_launches()
    pa.pa_decode_multi(dev(q, gen.BF16), kc, vc, dev_i32(bt), dev_i32(ctx), c["scale"], out, shape,
                       Tq, maxlen, ws, wsb)
    assert pa.pa_last_device_error()[0] == pa.PA_OK
    # Tq x g = 16 columns: one tensor-core kernel reads every K/V tile once
    # for all four queries (contexts under 512 tokens: no merge)
    assert pa.pa_kernel_launches() - n0 == 1
    hk, hv = c["k_cache"].copy(), c["v_cache"].copy()
    orc.cache_append(k_new, v_new, slots, hk, hv)
    ref = orc.decode_multi(gen.BF16, q, hk, hv, bt, ctx, c["scale"])
    assert_decode_close(host_bits(out), ref, gen.BF16, "verification step")


@pytest.mark.parametrize("Tq,group,Hkv,block_size", [
    (3, 2, 3, 16),    # odd kv heads: one head per item, 6 of 8 columns
    (4, 1, 2, 8),     # 8-token blocks: one head per item, two 8-row boxes per group
    (5, 4, 2, 16),    # 20 of 32 columns
    (2, 16, 2, 16),   # 32 columns of one head
    (8, 1, 4, 16),    # two heads per item, 16 columns
    (7, 2, 2, 256),   # two heads per item, 14 of 16 columns, 256-token blocks
])
def test_multi_one_read_for_all_queries(orc, Tq, group, Hkv, block_size):
    """The tensor-core path that reads each tile once for all Tq queries, with
    the causal limit of every query falling inside, at and across partition
    and tile boundaries."""
    ctx = [1, Tq - 1 if Tq > 1 else 1, Tq, 63 + Tq, 64 + Tq, 127 + Tq, 512, 513, 515, 1030, 1540]
    c = _case(1600 + 13 * Tq + group + Hkv + block_size, Tq, ctx, group, 128, gen.BF16,
              block_size=block_size, Hkv=Hkv)
    for pt in (0, 128):
        out = _gpu_multi(c, gen.BF16, Tq, partition_tokens=pt)
        ref = orc.decode_multi(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                               c["context_lens"], c["scale"])
        assert_decode_close(out, ref, gen.BF16, f"Tq{Tq} g{group} Hkv{Hkv} bs{block_size} pt{pt}")
