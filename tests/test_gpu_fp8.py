"""E4M3 (FP8) cache against the CPU oracle, through the C ABI (needs a B200).

pa_cache_append_fp8 must leave the code pools byte-identical to the oracle's
encoding; pa_decode_fp8 must meet the decode tolerance against the oracle's
fp64 result over the same codes and scales; pa_copy_blocks copies 1-byte
blocks bit-exactly.
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


def _u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def _f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _shape(c, dtype, Hq, partition_tokens=0, variant=0):
    NB, bs, Hkv, D = c["k_cache"].shape
    return pa.make_shape(num_seqs=len(c["context_lens"]), num_q_heads=Hq, num_kv_heads=Hkv,
                         head_dim=D, block_size=bs, num_blocks=NB,
                         max_blocks_per_seq=c["block_tables"].shape[1],
                         partition_tokens=partition_tokens, dtype=dtype, variant=variant,
                         cache_format=pa.PA_CACHE_FP8_E4M3)


def _scales(rng, Hkv):
    return (rng.uniform(0.004, 0.02, Hkv).astype(np.float32),
            rng.uniform(0.004, 0.02, Hkv).astype(np.float32))


def _quantised_case(orc, rng, dtype, Hq, Hkv, D, bs, ctx):
    """A paged case whose pools the oracle has encoded to E4M3 from N(0,1) values."""
    c = gen.random_decode_case(rng, num_seqs=len(ctx), num_q_heads=Hq, num_kv_heads=Hkv,
                               head_dim=D, block_size=bs, dtype=dtype, context_lens=ctx,
                               poison=False)
    return _quantise(orc, rng, c, dtype)


def _quantise(orc, rng, c, dtype):
    """The case with both pools encoded to E4M3 by the oracle (per-head scales)."""
    NB, bs, Hkv, D = c["k_cache"].shape
    ks, vs = _scales(rng, Hkv)
    kc = np.zeros((NB, bs, Hkv, D), dtype=np.uint8)
    vc = np.zeros_like(kc)
    slots = np.arange(NB * bs, dtype=np.int32)
    orc.cache_append_fp8(dtype, c["k_cache"].reshape(NB * bs, Hkv, D),
                         c["v_cache"].reshape(NB * bs, Hkv, D), slots, ks, vs, kc, vc)
    # slots no sequence holds get the E4M3 NaN code: a read past a context shows
    valid = gen.valid_slot_mask(c["block_tables"], c["context_lens"], NB, bs)
    kc.reshape(NB * bs, -1)[~valid] = 0x7F
    vc.reshape(NB * bs, -1)[~valid] = 0x7F
    return dict(c, k_cache=kc, v_cache=vc, k_scale=ks, v_scale=vs)


def _gpu_decode_fp8(c, dtype, Hq, partition_tokens=0, variant=0, shared_prefix=0):
    shape = _shape(c, dtype, Hq, partition_tokens, variant)
    shape.shared_prefix = shared_prefix
    maxlen = int(np.max(c["context_lens"], initial=0))
    wsb = pa.pa_decode_workspace_bytes(shape, maxlen)
    ws = torch.empty(max(16, wsb), dtype=torch.uint8, device="cuda")
    out = torch.full(c["q"].shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    pa.pa_decode_fp8(dev(c["q"], dtype), _u8(c["k_cache"]), _u8(c["v_cache"]), _f32(c["k_scale"]),
                     _f32(c["v_scale"]), dev_i32(c["block_tables"]), dev_i32(c["context_lens"]),
                     c["scale"], out, shape, maxlen, ws, wsb)
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_OK, f"device check fired: {bits:#x}"
    return host_bits(out)


@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
def test_fp8_append_bit_exact(orc, dtype, head_dim):
    rng = np.random.default_rng(700 + 10 * dtype + head_dim)
    NB, bs, Hkv, D, T = 24, 16, 4, head_dim, 60
    ks, vs = _scales(rng, Hkv)
    k = gen.normal_bits(rng, (T, Hkv, D), dtype)
    v = gen.normal_bits(rng, (T, Hkv, D), dtype)
    # edge values: saturating, tiny (subnormal codes), zeros, exact ties
    kf = gen.bits_to_f32(k, dtype)
    kf[0, :, :8] = 1e4
    kf[1, :, :8] = -1e4
    kf[2, :, :8] = 1e-5
    kf[3, :, :8] = -0.0
    k[:4] = gen.to_bits(kf[:4], dtype)
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int32)
    slots[[5, 17]] = -1
    kc0 = rng.integers(0, 256, size=(NB, bs, Hkv, D), dtype=np.uint8)
    vc0 = rng.integers(0, 256, size=(NB, bs, Hkv, D), dtype=np.uint8)
    shape = pa.make_shape(num_seqs=1, num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                          num_blocks=NB, max_blocks_per_seq=1, dtype=dtype,
                          cache_format=pa.PA_CACHE_FP8_E4M3)
    dk, dv = _u8(kc0), _u8(vc0)
    pa.pa_cache_append_fp8(dev(k, dtype), dev(v, dtype), dev_i32(slots), T, dk, dv, _f32(ks),
                           _f32(vs), shape)
    assert pa.pa_last_device_error()[0] == pa.PA_OK
    ek, ev = kc0.copy(), vc0.copy()
    orc.cache_append_fp8(dtype, k, v, slots, ks, vs, ek, ev)
    gk, gv = dk.cpu().numpy(), dv.cpu().numpy()
    assert np.array_equal(gk, ek), f"{int((gk != ek).sum())} K codes differ"
    assert np.array_equal(gv, ev), f"{int((gv != ev).sum())} V codes differ"


def test_fp8_append_ties_and_every_code(orc):
    """Every finite code value, and every midpoint between neighbours, through append."""
    vals = np.array([orc.e4m3_to_f64(c) for c in range(256)])
    finite = vals[~np.isnan(vals)]
    mids = (np.sort(finite)[:-1] + np.sort(finite)[1:]) / 2
    x = np.concatenate([finite, mids, [500.0, -500.0, 449.0]]).astype(np.float32)
    D, Hkv = 64, 1
    T = -(-len(x) // D)
    xf = np.zeros(T * D, dtype=np.float32)
    xf[:len(x)] = x
    bits = gen.to_bits(xf.reshape(T, Hkv, D), gen.F16)   # all exact in fp16
    assert np.array_equal(gen.bits_to_f32(bits, gen.F16).ravel()[:len(x)], x)
    one = np.ones(Hkv, dtype=np.float32)
    NB, bs = 2, 16
    shape = pa.make_shape(num_seqs=1, num_q_heads=1, num_kv_heads=1, head_dim=D, block_size=bs,
                          num_blocks=NB, max_blocks_per_seq=1, dtype=gen.F16,
                          cache_format=pa.PA_CACHE_FP8_E4M3)
    slots = np.arange(T, dtype=np.int32)
    dk = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8, device="cuda")
    dv = torch.zeros_like(dk)
    pa.pa_cache_append_fp8(dev(bits, gen.F16), dev(bits, gen.F16), dev_i32(slots), T, dk, dv,
                           _f32(one), _f32(one), shape)
    ek = np.zeros((NB, bs, Hkv, D), dtype=np.uint8)
    ev = ek.copy()
    orc.cache_append_fp8(gen.F16, bits, bits, slots, one, one, ek, ev)
    assert np.array_equal(dk.cpu().numpy(), ek) and np.array_equal(dv.cpu().numpy(), ev)


EDGE_CTX = [0, 1, 15, 16, 17, 33, 511, 512, 513, 1025, 2049]


@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("head_dim", [64, 128])
@pytest.mark.parametrize("group", [1, 4, 8, 16])
def test_fp8_decode_edge_contexts(orc, dtype, head_dim, group):
    rng = np.random.default_rng(800 + 7 * group + head_dim + dtype)
    Hkv = 2
    c = _quantised_case(orc, rng, dtype, Hkv * group, Hkv, head_dim, 16, EDGE_CTX)
    out = _gpu_decode_fp8(c, dtype, Hkv * group)
    ref = orc.decode_fp8(dtype, c["q"], c["k_cache"], c["v_cache"], c["k_scale"], c["v_scale"],
                         c["block_tables"], c["context_lens"], c["scale"])
    assert_decode_close(out, ref, dtype, f"fp8 g{group} D{head_dim}")
    assert np.all(out[0] == 0)


@pytest.mark.parametrize("partition_tokens", [16, 128, 512, 2048])
@pytest.mark.parametrize("block_size", [16, 256])
def test_fp8_decode_partitions_and_blocks(orc, partition_tokens, block_size):
    rng = np.random.default_rng(900 + partition_tokens + block_size)
    ctx = [1, 47, 256, 257, 700, 2048, 2100]
    c = _quantised_case(orc, rng, gen.BF16, 8, 2, 128, block_size, ctx)
    out = _gpu_decode_fp8(c, gen.BF16, 8, partition_tokens)
    ref = orc.decode_fp8(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["k_scale"], c["v_scale"],
                         c["block_tables"], c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.BF16, f"fp8 bs{block_size} pt{partition_tokens}")


@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("block_size", [8, 16])
@pytest.mark.parametrize("variant", [1, 2], ids=["cuda_cores", "tensor_cores"])
def test_fp8_decode_variants(orc, dtype, group, block_size, variant):
    """Both kernels on an E4M3 cache: the tensor-core one widens each tile to
    16 bits in shared memory (one head per item, or two)."""
    rng = np.random.default_rng(1200 + 11 * group + block_size + 3 * variant + dtype)
    for Hkv in (2, 3):
        c = _quantised_case(orc, rng, dtype, Hkv * group, Hkv, 128, block_size, EDGE_CTX)
        for pt in (0, 128):
            out = _gpu_decode_fp8(c, dtype, Hkv * group, pt, variant)
            ref = orc.decode_fp8(dtype, c["q"], c["k_cache"], c["v_cache"], c["k_scale"],
                                 c["v_scale"], c["block_tables"], c["context_lens"], c["scale"])
            assert_decode_close(out, ref, dtype,
                                f"fp8 v{variant} g{group} bs{block_size} Hkv{Hkv} pt{pt}")
            assert np.all(out[0] == 0)


@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
@pytest.mark.parametrize("group", [1, 4, 8])
def test_fp8_shared_prefix(orc, dtype, group):
    """Shared prefixes on an E4M3 cache: groups read once, own tokens after."""
    rng = np.random.default_rng(1300 + group + dtype)
    mm = 32 // group
    groups = [(700, [700 + int(x) for x in rng.integers(1, 40, size=mm + 2)]),
              (256, [256, 261]), (100, [110, 120]), (0, [0]), (1000, [1030, 500]),
              (300, [310, 305, 301, 300][:max(2, min(4, mm))]), (0, [37])]
    c = gen.grouped_decode_case(rng, groups=groups, num_q_heads=2 * group, num_kv_heads=2,
                                head_dim=128, block_size=16, dtype=dtype, poison=False)
    c = _quantise(orc, rng, c, dtype)
    out = _gpu_decode_fp8(c, dtype, 2 * group, shared_prefix=1)
    ref = orc.decode_fp8(dtype, c["q"], c["k_cache"], c["v_cache"], c["k_scale"], c["v_scale"],
                         c["block_tables"], c["context_lens"], c["scale"])
    assert_decode_close(out, ref, dtype, f"fp8 shared g{group}")


def test_fp8_step_append_copy_decode(orc):
    """One beam-workload step on an E4M3 cache: copy-on-write, append, decode."""
    case = gen.make_case("llama2_70b_beam", n_steps=1, poison=False, num_seqs=32)
    st = case.steps[0]
    rng = np.random.default_rng(1000)
    NB, bs, Hkv, D = case.k_cache.shape
    ks, vs = _scales(rng, Hkv)
    kc = np.zeros((NB, bs, Hkv, D), dtype=np.uint8)
    vc = np.zeros_like(kc)
    slots = np.arange(NB * bs, dtype=np.int32)
    orc.cache_append_fp8(case.dtype, case.k_cache.reshape(NB * bs, Hkv, D),
                         case.v_cache.reshape(NB * bs, Hkv, D), slots, ks, vs, kc, vc)
    shape = pa.make_shape(num_seqs=case.num_seqs, num_q_heads=case.num_q_heads, num_kv_heads=Hkv,
                          head_dim=D, block_size=bs, num_blocks=NB,
                          max_blocks_per_seq=case.max_blocks_per_seq, dtype=case.dtype,
                          cache_format=pa.PA_CACHE_FP8_E4M3)
    dk, dv = _u8(kc), _u8(vc)
    dks, dvs = _f32(ks), _f32(vs)
    pa.pa_copy_blocks(dev_i32(st.pairs), len(st.pairs), dk, dv, shape)
    pa.pa_cache_append_fp8(dev(st.k_new, case.dtype), dev(st.v_new, case.dtype),
                           dev_i32(st.slot_mapping), case.num_seqs, dk, dv, dks, dvs, shape)
    maxlen = int(st.context_lens.max())
    wsb = pa.pa_decode_workspace_bytes(shape, maxlen)
    ws = torch.empty(max(16, wsb), dtype=torch.uint8, device="cuda")
    out = torch.empty(st.q.shape, dtype=pa.torch_dtype(case.dtype), device="cuda")
    pa.pa_decode_fp8(dev(st.q, case.dtype), dk, dv, dks, dvs, dev_i32(st.block_tables),
                     dev_i32(st.context_lens), case.scale, out, shape, maxlen, ws, wsb)
    assert pa.pa_last_device_error()[0] == pa.PA_OK
    assert len(st.pairs) > 0
    orc.copy_blocks(st.pairs, kc, vc)
    orc.cache_append_fp8(case.dtype, st.k_new, st.v_new, st.slot_mapping, ks, vs, kc, vc)
    assert np.array_equal(dk.cpu().numpy(), kc) and np.array_equal(dv.cpu().numpy(), vc)
    ref = orc.decode_fp8(case.dtype, st.q, kc, vc, ks, vs, st.block_tables, st.context_lens,
                         case.scale)
    assert_decode_close(host_bits(out), ref, case.dtype, "fp8 beam step")


def test_fp8_entry_points_must_match_the_format(orc):
    rng = np.random.default_rng(1100)
    c = _quantised_case(orc, rng, gen.F16, 4, 4, 64, 16, [5, 9])
    shape16 = pa.make_shape(num_seqs=2, num_q_heads=4, num_kv_heads=4, head_dim=64, block_size=16,
                            num_blocks=c["num_blocks"], max_blocks_per_seq=1, dtype=gen.F16)
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    out = torch.empty(c["q"].shape, dtype=torch.float16, device="cuda")
    with pytest.raises(pa.PaError) as e:   # 16-bit shape through the FP8 entry point
        pa.pa_decode_fp8(dev(c["q"], gen.F16), _u8(c["k_cache"]), _u8(c["v_cache"]),
                         _f32(c["k_scale"]), _f32(c["v_scale"]), dev_i32(c["block_tables"]),
                         dev_i32(c["context_lens"]), c["scale"], out, shape16, 9, ws, 4096)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PaError) as e:   # FP8 shape through pa_decode
        pa.pa_decode(dev(c["q"], gen.F16), _u8(c["k_cache"]), _u8(c["v_cache"]),
                     dev_i32(c["block_tables"]), dev_i32(c["context_lens"]), c["scale"], out,
                     _shape(c, gen.F16, 4), 9, ws, 4096)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
