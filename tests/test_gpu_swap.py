"""Block swap between the device pool and a pinned host pool, and 8-token
blocks, against the CPU oracle (needs a B200)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from paged_kv_cache_458_b200 import gen, pa  # noqa: E402
from gpu_util import dev, dev_i32, gpu_decode, host_bits  # noqa: E402
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


def _pinned(a, dtype=torch.float16):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dtype)
    return t.pin_memory()


def test_swap_out_and_in_round_trip(orc):
    """Swap a sequence's blocks out to pinned host memory, clobber them on the
    device, swap them back into other device blocks, and decode."""
    rng = np.random.default_rng(1600)
    c = gen.random_decode_case(rng, num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=gen.F16, context_lens=[200, 77, 300],
                               poison=False)
    NB = c["num_blocks"]
    bs, Hkv, D = 16, 2, 128
    shape = pa.make_shape(num_seqs=3, num_q_heads=8, num_kv_heads=2, head_dim=D, block_size=bs,
                          num_blocks=NB, max_blocks_per_seq=c["block_tables"].shape[1],
                          dtype=gen.F16)
    kc, vc = dev(c["k_cache"], gen.F16), dev(c["v_cache"], gen.F16)
    HB = 40
    hk = _pinned(np.zeros((HB, bs, Hkv, D), np.uint16))
    hv = _pinned(np.zeros((HB, bs, Hkv, D), np.uint16))
    # swap sequence 1 out
    seq1 = [int(b) for b in c["block_tables"][1, :(77 + bs - 1) // bs]]
    out_pairs = np.array([[b, i] for i, b in enumerate(seq1)], dtype=np.int32)
    pa.pa_swap_blocks(dev_i32(out_pairs), len(out_pairs), kc, vc, NB, hk, hv, HB, shape)
    torch.cuda.synchronize()
    assert pa.pa_last_device_error()[0] == pa.PA_OK
    ek = np.zeros((HB, bs, Hkv, D), np.uint16)
    ev = np.zeros_like(ek)
    orc.swap_blocks(out_pairs, c["k_cache"], c["v_cache"], ek, ev)
    assert np.array_equal(hk.view(torch.int16).numpy().view(np.uint16), ek)
    assert np.array_equal(hv.view(torch.int16).numpy().view(np.uint16), ev)
    # clobber those device blocks, then swap back into the same blocks
    for b in seq1:
        kc[b].fill_(float("nan"))
        vc[b].fill_(float("nan"))
    in_pairs = out_pairs[:, ::-1].copy()
    pa.pa_swap_blocks(dev_i32(in_pairs), len(in_pairs), hk, hv, HB, kc, vc, NB, shape)
    assert pa.pa_last_device_error()[0] == pa.PA_OK
    assert np.array_equal(host_bits(kc).reshape(c["k_cache"].shape), c["k_cache"])
    assert np.array_equal(host_bits(vc).reshape(c["v_cache"].shape), c["v_cache"])
    out, _, _ = gpu_decode(gen.F16, c["q"], host_bits(kc).reshape(c["k_cache"].shape),
                           host_bits(vc).reshape(c["v_cache"].shape), c["block_tables"],
                           c["context_lens"], c["scale"])
    ref = orc.decode(gen.F16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.F16, "after swap-in")


def test_swap_refuses_pageable_host_memory():
    shape = pa.make_shape(num_seqs=1, num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                          num_blocks=8, max_blocks_per_seq=1, dtype=gen.F16)
    k = torch.zeros((8, 16, 2, 64), dtype=torch.float16, device="cuda")
    v = torch.zeros_like(k)
    hk = torch.zeros((8, 16, 2, 64), dtype=torch.float16)   # pageable
    hv = torch.zeros_like(hk)
    n0 = pa.pa_kernel_launches()
    with pytest.raises(pa.PaError) as e:
        pa.pa_swap_blocks(dev_i32(np.array([[0, 1]], np.int32)), 1, k, v, 8, hk, hv, 8, shape)
    assert e.value.status == pa.PA_ERR_INVALID_ARG and pa.pa_kernel_launches() == n0


def test_swap_rejects_overlap_and_reports_bad_pairs():
    shape = pa.make_shape(num_seqs=1, num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
                          num_blocks=8, max_blocks_per_seq=1, dtype=gen.F16)
    k = torch.zeros((8, 16, 2, 64), dtype=torch.float16, device="cuda")
    v = torch.zeros_like(k)
    pairs = dev_i32(np.array([[0, 1]], np.int32))
    with pytest.raises(pa.PaError) as e:
        pa.pa_swap_blocks(pairs, 1, k, v, 8, k, v, 8, shape)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    k2, v2 = torch.zeros_like(k), torch.zeros_like(v)
    pa.pa_swap_blocks(dev_i32(np.array([[0, 9]], np.int32)), 1, k, v, 8, k2, v2, 8, shape)
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_ERR_DEVICE_CHECK and bits & 0x8


@pytest.mark.parametrize("variant", [1, 2], ids=["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("dtype", [gen.F16, gen.BF16], ids=["f16", "bf16"])
def test_block_size_8(orc, variant, dtype):
    """8-token blocks (two TMA boxes per 16-token group), stale entries past the context."""
    rng = np.random.default_rng(1700 + variant + 10 * dtype)
    ctx = [1, 7, 8, 9, 15, 16, 17, 23, 24, 25, 300, 1029]
    c = gen.random_decode_case(rng, num_seqs=len(ctx), num_q_heads=16, num_kv_heads=2,
                               head_dim=128, block_size=8, dtype=dtype, context_lens=ctx)
    bt = c["block_tables"].copy()
    for s, L in enumerate(ctx):
        bt[s, (L + 7) // 8:] = -5   # entries past the context are never read
    out, _, _ = gpu_decode(dtype, c["q"], c["k_cache"], c["v_cache"], bt, c["context_lens"],
                           c["scale"], variant=variant)
    ref = orc.decode(dtype, c["q"], c["k_cache"], c["v_cache"], bt, c["context_lens"], c["scale"])
    assert_decode_close(out, ref, dtype, f"bs8 variant {variant}")


def test_block_size_8_shared_prefix(orc):
    from gpu_util import SHARED

    rng = np.random.default_rng(1800)
    groups = [(300, [310, 305, 301, 300]), (700, [720, 705]), (0, [33])]
    c = gen.grouped_decode_case(rng, groups=groups, num_q_heads=16, num_kv_heads=2, head_dim=128,
                                block_size=8, dtype=gen.BF16)
    out, _, _ = gpu_decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"], variant=SHARED)
    ref = orc.decode(gen.BF16, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert_decode_close(out, ref, gen.BF16, "bs8 shared prefix")
