"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library cannot allocate the split-K workspace that
pa_decode needs -- a plug-in inside a host runtime that owns all device memory
and offers no allocator, or a decode loop that must not call cudaMalloc while
it runs.  pa_decode_noalloc takes that scratch from a fixed array inside the
library instead.  This file checks, through the C ABI, that two calls in a
row give the same output as pa_decode with a caller-owned workspace (within
the tests' decode tolerance), that the second call is not disturbed by what
the first left in the shared array, and that a request larger than the
array is refused.  It is named to be collected last and needs nothing from
the other test files, so it also runs alone in a fresh process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from paged_kv_cache_458_b200 import gen, pa  # noqa: E402
from gpu_util import dev, dev_i32, host_bits, shape_of  # noqa: E402
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


def _inputs(seed, ctx, group=4, dtype=gen.BF16):
    c = gen.random_decode_case(np.random.default_rng(seed), num_seqs=len(ctx),
                               num_q_heads=2 * group, num_kv_heads=2, head_dim=128,
                               block_size=16, dtype=dtype, context_lens=ctx)
    shape = shape_of(dtype, c["q"], c["k_cache"], c["block_tables"])
    d = dict(q=dev(c["q"], dtype), k=dev(c["k_cache"], dtype), v=dev(c["v_cache"], dtype),
             bt=dev_i32(c["block_tables"]), cl=dev_i32(c["context_lens"]))
    return c, shape, d, int(max(ctx))


def _with_workspace(c, shape, d, maxlen, dtype):
    out = torch.empty(c["q"].shape, dtype=pa.torch_dtype(dtype), device="cuda")
    wsb = pa.pa_decode_workspace_bytes(shape, maxlen)
    ws = torch.empty(max(16, wsb), dtype=torch.uint8, device="cuda")
    pa.pa_decode(d["q"], d["k"], d["v"], d["bt"], d["cl"], c["scale"], out, shape, maxlen, ws, wsb)
    return out


def _no_alloc(c, shape, d, maxlen, dtype):
    out = torch.full(c["q"].shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    pa.pa_decode_noalloc(d["q"], d["k"], d["v"], d["bt"], d["cl"], c["scale"], out, shape, maxlen)
    return out


def test_two_calls_in_a_row_match_pa_decode():
    dtype = gen.BF16
    # first call: long contexts, many partitions (fills much of the scratch)
    c1, s1, d1, m1 = _inputs(31, [3000, 1, 2049, 700, 4096, 513], group=4)
    assert pa.pa_decode_workspace_bytes(s1, m1) > 0
    # second call: other shapes and contexts, so stale scratch from call 1 would show
    c2, s2, d2, m2 = _inputs(32, [1500, 600, 33, 2500], group=8)
    ref1 = _with_workspace(c1, s1, d1, m1, dtype)
    ref2 = _with_workspace(c2, s2, d2, m2, dtype)
    got1 = _no_alloc(c1, s1, d1, m1, dtype)
    got2 = _no_alloc(c2, s2, d2, m2, dtype)
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_OK, f"device check fired: {bits:#x}"
    for got, ref, what in ((got1, ref1, "first call"), (got2, ref2, "second call")):
        r = host_bits(ref).astype(np.uint16)
        ref64 = gen.bits_to_f32(r, dtype).astype(np.float64).reshape(ref.shape)
        assert_decode_close(host_bits(got), ref64, dtype, what)


def test_request_larger_than_the_scratch_is_refused():
    # 64 sequences x 64 query heads x 16 partitions x 130 floats = 34 MB > 32 MiB
    shape = pa.make_shape(num_seqs=64, num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=16,
                          num_blocks=1024, max_blocks_per_seq=512, partition_tokens=512,
                          dtype=pa.PA_BF16)
    assert pa.pa_decode_workspace_bytes(shape, 8192) > pa.PA_NOALLOC_SCRATCH_BYTES
    n0 = pa.pa_kernel_launches()
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_noalloc(16, 16, 16, 16, 16, 0.1, 16, shape, 8192)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    assert pa.pa_kernel_launches() == n0
