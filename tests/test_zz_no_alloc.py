"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library cannot allocate the split-K workspace that
pa_decode needs -- a plug-in inside a host runtime that owns all device memory
and offers no allocator, or a decode loop that must not call cudaMalloc while
it runs.  pa_decode_noalloc takes that scratch from a fixed array inside the
library instead.  This file checks, through the C ABI:

- two calls in a row, of different shapes, each against the fp64 oracle
  (the decode tolerance) and bit for bit against pa_decode with a
  caller-owned workspace (the same kernels write the same partials into
  fixed slots and merge them in a fixed order, so anything the first call
  left in the shared array that leaked into the second would show);
- the same with shared_prefix = 1, whose group plan and work counter also
  live in the shared array, with two different groupings in a row;
- that a request larger than the array is refused with nothing launched.

It is named to be collected last and needs nothing from the other test files,
so it also runs alone in a fresh process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from paged_kv_cache_458_b200 import gen, pa  # noqa: E402
from gpu_util import SHARED, dev, dev_i32, host_bits, shape_of  # noqa: E402
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


def _on_device(c, dtype, variant=0):
    shape = shape_of(dtype, c["q"], c["k_cache"], c["block_tables"], variant=variant)
    d = dict(q=dev(c["q"], dtype), k=dev(c["k_cache"], dtype), v=dev(c["v_cache"], dtype),
             bt=dev_i32(c["block_tables"]), cl=dev_i32(c["context_lens"]))
    return shape, d, int(np.max(c["context_lens"], initial=0))


def _with_workspace(c, shape, d, maxlen, dtype):
    out = torch.full(c["q"].shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    wsb = pa.pa_decode_workspace_bytes(shape, maxlen)
    # arbitrary bytes: the workspace needs no initial contents
    ws = torch.randint(0, 256, (max(16, wsb),), dtype=torch.uint8, device="cuda")
    pa.pa_decode(d["q"], d["k"], d["v"], d["bt"], d["cl"], c["scale"], out, shape, maxlen, ws, wsb)
    return host_bits(out)


def _no_alloc(c, shape, d, maxlen, dtype):
    out = torch.full(c["q"].shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    pa.pa_decode_noalloc(d["q"], d["k"], d["v"], d["bt"], d["cl"], c["scale"], out, shape, maxlen)
    return host_bits(out)


def _check_pair(orc, cases, dtype, variant):
    """Both calls through pa_decode_noalloc in a row, then each against the
    oracle and against pa_decode with its own workspace."""
    dev_cases = [(c,) + _on_device(c, dtype, variant) for c in cases]
    for _, shape, _, maxlen in dev_cases:
        assert 0 < pa.pa_decode_workspace_bytes(shape, maxlen) <= pa.PA_NOALLOC_SCRATCH_BYTES
    got = [_no_alloc(c, s, d, m, dtype) for c, s, d, m in dev_cases]
    status, bits = pa.pa_last_device_error()
    assert status == pa.PA_OK, f"device check fired: {bits:#x}"
    ref = [_with_workspace(c, s, d, m, dtype) for c, s, d, m in dev_cases]
    for i, (c, g, r) in enumerate(zip(cases, got, ref)):
        exact = orc.decode(dtype, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"])
        assert_decode_close(g, exact, dtype, f"call {i + 1} vs the oracle")
        assert np.array_equal(g, r), f"call {i + 1}: differs from pa_decode with a workspace"


def test_two_calls_in_a_row(orc):
    dtype = gen.BF16
    rng = np.random.default_rng(31)
    # first call: long contexts, many partitions (fills much of the scratch);
    # second: other shapes and contexts, so stale scratch from call 1 would show
    c1 = gen.random_decode_case(rng, num_seqs=6, num_q_heads=8, num_kv_heads=2, head_dim=128,
                                block_size=16, dtype=dtype,
                                context_lens=[3000, 1, 2049, 700, 4096, 513])
    c2 = gen.random_decode_case(rng, num_seqs=4, num_q_heads=16, num_kv_heads=2, head_dim=128,
                                block_size=16, dtype=dtype, context_lens=[1500, 600, 33, 2500])
    _check_pair(orc, [c1, c2], dtype, variant=0)


def test_two_shared_prefix_calls_in_a_row(orc):
    """The plan and the tagged work counter sit in the shared array too."""
    dtype = gen.F16
    rng = np.random.default_rng(32)
    c1 = gen.grouped_decode_case(rng, groups=[(700, [710, 730, 760, 705]), (300, [310, 305]),
                                              (0, [37])],
                                 num_q_heads=16, num_kv_heads=2, head_dim=128, block_size=16,
                                 dtype=dtype)
    # different groupings in the same sequence positions: stale plan entries
    # from call 1 would put members in the wrong groups
    c2 = gen.grouped_decode_case(rng, groups=[(0, [50]), (1200, [1210, 1300, 1250]),
                                              (260, [270, 300, 290, 280])],
                                 num_q_heads=16, num_kv_heads=2, head_dim=128, block_size=16,
                                 dtype=dtype)
    _check_pair(orc, [c1, c2], dtype, variant=SHARED)


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
