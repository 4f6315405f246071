"""pa_decode captured into a CUDA graph and replayed, against the CPU oracle.

The tensor-core kernels take their items from a counter in the workspace,
tagged with a per-call epoch that a graph fixes at capture; a captured call
must still cover every item on every replay.  The output is NaN-filled before
each replay, so a skipped item shows up.  With shared prefixes at group 1 the
call forks the own-token pass onto a second stream and joins it again; the
capture takes both branches.
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


CTX = [5, 300, 1100, 2050, 700, 129, 1, 513]


@pytest.mark.parametrize("variant,shared,group",
                         [(1, 0, 4), (2, 0, 4), (2, 0, 8), (2, 0, 16), (0, 1, 8), (0, 1, 1)],
                         ids=["cuda_cores", "tc_pairs_g4", "tc_pairs_g8", "tc_g16", "shared_prefix",
                              "shared_prefix_second_stream"])
def test_decode_graph_replays(orc, variant, shared, group):
    rng = np.random.default_rng(1700 + 10 * variant + shared + group)
    Hkv, dtype = 2, gen.BF16
    c = gen.random_decode_case(rng, num_seqs=len(CTX), num_q_heads=Hkv * group, num_kv_heads=Hkv,
                               head_dim=128, block_size=16, dtype=dtype, context_lens=CTX,
                               shared_prefix_blocks=40 if shared else 0)
    NB, bs, _, D = c["k_cache"].shape
    shape = pa.make_shape(num_seqs=len(CTX), num_q_heads=Hkv * group, num_kv_heads=Hkv, head_dim=D,
                          block_size=bs, num_blocks=NB, max_blocks_per_seq=c["block_tables"].shape[1],
                          dtype=dtype, variant=variant, shared_prefix=shared)
    maxlen = max(CTX)
    wsb = pa.pa_decode_workspace_bytes(shape, maxlen)
    ws = torch.randint(0, 256, (wsb,), dtype=torch.uint8, device="cuda")
    args = (dev(c["q"], dtype), dev(c["k_cache"], dtype), dev(c["v_cache"], dtype),
            dev_i32(c["block_tables"]), dev_i32(c["context_lens"]), c["scale"])
    out = torch.full(c["q"].shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    ref = orc.decode(dtype, c["q"], c["k_cache"], c["v_cache"], c["block_tables"], c["context_lens"],
                     c["scale"])
    # eager first: sets the kernels' attributes and looks up the error word
    pa.pa_decode(*args, out, shape, maxlen, ws, wsb)
    torch.cuda.synchronize()
    assert_decode_close(host_bits(out), ref, dtype, "eager")
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        pa.pa_decode(*args, out, shape, maxlen, ws, wsb, stream=s)
    for r in range(3):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        status, bits = pa.pa_last_device_error()
        assert status == pa.PA_OK, f"device check fired on replay {r}: {bits:#x}"
        assert_decode_close(host_bits(out), ref, dtype, f"replay {r}")
    del g
