"""Device-side helpers for the GPU parity tests (all compute goes through libpa)."""
import numpy as np
import torch

from paged_kv_cache_458_b200 import gen, pa


def dev(bits: np.ndarray, dtype: int) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(pa.torch_dtype(dtype)).cuda()


def dev_i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


# Decode modes of the tests: the three values of pa_shape.variant, and
# SHARED = automatic variant with shared_prefix on.
SHARED = 3
MODES = {0: "auto", 1: "cuda_cores", 2: "tensor_cores", SHARED: "shared_prefix"}


def shape_of(dtype, q, k_cache, block_tables, partition_tokens=0, variant=0):
    """pa_shape of host arrays; variant SHARED means automatic + shared_prefix."""
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    shared = int(variant == SHARED)
    return pa.make_shape(num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                         num_blocks=NB, max_blocks_per_seq=block_tables.shape[1],
                         partition_tokens=partition_tokens, dtype=dtype,
                         variant=0 if shared else variant, shared_prefix=shared)


def gpu_decode(dtype, q, k_cache, v_cache, block_tables, context_lens, scale, partition_tokens=0,
               max_context_len=None, expect_ok=True, variant=0):
    """Run pa_decode on host arrays; returns (out bits, device error status, bits)."""
    shape = shape_of(dtype, q, k_cache, block_tables, partition_tokens, variant)
    if max_context_len is None:
        max_context_len = int(np.max(context_lens, initial=0))
    kc, vc = dev(k_cache, dtype), dev(v_cache, dtype)
    qd = dev(q, dtype)
    bt, cl = dev_i32(block_tables), dev_i32(context_lens)
    out = torch.full(q.shape, float("nan"), dtype=pa.torch_dtype(dtype), device="cuda")
    wsb = pa.pa_decode_workspace_bytes(shape, max_context_len)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    pa.pa_decode(qd, kc, vc, bt, cl, scale, out, shape, max_context_len, ws, wsb)
    status, bits = pa.pa_last_device_error()
    if expect_ok:
        assert status == pa.PA_OK, f"device check fired: bits {bits:#x}"
    return host_bits(out), status, bits
