"""ctypes binding of libpa.so (include/pa.h): argument marshalling only.

Every function here forwards to the C entry point of the same name; all
arithmetic runs in the library's CUDA kernels.  Tensors are PyTorch tensors
(device memory and streams are PyTorch's); a plain integer is accepted
wherever a device pointer is expected.  If libpa.so has not been built the
first call raises ``LibraryMissing`` -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpa.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "pa.h")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_OOM, PA_ERR_DEVICE_CHECK = range(6)
PA_F16, PA_BF16 = 0, 1
PA_DECODE_AUTO, PA_DECODE_CUDA_CORES, PA_DECODE_TENSOR_CORES = 0, 1, 2
PA_DECODE_RESOLVED_SHARED_PREFIX = 3
PA_CACHE_AS_DTYPE, PA_CACHE_FP8_E4M3 = 0, 1
PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_CONTEXT_LEN = 0x2
PA_DEVERR_SLOT = 0x4
PA_DEVERR_PAIR = 0x8
PA_DEVERR_WAIT_TIMEOUT = 0x10


class LibraryMissing(ImportError):
    pass


class PaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} failed: {status_string(status)} (status {status})"
        if status == PA_ERR_CUDA:
            msg += f": {pa_last_cuda_error()}"
        super().__init__(msg)


class pa_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_seqs", "num_q_heads", "num_kv_heads", "head_dim", "block_size", "num_blocks",
        "max_blocks_per_seq", "partition_tokens", "dtype", "variant", "shared_prefix",
        "cache_format")]

    def __repr__(self):
        return "pa_shape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_lock = threading.Lock()
_lib = None


def _declare(lib):
    c = ctypes
    P, I32, SZ, U64 = c.c_void_p, c.c_int32, c.c_size_t, c.c_uint64
    SP = c.POINTER(pa_shape)
    lib.pa_decode_workspace_bytes.restype = SZ
    lib.pa_decode_workspace_bytes.argtypes = [SP, I32]
    lib.pa_decode.restype = c.c_int
    lib.pa_decode.argtypes = [P, P, P, P, P, c.c_float, P, SP, I32, P, SZ, P]
    lib.pa_decode_noalloc.restype = c.c_int
    lib.pa_decode_noalloc.argtypes = [P, P, P, P, P, c.c_float, P, SP, I32, P]
    lib.pa_cache_append.restype = c.c_int
    lib.pa_cache_append.argtypes = [P, P, P, I32, P, P, SP, P]
    lib.pa_cache_append_fp8.restype = c.c_int
    lib.pa_cache_append_fp8.argtypes = [P, P, P, I32, P, P, P, P, SP, P]
    lib.pa_decode_fp8.restype = c.c_int
    lib.pa_decode_fp8.argtypes = [P, P, P, P, P, P, P, c.c_float, P, SP, I32, P, SZ, P]
    lib.pa_copy_blocks.restype = c.c_int
    lib.pa_copy_blocks.argtypes = [P, I32, P, P, SP, P]
    lib.pa_swap_blocks.restype = c.c_int
    lib.pa_swap_blocks.argtypes = [P, I32, P, P, I32, P, P, I32, SP, P]
    lib.pa_last_device_error.restype = c.c_int
    lib.pa_last_device_error.argtypes = [P, c.POINTER(c.c_uint32)]
    lib.pa_status_string.restype = c.c_char_p
    lib.pa_status_string.argtypes = [c.c_int]
    lib.pa_kernel_launches.restype = U64
    lib.pa_kernel_launches.argtypes = []
    lib.pa_build_info.restype = c.c_char_p
    lib.pa_build_info.argtypes = []
    lib.pa_decode_multi_workspace_bytes.restype = SZ
    lib.pa_decode_multi_workspace_bytes.argtypes = [SP, I32, I32]
    lib.pa_decode_multi.restype = c.c_int
    lib.pa_decode_multi.argtypes = [P, P, P, P, P, c.c_float, P, SP, I32, I32, P, SZ, P]
    lib.pa_decode_partition_tokens.restype = c.c_int
    lib.pa_decode_partition_tokens.argtypes = [SP]
    lib.pa_decode_resolved_variant.restype = c.c_int
    lib.pa_decode_resolved_variant.argtypes = [SP]
    lib.pa_last_cuda_error.restype = c.c_char_p
    lib.pa_last_cuda_error.argtypes = []
    lib.pa_alloc_create.restype = P
    lib.pa_alloc_create.argtypes = [I32, I32, P]
    lib.pa_alloc_destroy.restype = None
    lib.pa_alloc_destroy.argtypes = [P]
    for name in ("pa_alloc_add_seq", "pa_alloc_extend"):
        getattr(lib, name).restype = c.c_int
        getattr(lib, name).argtypes = [P, I32, I32]
    lib.pa_alloc_fork.restype = c.c_int
    lib.pa_alloc_fork.argtypes = [P, I32, I32]
    lib.pa_alloc_free_seq.restype = c.c_int
    lib.pa_alloc_free_seq.argtypes = [P, I32]
    lib.pa_alloc_append_slots.restype = c.c_int
    lib.pa_alloc_append_slots.argtypes = [P, P, I32, P, P, P]
    lib.pa_alloc_block_tables.restype = c.c_int
    lib.pa_alloc_block_tables.argtypes = [P, P, I32, I32, P, P]
    lib.pa_alloc_num_free.restype = I32
    lib.pa_alloc_num_free.argtypes = [P]
    lib.pa_alloc_refcount.restype = I32
    lib.pa_alloc_refcount.argtypes = [P, I32]
    return lib


def lib():
    """The loaded libpa.so (raises LibraryMissing if it was not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise LibraryMissing(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m paged_kv_cache_458_b200.build` (there is no fallback path)")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/pa.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def status_string(status: int) -> str:
    try:
        return lib().pa_status_string(int(status)).decode()
    except LibraryMissing:
        return f"status {status}"


def _check(fn: str, status: int) -> None:
    if status != PA_OK:
        raise PaError(fn, status)


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_shape(*, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
               max_blocks_per_seq, partition_tokens=0, dtype=PA_F16, variant=0,
               shared_prefix=0, cache_format=PA_CACHE_AS_DTYPE) -> pa_shape:
    return pa_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                    max_blocks_per_seq, partition_tokens, dtype, variant, shared_prefix,
                    cache_format)


def torch_dtype(dtype: int):
    import torch

    return torch.float16 if dtype == PA_F16 else torch.bfloat16


# ---------------------------------------------------------------------------
# the three calls of the hot path


def pa_decode_workspace_bytes(shape: pa_shape, max_context_len: int) -> int:
    return int(lib().pa_decode_workspace_bytes(ctypes.byref(shape), int(max_context_len)))


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
              shape: pa_shape, max_context_len: int, workspace=None, workspace_bytes: int | None = None,
              stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_decode", lib().pa_decode(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        float(scale), _ptr(out), ctypes.byref(shape), int(max_context_len), _ptr(workspace),
        int(workspace_bytes), _stream(stream)))


def pa_decode_multi_workspace_bytes(shape: pa_shape, num_query_tokens: int,
                                    max_context_len: int) -> int:
    return int(lib().pa_decode_multi_workspace_bytes(ctypes.byref(shape), int(num_query_tokens),
                                                     int(max_context_len)))


def pa_decode_multi(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
                    shape: pa_shape, num_query_tokens: int, max_context_len: int, workspace=None,
                    workspace_bytes: int | None = None, stream=None) -> None:
    """Tq query tokens per sequence, causal over the new tokens (see pa.h)."""
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_decode_multi", lib().pa_decode_multi(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        float(scale), _ptr(out), ctypes.byref(shape), int(num_query_tokens), int(max_context_len),
        _ptr(workspace), int(workspace_bytes), _stream(stream)))


def pa_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale: float, out,
                      shape: pa_shape, max_context_len: int, stream=None) -> None:
    """pa_decode with its split-K scratch taken from a fixed array inside the
    library, for callers that cannot allocate device memory (see pa.h)."""
    _check("pa_decode_noalloc", lib().pa_decode_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(context_lens),
        float(scale), _ptr(out), ctypes.byref(shape), int(max_context_len), _stream(stream)))


PA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def pa_cache_append(k, v, slot_mapping, num_tokens: int, k_cache, v_cache, shape: pa_shape,
                    stream=None) -> None:
    _check("pa_cache_append", lib().pa_cache_append(
        _ptr(k), _ptr(v), _ptr(slot_mapping), int(num_tokens), _ptr(k_cache), _ptr(v_cache),
        ctypes.byref(shape), _stream(stream)))


def pa_cache_append_fp8(k, v, slot_mapping, num_tokens: int, k_cache, v_cache, k_scale, v_scale,
                        shape: pa_shape, stream=None) -> None:
    _check("pa_cache_append_fp8", lib().pa_cache_append_fp8(
        _ptr(k), _ptr(v), _ptr(slot_mapping), int(num_tokens), _ptr(k_cache), _ptr(v_cache),
        _ptr(k_scale), _ptr(v_scale), ctypes.byref(shape), _stream(stream)))


def pa_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, scale: float,
                  out, shape: pa_shape, max_context_len: int, workspace=None,
                  workspace_bytes: int | None = None, stream=None) -> None:
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("pa_decode_fp8", lib().pa_decode_fp8(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
        _ptr(context_lens), float(scale), _ptr(out), ctypes.byref(shape), int(max_context_len),
        _ptr(workspace), int(workspace_bytes), _stream(stream)))


def pa_copy_blocks(src_dst_pairs, num_pairs: int, k_cache, v_cache, shape: pa_shape,
                   stream=None) -> None:
    _check("pa_copy_blocks", lib().pa_copy_blocks(
        _ptr(src_dst_pairs), int(num_pairs), _ptr(k_cache), _ptr(v_cache), ctypes.byref(shape),
        _stream(stream)))


def pa_swap_blocks(src_dst_pairs, num_pairs: int, src_k, src_v, src_num_blocks: int, dst_k, dst_v,
                   dst_num_blocks: int, shape: pa_shape, stream=None) -> None:
    """Copy whole blocks between two pools (device and/or pinned host memory)."""
    _check("pa_swap_blocks", lib().pa_swap_blocks(
        _ptr(src_dst_pairs), int(num_pairs), _ptr(src_k), _ptr(src_v), int(src_num_blocks),
        _ptr(dst_k), _ptr(dst_v), int(dst_num_blocks), ctypes.byref(shape), _stream(stream)))


def pa_last_device_error(stream=None) -> tuple[int, int]:
    """(status, error bits); synchronises the stream."""
    bits = ctypes.c_uint32(0)
    st = lib().pa_last_device_error(_stream(stream), ctypes.byref(bits))
    return int(st), int(bits.value)


def pa_kernel_launches() -> int:
    return int(lib().pa_kernel_launches())


def pa_decode_partition_tokens(shape: pa_shape) -> int:
    v = lib().pa_decode_partition_tokens(ctypes.byref(shape))
    if v < 0:
        raise PaError("pa_decode_partition_tokens", -v)
    return v


def pa_decode_resolved_variant(shape: pa_shape) -> int:
    v = lib().pa_decode_resolved_variant(ctypes.byref(shape))
    if v < 0:
        raise PaError("pa_decode_resolved_variant", -v)
    return v


def pa_last_cuda_error() -> str:
    return lib().pa_last_cuda_error().decode()


def pa_build_info() -> str:
    return lib().pa_build_info().decode()


# ---------------------------------------------------------------------------
# host block allocator


class Allocator:
    """The C host allocator (pa_alloc_*): free list, refcounts, block tables."""

    def __init__(self, num_blocks: int, block_size: int, order=None):
        import numpy as np

        self._np = np
        self.block_size = int(block_size)
        self._order = None if order is None else np.ascontiguousarray(order, dtype=np.int32)
        h = lib().pa_alloc_create(int(num_blocks), int(block_size),
                                  None if self._order is None else self._order.ctypes.data)
        if not h:
            raise PaError("pa_alloc_create", PA_ERR_INVALID_ARG)
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            lib().pa_alloc_destroy(self._h)
            self._h = None

    __del__ = close

    def add_seq(self, seq: int, n_tokens: int):
        _check("pa_alloc_add_seq", lib().pa_alloc_add_seq(self._h, int(seq), int(n_tokens)))

    def extend(self, seq: int, n_tokens: int):
        _check("pa_alloc_extend", lib().pa_alloc_extend(self._h, int(seq), int(n_tokens)))

    def fork(self, parent: int, child: int):
        _check("pa_alloc_fork", lib().pa_alloc_fork(self._h, int(parent), int(child)))

    def free_seq(self, seq: int):
        _check("pa_alloc_free_seq", lib().pa_alloc_free_seq(self._h, int(seq)))

    def append_slots(self, seqs):
        np = self._np
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        n = seqs.shape[0]
        slots = np.empty(n, dtype=np.int32)
        pairs = np.empty((max(n, 1), 2), dtype=np.int32)
        npairs = ctypes.c_int32(0)
        _check("pa_alloc_append_slots", lib().pa_alloc_append_slots(
            self._h, seqs.ctypes.data, n, slots.ctypes.data, pairs.ctypes.data,
            ctypes.addressof(npairs)))
        return slots, pairs[:npairs.value].copy()

    def block_tables(self, seqs, max_blocks_per_seq: int):
        np = self._np
        seqs = np.ascontiguousarray(seqs, dtype=np.int32)
        n = seqs.shape[0]
        tables = np.empty((n, max_blocks_per_seq), dtype=np.int32)
        lens = np.empty(n, dtype=np.int32)
        _check("pa_alloc_block_tables", lib().pa_alloc_block_tables(
            self._h, seqs.ctypes.data, n, int(max_blocks_per_seq), tables.ctypes.data,
            lens.ctypes.data))
        return tables, lens

    def num_free(self) -> int:
        return int(lib().pa_alloc_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(lib().pa_alloc_refcount(self._h, int(block)))
