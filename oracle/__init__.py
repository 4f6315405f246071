"""CPU oracle for paged decode attention (fp64, plain C loops).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this package and this package never imports the product library.

``pa_oracle.c`` is compiled with gcc into ``_build/liboracle.so`` on first use
(or by ``build()``).  The wrappers below only marshal NumPy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "pa_oracle.c")
LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")

_lock = threading.Lock()
_lib = None


def compile_oracle(source: str = SOURCE, out: str = LIB_PATH, extra_flags=()) -> str:
    """Compile an oracle source file into a shared library (gcc, -O2, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", *extra_flags, source, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


def build() -> str:
    return compile_oracle()


def _needs_build() -> bool:
    return (not os.path.exists(LIB_PATH)
            or os.path.getmtime(LIB_PATH) < os.path.getmtime(SOURCE))


def _declare(lib):
    c = ctypes
    P = c.c_void_p
    lib.oracle_f16_to_f64.restype = c.c_double
    lib.oracle_f16_to_f64.argtypes = [c.c_uint16]
    lib.oracle_bf16_to_f64.restype = c.c_double
    lib.oracle_bf16_to_f64.argtypes = [c.c_uint16]
    lib.oracle_num_threads.restype = c.c_int
    lib.oracle_num_threads.argtypes = [c.c_int]
    dec = [c.c_int] * 8 + [P, P, P, P, P, c.c_double]
    lib.oracle_decode.restype = c.c_int
    lib.oracle_decode.argtypes = dec + [P, c.c_int]
    lib.oracle_decode_partitioned.restype = c.c_int
    lib.oracle_decode_partitioned.argtypes = dec + [c.c_int, P, c.c_int]
    lib.oracle_cache_append.restype = c.c_int
    lib.oracle_cache_append.argtypes = [c.c_longlong, c.c_longlong, c.c_int, P, P, P, P, P]
    lib.oracle_copy_blocks.restype = c.c_int
    lib.oracle_copy_blocks.argtypes = [c.c_int, c.c_longlong, c.c_int, P, P, P]
    lib.oracle_swap_blocks.restype = c.c_int
    lib.oracle_swap_blocks.argtypes = [c.c_int, c.c_int, c.c_longlong, c.c_int, P, P, P, P, P]
    lib.oracle_decode_multi.restype = c.c_int
    lib.oracle_decode_multi.argtypes = [c.c_int] * 9 + [P, P, P, P, P, c.c_double, P, c.c_int]
    lib.oracle_e4m3_to_f64.restype = c.c_double
    lib.oracle_e4m3_to_f64.argtypes = [c.c_uint8]
    lib.oracle_e4m3_from_f32.restype = c.c_uint8
    lib.oracle_e4m3_from_f32.argtypes = [c.c_float]
    lib.oracle_decode_fp8.restype = c.c_int
    lib.oracle_decode_fp8.argtypes = [c.c_int] * 8 + [P, P, P, P, P, P, P, c.c_double, P, c.c_int]
    lib.oracle_cache_append_fp8.restype = c.c_int
    lib.oracle_cache_append_fp8.argtypes = [c.c_int, c.c_longlong, c.c_int, c.c_int, c.c_int,
                                            P, P, P, P, P, P, P]
    return lib


def load(path: str | None = None):
    """Load the oracle library (compiling it first if needed).

    ``path`` loads another build of an oracle source (used by the tests that
    check the pins catch planted mistakes).
    """
    global _lib
    if path is not None:
        return Oracle(_declare(ctypes.CDLL(path)))
    with _lock:
        if _lib is None:
            if _needs_build():
                compile_oracle()
            _lib = Oracle(_declare(ctypes.CDLL(LIB_PATH)))
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    pass


class Oracle:
    """NumPy-facing wrappers around the C oracle."""

    def __init__(self, lib):
        self.lib = lib

    def f16_to_f64(self, bits: int) -> float:
        return self.lib.oracle_f16_to_f64(int(bits))

    def bf16_to_f64(self, bits: int) -> float:
        return self.lib.oracle_bf16_to_f64(int(bits))

    def num_threads(self, requested: int = 0) -> int:
        return self.lib.oracle_num_threads(int(requested))

    @staticmethod
    def _decode_args(dtype, q, k_cache, v_cache, block_tables, context_lens):
        q = np.ascontiguousarray(q, dtype=np.uint16)
        kc = np.ascontiguousarray(k_cache, dtype=np.uint16)
        vc = np.ascontiguousarray(v_cache, dtype=np.uint16)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, Hq, D = q.shape
        NB, bs, Hkv, D2 = kc.shape
        assert D2 == D and vc.shape == kc.shape
        assert bt.ndim == 2 and bt.shape[0] == S and cl.shape == (S,)
        return (q, kc, vc, bt, cl), (int(dtype), S, Hq, Hkv, D, bs, NB, bt.shape[1])

    def decode(self, dtype, q, k_cache, v_cache, block_tables, context_lens, scale,
               num_threads: int = 0) -> np.ndarray:
        """fp64 [S][Hq][D] attention output (unrounded)."""
        arrs, dims = self._decode_args(dtype, q, k_cache, v_cache, block_tables, context_lens)
        S, Hq, D = dims[1], dims[2], dims[4]
        out = np.empty((S, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_decode(*dims, *(_ptr(a) for a in arrs), float(scale), _ptr(out),
                                    int(num_threads))
        if rc:
            raise OracleError(f"oracle_decode refused its input (rc={rc})")
        return out

    def decode_partitioned(self, dtype, q, k_cache, v_cache, block_tables, context_lens, scale,
                           partition_tokens: int, num_threads: int = 0) -> np.ndarray:
        arrs, dims = self._decode_args(dtype, q, k_cache, v_cache, block_tables, context_lens)
        S, Hq, D = dims[1], dims[2], dims[4]
        out = np.empty((S, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_decode_partitioned(*dims, *(_ptr(a) for a in arrs), float(scale),
                                                int(partition_tokens), _ptr(out), int(num_threads))
        if rc:
            raise OracleError(f"oracle_decode_partitioned refused its input (rc={rc})")
        return out

    def cache_append(self, k, v, slot_mapping, k_cache, v_cache) -> None:
        """In place on ``k_cache``/``v_cache`` ([NB][bs][Hkv][D], any 1- or 2-byte dtype)."""
        assert k_cache.flags["C_CONTIGUOUS"] and v_cache.flags["C_CONTIGUOUS"]
        k = np.ascontiguousarray(k)
        v = np.ascontiguousarray(v)
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int32)
        NB, bs = k_cache.shape[:2]
        row_bytes = k_cache.itemsize * int(np.prod(k_cache.shape[2:]))
        T = sm.shape[0]
        assert k.nbytes == T * row_bytes and v.nbytes == T * row_bytes
        rc = self.lib.oracle_cache_append(NB * bs, row_bytes, T, _ptr(k), _ptr(v), _ptr(sm),
                                          _ptr(k_cache), _ptr(v_cache))
        if rc:
            raise OracleError(f"oracle_cache_append refused its input (rc={rc})")

    def copy_blocks(self, pairs, k_cache, v_cache) -> None:
        assert k_cache.flags["C_CONTIGUOUS"] and v_cache.flags["C_CONTIGUOUS"]
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        NB = k_cache.shape[0]
        block_bytes = k_cache.nbytes // NB if NB else 1
        rc = self.lib.oracle_copy_blocks(NB, block_bytes, pr.shape[0], _ptr(pr), _ptr(k_cache),
                                         _ptr(v_cache))
        if rc:
            raise OracleError(f"oracle_copy_blocks refused its input (rc={rc})")

    def swap_blocks(self, pairs, src_k, src_v, dst_k, dst_v) -> None:
        """In place on ``dst_k``/``dst_v``: dst block p[1] = src block p[0] per pair."""
        for a in (dst_k, dst_v):
            assert a.flags["C_CONTIGUOUS"]
        src_k = np.ascontiguousarray(src_k)
        src_v = np.ascontiguousarray(src_v)
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        bb = src_k.nbytes // src_k.shape[0] if src_k.shape[0] else 1
        assert dst_k.nbytes // max(1, dst_k.shape[0]) == bb
        rc = self.lib.oracle_swap_blocks(src_k.shape[0], dst_k.shape[0], bb, pr.shape[0], _ptr(pr),
                                         _ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v))
        if rc:
            raise OracleError(f"oracle_swap_blocks refused its input (rc={rc})")

    def decode_multi(self, dtype, q, k_cache, v_cache, block_tables, context_lens, scale,
                     num_threads: int = 0) -> np.ndarray:
        """fp64 [S][Tq][Hq][D]: Tq query tokens per sequence (q [S][Tq][Hq][D]),
        query t attending to tokens 0 .. ctx - Tq + t."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        S, Tq, Hq, D = q.shape
        arrs, dims = self._decode_args(dtype, q.reshape(S, Tq * Hq, D), k_cache, v_cache,
                                       block_tables, context_lens)
        _, _, _, Hkv, _, bs, NB, MBS = dims
        out = np.empty((S, Tq, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_decode_multi(int(dtype), S, Tq, Hq, Hkv, D, bs, NB, MBS,
                                          *(_ptr(a) for a in arrs), float(scale), _ptr(out),
                                          int(num_threads))
        if rc:
            raise OracleError(f"oracle_decode_multi refused its input (rc={rc})")
        return out

    # ---- FP8 (E4M3) cache

    def e4m3_to_f64(self, code: int) -> float:
        return self.lib.oracle_e4m3_to_f64(int(code))

    def e4m3_from_f32(self, y: float) -> int:
        return int(self.lib.oracle_e4m3_from_f32(float(np.float32(y))))

    def decode_fp8(self, dtype, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                   scale, num_threads: int = 0) -> np.ndarray:
        """fp64 [S][Hq][D] attention output over an E4M3 cache (uint8 codes,
        [NB][bs][Hkv][D]) with fp32 per-kv-head scales."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        kc = np.ascontiguousarray(k_cache, dtype=np.uint8)
        vc = np.ascontiguousarray(v_cache, dtype=np.uint8)
        ks = np.ascontiguousarray(k_scale, dtype=np.float32)
        vs = np.ascontiguousarray(v_scale, dtype=np.float32)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        S, Hq, D = q.shape
        NB, bs, Hkv, D2 = kc.shape
        assert D2 == D and vc.shape == kc.shape and ks.shape == (Hkv,) and vs.shape == (Hkv,)
        out = np.empty((S, Hq, D), dtype=np.float64)
        rc = self.lib.oracle_decode_fp8(int(dtype), S, Hq, Hkv, D, bs, NB, bt.shape[1], _ptr(q),
                                        _ptr(kc), _ptr(vc), _ptr(ks), _ptr(vs), _ptr(bt), _ptr(cl),
                                        float(scale), _ptr(out), int(num_threads))
        if rc:
            raise OracleError(f"oracle_decode_fp8 refused its input (rc={rc})")
        return out

    def cache_append_fp8(self, dtype, k, v, slot_mapping, k_scale, v_scale, k_cache,
                         v_cache) -> None:
        """In place on the uint8 code pools ``k_cache``/``v_cache`` ([NB][bs][Hkv][D]);
        ``k``/``v`` are [T][Hkv][D] fp16/bf16 bits."""
        assert k_cache.flags["C_CONTIGUOUS"] and v_cache.flags["C_CONTIGUOUS"]
        assert k_cache.dtype == np.uint8 and v_cache.dtype == np.uint8
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int32)
        ks = np.ascontiguousarray(k_scale, dtype=np.float32)
        vs = np.ascontiguousarray(v_scale, dtype=np.float32)
        NB, bs, Hkv, D = k_cache.shape
        T = sm.shape[0]
        assert k.shape == (T, Hkv, D) and v.shape == (T, Hkv, D)
        rc = self.lib.oracle_cache_append_fp8(int(dtype), NB * bs, Hkv, D, T, _ptr(k), _ptr(v),
                                              _ptr(sm), _ptr(ks), _ptr(vs), _ptr(k_cache),
                                              _ptr(v_cache))
        if rc:
            raise OracleError(f"oracle_cache_append_fp8 refused its input (rc={rc})")
