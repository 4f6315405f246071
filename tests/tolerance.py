"""Acceptance bound for decode outputs against the fp64 oracle.

The bound is max |err| <= 2e-3 and mean |err| <= 2e-4 per output tensor,
with the kernel's fp16/bf16 output compared against the oracle's unrounded
fp64 result.  Rounding the exact value to the output type alone costs up to
half a unit in the last place, and fp32 arithmetic near a rounding boundary
can move the result by one more half unit.  Where one ulp of the output type
exceeds 2e-3 (bf16 at |o| >= 0.5, fp16 at |o| >= 4) the per-element bound is
one ulp of that type at the exact value instead.  The number of elements that used that branch is reported.

The mean bound is mean |err| <= max(2e-4, mean |round(ref) - ref| + 5e-5),
where round(ref) is the exact result rounded to the output type.  Rounding
alone averages a quarter ulp, 4.9e-4 for bf16 outputs in [0.25, 0.5), so a
plain 2e-4 could not be met by any implementation on short contexts; above
that floor a kernel may add at most 5e-5.  (Measured over every parity case
of the GPU suite, the kernels' mean error exceeds the rounding floor by at
most 1.1e-9: they round as well as a correctly rounded result.)
"""
import json
import os

import numpy as np

from paged_kv_cache_458_b200 import gen

# With PA_TOLERANCE_LOG set to a file path, every check appends one JSON line:
# the case, its error statistics and how much of each bound they use.
_LOG = os.environ.get("PA_TOLERANCE_LOG")

MAX_ABS = 2e-3
MEAN_ABS = 2e-4
MEAN_OVER_FLOOR = 5e-5  # what a kernel may add to the output's own rounding, on average
_MANTISSA = {gen.F16: 10, gen.BF16: 7}
_MIN_EXP = {gen.F16: -14, gen.BF16: -126}


def ulp(ref: np.ndarray, dtype: int) -> np.ndarray:
    a = np.abs(ref)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, _MIN_EXP[dtype])
    return np.exp2(e - _MANTISSA[dtype])


def rounding_floor(ref: np.ndarray, dtype: int) -> float:
    """Mean |round(ref) - ref| with round() to the output type."""
    if ref.size == 0:
        return 0.0
    r = gen.bits_to_f32(gen.to_bits(ref.astype(np.float32), dtype), dtype).astype(np.float64)
    return float(np.mean(np.abs(r - ref)))


def decode_errors(out_bits: np.ndarray, ref: np.ndarray, dtype: int) -> dict:
    got = gen.bits_to_f32(out_bits, dtype).astype(np.float64).reshape(ref.shape)
    err = np.abs(got - ref)
    allowed = np.maximum(MAX_ABS, ulp(ref, dtype))
    return dict(max_abs=float(np.nanmax(err)) if err.size else 0.0,
                mean_abs=float(np.mean(err)) if err.size else 0.0,
                mean_floor=rounding_floor(ref, dtype),
                n_nan=int(np.isnan(got).sum()),
                n_over=int((err > allowed).sum()),
                n_ulp_branch=int((ulp(ref, dtype) > MAX_ABS).sum()),
                n=int(err.size))


def _log(st, dtype, what):
    if not _LOG:
        return
    rec = dict(st, what=what, dtype=gen.DTYPE_NAMES[dtype],
               test=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
               max_used=st["max_abs"] / MAX_ABS,
               mean_over_floor=st["mean_abs"] - st["mean_floor"])
    with open(_LOG, "a") as f:
        f.write(json.dumps(rec) + "\n")


def assert_decode_close(out_bits, ref, dtype, what=""):
    st = decode_errors(out_bits, ref, dtype)
    _log(st, dtype, what)
    assert st["n_nan"] == 0, f"{what}: {st['n_nan']} NaN outputs"
    assert st["n_over"] == 0, f"{what}: {st['n_over']} elements above the bound (max {st['max_abs']:.3e})"
    assert st["mean_abs"] <= max(MEAN_ABS, st["mean_floor"] + MEAN_OVER_FLOOR), \
        f"{what}: mean abs error {st['mean_abs']:.3e} (rounding alone {st['mean_floor']:.3e})"
    return st
