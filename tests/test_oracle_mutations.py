"""Planted mistakes in the oracle must be caught by the pins (no GPU).

Each mutant is a copy of oracle/pa_oracle.c with one plausible mistake (a
wrong index, a dropped term, a sign, a transposed operand, an off-by-one, a
wrong exponent bias).  It is compiled on the CPU and the whole pin suite is
run against it in a child process; at least one pin has to fail.  The real
oracle source is never modified.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

MUTANTS = {
    "logical_block_uses_modulo": ("int logical = j / bs;", "int logical = j % bs;"),
    "offset_uses_division": ("(long long)phys * bs + (j % bs)", "(long long)phys * bs + (j / bs)"),
    "kv_head_dropped_from_row": ("return (slot * Hkv + kvh) * (long long)D;",
                                 "return (slot * Hkv) * (long long)D;"),
    "gqa_interleaved_heads": ("block_tables, s, h / g, 0, L, scale, x, &m, &l, acc);",
                              "block_tables, s, h % Hkv, 0, L, scale, x, &m, &l, acc);"),
    "scale_dropped": ("x[j] = scale * dot;", "x[j] = dot;"),
    "exp_sign_flipped": ("double p = exp(x[j] - m);", "double p = exp(m - x[j]);"),
    "max_not_subtracted": ("double p = exp(x[j] - m);", "double p = exp(x[j]);"),
    "v_replaced_by_k": ("acc[d] += p * widen(dtype, vc[r + d]);",
                        "acc[d] += p * widen(dtype, kc[r + d]);"),
    "normalisation_dropped": ("for (int d = 0; d < D; ++d) o[d] = acc[d] / l;",
                              "for (int d = 0; d < D; ++d) o[d] = acc[d];"),
    "one_token_too_many": ("int n = t1 - t0;", "int n = t1 - t0 + 1;"),
    "one_token_too_few": ("int n = t1 - t0;", "int n = t1 - t0 - 1;"),
    "running_min_not_max": ("if (x[j] > m) m = x[j];", "if (x[j] < m) m = x[j];"),
    "f16_exponent_bias": ("v = ldexp((double)(f | 0x400), e - 25);",
                          "v = ldexp((double)(f | 0x400), e - 24);"),
    "f16_subnormal_scale": ("v = ldexp((double)f, -24);", "v = ldexp((double)f, -25);"),
    "f16_implicit_bit_dropped": ("v = ldexp((double)(f | 0x400), e - 25);",
                                 "v = ldexp((double)f, e - 25);"),
    "bf16_shift": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    "q_and_k_same_row": ("dot += widen(dtype, qrow[d]) * widen(dtype, kc[r + d]);",
                         "dot += widen(dtype, qrow[d]) * widen(dtype, qrow[d]);"),
    "merge_weights_dropped": ("den += exp(pm[p] - M) * pl[p];", "den += pl[p];"),
    "merge_numerator_unweighted": ("num += exp(pm[p] - M) * pacc[(long long)p * D + d];",
                                   "num += pacc[(long long)p * D + d];"),
    "append_off_by_one_slot": ("memcpy(k_cache + slot * row_bytes,",
                               "memcpy(k_cache + (slot ^ 1) * row_bytes,"),
    "copy_direction_swapped": (
        "memmove(k_cache + (long long)dst * block_bytes, k_cache + (long long)src * block_bytes,",
        "memmove(k_cache + (long long)src * block_bytes, k_cache + (long long)dst * block_bytes,"),
    "e4m3_exponent_bias": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 11);"),
    "e4m3_subnormal_step": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "e4m3_no_saturation": ("if (a >= 448.0) return sign | 0x7e;", "if (a >= 480.0) return sign | 0x7e;"),
    "e4m3_ties_away": ("double n = rint(ldexp(a, 3 - e));", "double n = floor(ldexp(a, 3 - e) + 0.5);"),
    "fp8_v_scale_dropped": ("acc[d] += w * (oracle_e4m3_to_f64(vc[r + d]) * vs);",
                            "acc[d] += w * oracle_e4m3_to_f64(vc[r + d]);"),
    "fp8_max_not_subtracted": ("double w = exp(x[j] - m);", "double w = exp(x[j]);"),
    "fp8_normalisation_dropped": ("o[d] = acc[d] / lsum;", "o[d] = acc[d];"),
    "fp8_k_scale_from_v": ("(double)k_scale[kvh], (double)v_scale[kvh], block_tables, s,",
                           "(double)v_scale[kvh], (double)v_scale[kvh], block_tables, s,"),
    "fp8_append_multiplies": ("oracle_e4m3_from_f32(xk / k_scale[h]);",
                              "oracle_e4m3_from_f32(xk * k_scale[h]);"),
    "fp8_append_head_index": ("int h = (int)(i / D);", "int h = (int)(i % Hkv);"),
    "multi_sees_next_token": ("int last = context_lens[s] - Tq + t;", "int last = context_lens[s] - Tq + t + 1;"),
    "multi_gqa_interleaved": ("int kv_head = h / g;", "int kv_head = h % Hkv;"),
    "multi_query_index_dropped": ("int t = (int)(st % Tq), s = (int)(st / Tq);",
                                  "int t = 0, s = (int)(st / Tq);"),
    "swap_direction": ("memcpy(dst_k + (long long)to * block_bytes, src_k + (long long)from * block_bytes,",
                       "memcpy(dst_k + (long long)from * block_bytes, src_k + (long long)to * block_bytes,"),
    "v_copy_skipped": (
        "memmove(v_cache + (long long)dst * block_bytes, v_cache + (long long)src * block_bytes,\n"
        "                (size_t)block_bytes);",
        "(void)0;"),
}

_RUNNER = r"""
import sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle, oracle_pins
orc = oracle.load({lib!r})
failed = []
for pin in oracle_pins.PINS:
    try:
        pin(orc)
    except Exception as e:  # AssertionError or a refusal
        failed.append(pin.__name__)
print("FAILED:" + ",".join(failed))
"""


def _run_mutant(name, tmpdir):
    old, new = MUTANTS[name]
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) == 1, f"{name}: mutation site must match exactly once"
    path = os.path.join(tmpdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.compile_oracle(path, os.path.join(tmpdir, f"lib{name}.so"))
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    tests = os.path.dirname(os.path.abspath(__file__))
    code = _RUNNER.format(root=root, tests=tests, lib=lib)
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, OMP_NUM_THREADS="1"))
    if p.returncode != 0:
        return name, ["<child process died>"]
    line = [ln for ln in p.stdout.splitlines() if ln.startswith("FAILED:")][-1]
    return name, [x for x in line[len("FAILED:"):].split(",") if x]


def test_every_planted_mistake_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = dict(ex.map(lambda n: _run_mutant(n, tmp), sorted(MUTANTS)))
    missed = [n for n, failed in results.items() if not failed]
    assert not missed, f"planted mistakes no pin caught: {missed}"


def test_unmutated_source_passes_all_pins():
    """Control: the runner itself reports no failure for the real oracle."""
    with tempfile.TemporaryDirectory() as tmp:
        lib = oracle.compile_oracle(oracle.SOURCE, os.path.join(tmp, "libctl.so"))
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        tests = os.path.dirname(os.path.abspath(__file__))
        p = subprocess.run([sys.executable, "-c", _RUNNER.format(root=root, tests=tests, lib=lib)],
                           capture_output=True, text=True, timeout=600)
        assert p.returncode == 0, p.stderr
        assert "FAILED:\n" in p.stdout + "\n" and "FAILED:pin" not in p.stdout
