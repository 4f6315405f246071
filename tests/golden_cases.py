"""Builds the hand-derived block-mapping examples of tests/golden/.

The fixture file cites the pages' mapping example (logical block 0 ->
physical block 7) and states each input and the closed-form output; this
module turns those statements into arrays and evaluates the closed form.
"""
import json
import math
import os

import numpy as np

from paged_kv_cache_458_b200 import gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "block_mapping_examples.json")


def load_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


def build(case):
    """Arrays for one example plus the expected fp64 output [1][1][D]."""
    D, bs, NB = case["head_dim"], case["block_size"], case["num_blocks"]
    dtype = gen.F16
    nan = gen.NAN_BITS[dtype]
    kc = np.full((NB, bs, 1, D), nan, dtype=np.uint16)
    vc = np.full((NB, bs, 1, D), nan, dtype=np.uint16)
    d = np.arange(D, dtype=np.float64)
    e0 = np.zeros(D)
    e0[0] = 1.0

    def put(block, off, K, V):
        kc[block, off, 0] = gen.f32_to_f16_bits(np.asarray(K, dtype=np.float32))
        vc[block, off, 0] = gen.f32_to_f16_bits(np.asarray(V, dtype=np.float32))

    if case["name"] == "logical0_to_physical7_two_tokens":
        V0 = (d % 8) - 4
        V1 = 0.5 * ((d % 5) - 2)
        put(7, 0, np.zeros(D), V0)
        put(7, 1, e0, V1)
        expected = (V0 + 3 * V1) / 4
    elif case["name"] == "crossing_into_second_block":
        for j in range(16):
            put(7, j, np.zeros(D), (j + d / 64) / 8)
        put(2, 0, e0, (16 + d / 64) / 8)
        expected = 47.0 / 32.0 + d / 512
    else:  # pragma: no cover
        raise KeyError(case["name"])
    table = np.array([case["block_table"]], dtype=np.int32)
    ctx = np.array([case["context_len"]], dtype=np.int32)
    q = gen.f32_to_f16_bits(e0.astype(np.float32)).reshape(1, 1, D)
    scale = {"ln(3)": math.log(3.0), "ln(16)": math.log(16.0)}[case["scale"]]
    return dict(dtype=dtype, q=q, k_cache=kc, v_cache=vc, block_tables=table,
                context_lens=ctx, scale=scale, expected=expected.reshape(1, 1, D))
