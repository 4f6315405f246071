"""Checks that tie the CPU oracle to facts other than itself.

Each ``pin_*`` function takes a loaded oracle and raises AssertionError when
the oracle disagrees with what the pages or the mathematics fix:

* exact widening of fp16/bf16 (NumPy's and PyTorch's own conversions);
* brute force in 50-digit arithmetic on tiny inputs (mpmath);
* closed forms: a context of one token returns that token's V row, identical
  keys return the mean of V, one dominant logit returns its V row, logits
  near 1000 stay finite, a context of zero returns zeros;
* the block-mapping examples in tests/golden (logical block 0 -> physical
  block 7, 5688vip.com section 2.2) whose outputs follow by hand;
* non-contiguous storage (zingnex.cn section 3.2 item 2): relabelling the
  physical blocks leaves the output bit-identical, and the paged result equals
  dense attention over the static [batch, heads, max_len, head_dim] layout of
  the same page's section 3.1;
* block sharing (section 3.2 item 3): shared blocks give the same output as
  private copies;
* grouped queries equal full multi-head attention with repeated kv heads;
* the partitioned (split-K) form equals the direct one;
* append and copy-on-write equal a NumPy scatter/copy over the whole pool, and
  a swap between two pools equals a block copy; a pool of 16-token blocks
  read as twice as many 8-token blocks gives the same output;
* the E4M3 cache: every code widens as PyTorch's float8_e4m3fn does, the
  encoder rounds as PyTorch's fp32 conversion below the saturation point,
  codes round-trip, ties go to the even code, large values saturate at 448;
  over codes that fp16 holds exactly the FP8 decode equals the fp16 decode;
  the scales act as factors of the logits and of the output, per kv head;
  append encodes each element of x / scale as PyTorch does.

The pins are plain functions so that tests/test_oracle_mutations.py can run
them against oracle builds with planted mistakes.
"""
from __future__ import annotations

import math

import numpy as np

from paged_kv_cache_458_b200 import gen
import golden_cases


def _case(seed, **kw):
    return gen.random_decode_case(np.random.default_rng(seed), **kw)


def _decode(orc, dtype, c, scale=None):
    return orc.decode(dtype, c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                      c["context_lens"], c["scale"] if scale is None else scale)


def _widen(bits, dtype):
    return gen.bits_to_f32(bits, dtype).astype(np.float64)


# ---------------------------------------------------------------- conversions

def pin_f16_widening(orc):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.f16_to_f64(b) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "fp16 NaN patterns differ"
    assert np.array_equal(got[~nan], ref[~nan]), "fp16 widening differs from NumPy"


def pin_bf16_widening(orc):
    import torch

    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.bf16_to_f64(b) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "bf16 NaN patterns differ"
    assert np.array_equal(got[~nan], ref[~nan]), "bf16 widening differs from PyTorch"


# ---------------------------------------------------------------- brute force

def _mp_decode(q, kc, vc, bt, cl, scale, dtype):
    import mpmath

    mpmath.mp.dps = 50
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = kc.shape
    g = Hq // Hkv
    out = np.zeros((S, Hq, D))
    qf, kf, vf = _widen(q, dtype), _widen(kc, dtype), _widen(vc, dtype)
    for s in range(S):
        for h in range(Hq):
            L = int(cl[s])
            if L == 0:
                continue
            rows = []
            for j in range(L):
                blk = int(bt[s, j // bs])
                rows.append((blk, j % bs))
            x = []
            for blk, off in rows:
                acc = mpmath.mpf(0)
                for d in range(D):
                    acc += mpmath.mpf(qf[s, h, d]) * mpmath.mpf(kf[blk, off, h // g, d])
                x.append(mpmath.mpf(scale) * acc)
            m = max(x)
            p = [mpmath.exp(xi - m) for xi in x]
            den = mpmath.fsum(p)
            for d in range(D):
                num = mpmath.fsum(pi * mpmath.mpf(vf[blk, off, h // g, d])
                                  for pi, (blk, off) in zip(p, rows))
                out[s, h, d] = float(num / den)
    return out


def pin_brute_force_tiny(orc):
    rng = np.random.default_rng(20240458)
    for trial in range(24):
        dtype = gen.F16 if trial % 2 == 0 else gen.BF16
        D = int(rng.integers(1, 5))
        bs = int(rng.integers(1, 4))
        Hkv = int(rng.integers(1, 3))
        g = int(rng.integers(1, 3))
        S = int(rng.integers(1, 3))
        ctx = rng.integers(0, 6, size=S)
        c = gen.random_decode_case(rng, num_seqs=S, num_q_heads=Hkv * g, num_kv_heads=Hkv,
                                   head_dim=D, block_size=bs, dtype=dtype, context_lens=ctx)
        scale = float(rng.uniform(0.2, 2.0))
        got = _decode(orc, dtype, c, scale)
        ref = _mp_decode(c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                         c["context_lens"], scale, dtype)
        err = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
        assert np.all(np.isfinite(got)), f"trial {trial}: non-finite oracle output"
        assert err.max() <= 1e-14, f"trial {trial}: brute-force mismatch {err.max():.3e}"


# ---------------------------------------------------------------- closed forms

def pin_context_one_returns_v0(orc):
    for dtype in (gen.F16, gen.BF16):
        c = _case(11, num_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                  dtype=dtype, context_lens=[1, 1, 1])
        out = _decode(orc, dtype, c)
        v = _widen(c["v_cache"], dtype)
        for s in range(3):
            blk = c["block_tables"][s, 0]
            for h in range(4):
                assert np.array_equal(out[s, h], v[blk, 0, h // 2]), "ctx=1 must return V_0"


def pin_identical_keys_give_mean_of_v(orc):
    for dtype in (gen.F16, gen.BF16):
        c = _case(12, num_seqs=2, num_q_heads=2, num_kv_heads=1, head_dim=32, block_size=16,
                  dtype=dtype, context_lens=[37, 5])
        kc = c["k_cache"]
        key = kc[c["block_tables"][0, 0], 0, 0].copy()
        for s in range(2):
            L = int(c["context_lens"][s])
            for j in range(L):
                kc[c["block_tables"][s, j // 16], j % 16, 0] = key
        out = _decode(orc, dtype, c)
        v = _widen(c["v_cache"], dtype)
        for s in range(2):
            L = int(c["context_lens"][s])
            rows = np.stack([v[c["block_tables"][s, j // 16], j % 16, 0] for j in range(L)])
            ref = rows.mean(axis=0)
            for h in range(2):
                assert np.allclose(out[s, h], ref, rtol=1e-13, atol=1e-13), \
                    "identical keys must give the mean of V"


def pin_dominant_logit_selects_its_row(orc):
    dtype = gen.F16
    c = _case(13, num_seqs=1, num_q_heads=1, num_kv_heads=1, head_dim=16, block_size=16,
              dtype=dtype, context_lens=[23])
    D = 16
    q = np.zeros(D, dtype=np.float32)
    q[3] = 1.0
    c["q"] = gen.f32_to_f16_bits(q).reshape(1, 1, D)
    kc = c["k_cache"]
    rng = np.random.default_rng(5)
    target = 17
    for j in range(23):
        k = rng.uniform(-0.5, 0.5, size=D).astype(np.float32)
        k[3] = 60.0 if j == target else float(rng.uniform(-1.0, 1.0))
        kc[c["block_tables"][0, j // 16], j % 16, 0] = gen.f32_to_f16_bits(k)
    out = _decode(orc, dtype, c, scale=1.0)
    v = _widen(c["v_cache"], dtype)[c["block_tables"][0, target // 16], target % 16, 0]
    # every other logit is at least 59 below: total weight elsewhere < 23 e^-59
    assert np.allclose(out[0, 0], v, rtol=1e-15, atol=1e-20 + 23 * math.exp(-59) * 8), \
        "a dominant logit must select its own V row"


def pin_large_logits_stay_finite(orc):
    """Softmax is shift invariant; logits near 1000 must not overflow."""
    D = 8
    dtype = gen.F16
    c = _case(14, num_seqs=1, num_q_heads=1, num_kv_heads=1, head_dim=D, block_size=16,
              dtype=dtype, context_lens=[2])
    q = np.zeros(D, dtype=np.float32)
    q[0] = 1.0
    c["q"] = gen.f32_to_f16_bits(q).reshape(1, 1, D)
    k0 = np.zeros(D, dtype=np.float32)
    k0[0] = 1.0
    k1 = np.zeros(D, dtype=np.float32)
    k1[0] = 1.0 + 2.0 ** -10
    blk = c["block_tables"][0, 0]
    c["k_cache"][blk, 0, 0] = gen.f32_to_f16_bits(k0)
    c["k_cache"][blk, 1, 0] = gen.f32_to_f16_bits(k1)
    scale = 1000.0
    out = _decode(orc, dtype, c, scale=scale)
    v = _widen(c["v_cache"], dtype)
    w = math.exp(scale * 2.0 ** -10)
    ref = (v[blk, 0, 0] + w * v[blk, 1, 0]) / (1.0 + w)
    assert np.all(np.isfinite(out)), "logits near 1000 overflowed"
    assert np.allclose(out[0, 0], ref, rtol=1e-13, atol=1e-13)


def pin_context_zero_gives_zeros(orc):
    c = _case(15, num_seqs=3, num_q_heads=2, num_kv_heads=2, head_dim=64, block_size=16,
              dtype=gen.F16, context_lens=[0, 5, 0])
    out = _decode(orc, gen.F16, c)
    assert np.array_equal(out[0], np.zeros_like(out[0])) and np.array_equal(out[2], np.zeros_like(out[2]))
    assert np.all(np.isfinite(out[1]))


def pin_golden_block_mapping(orc):
    for case in golden_cases.load_cases():
        c = golden_cases.build(case)
        out = orc.decode(c["dtype"], c["q"], c["k_cache"], c["v_cache"], c["block_tables"],
                         c["context_lens"], c["scale"])
        assert np.allclose(out, c["expected"], rtol=1e-14, atol=1e-14), \
            f"{case['name']}: oracle differs from the hand-derived output"


# ---------------------------------------------------------------- structure

def pin_permutation_invariance(orc):
    """Relabel physical blocks by a random permutation and move their contents."""
    for dtype, bs in ((gen.F16, 16), (gen.BF16, 256), (gen.F16, 3)):
        rng = np.random.default_rng(16 + bs)
        c = gen.random_decode_case(rng, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=32,
                                   block_size=bs, dtype=dtype, context_lens=[1, 40, 300, 17])
        base = _decode(orc, dtype, c)
        NB = c["num_blocks"]
        pi = rng.permutation(NB)
        kc = np.empty_like(c["k_cache"])
        vc = np.empty_like(c["v_cache"])
        kc[pi] = c["k_cache"]
        vc[pi] = c["v_cache"]
        bt = c["block_tables"].copy()
        m = bt >= 0
        bt[m] = pi[bt[m]]
        perm = orc.decode(dtype, c["q"], kc, vc, bt, c["context_lens"], c["scale"])
        assert np.array_equal(base, perm), "output changed under a relabelling of physical blocks"


def _dense_attention(c, dtype):
    """Static contiguous layout [S, Hkv, max_len, D] + library softmax."""
    from scipy.special import softmax

    q = _widen(c["q"], dtype)
    kc, vc = _widen(c["k_cache"], dtype), _widen(c["v_cache"], dtype)
    bt, cl = c["block_tables"], c["context_lens"]
    S, Hq, D = q.shape
    NB, bs, Hkv, _ = kc.shape
    g = Hq // Hkv
    Lmax = int(cl.max())
    Kd = np.zeros((S, Hkv, Lmax, D))
    Vd = np.zeros((S, Hkv, Lmax, D))
    for s in range(S):
        L = int(cl[s])
        j = np.arange(L)
        blocks = bt[s, j // bs]
        Kd[s, :, :L] = np.transpose(kc[blocks, j % bs], (1, 0, 2))
        Vd[s, :, :L] = np.transpose(vc[blocks, j % bs], (1, 0, 2))
    out = np.zeros((S, Hq, D))
    for s in range(S):
        L = int(cl[s])
        if L == 0:
            continue
        Kg = np.repeat(Kd[s, :, :L], g, axis=0)          # [Hq, L, D]
        Vg = np.repeat(Vd[s, :, :L], g, axis=0)
        logits = c["scale"] * np.einsum("hd,hld->hl", q[s], Kg)
        p = softmax(logits, axis=-1)
        out[s] = np.einsum("hl,hld->hd", p, Vg)
    return out


def pin_dense_equality(orc):
    for dtype, bs, g in ((gen.F16, 16, 1), (gen.BF16, 16, 4), (gen.F16, 256, 8)):
        rng = np.random.default_rng(17 + g)
        c = gen.random_decode_case(rng, num_seqs=5, num_q_heads=2 * g, num_kv_heads=2,
                                   head_dim=64, block_size=bs, dtype=dtype,
                                   context_lens=[1, 16, 17, 300, 600])
        got = _decode(orc, dtype, c)
        ref = _dense_attention(c, dtype)
        err = np.abs(got - ref) / np.maximum(1e-3, np.abs(ref))
        assert err.max() <= 1e-12, f"paged vs dense mismatch {err.max():.3e}"


def pin_gqa_equals_repeated_mha(orc):
    dtype = gen.BF16
    g, Hkv = 4, 2
    c = _case(18, num_seqs=3, num_q_heads=g * Hkv, num_kv_heads=Hkv, head_dim=32, block_size=16,
              dtype=dtype, context_lens=[5, 33, 64])
    gqa = _decode(orc, dtype, c)
    mha = orc.decode(dtype, c["q"], np.ascontiguousarray(np.repeat(c["k_cache"], g, axis=2)),
                     np.ascontiguousarray(np.repeat(c["v_cache"], g, axis=2)),
                     c["block_tables"], c["context_lens"], c["scale"])
    assert np.array_equal(gqa, mha), "grouped-query output differs from repeated-head MHA"
    # and the groups are contiguous: q heads 0..g-1 share kv head 0
    solo = orc.decode(dtype, np.ascontiguousarray(c["q"][:, :g]),
                      np.ascontiguousarray(c["k_cache"][:, :, :1]),
                      np.ascontiguousarray(c["v_cache"][:, :, :1]),
                      c["block_tables"], c["context_lens"], c["scale"])
    assert np.array_equal(gqa[:, :g], solo), "q heads 0..g-1 must read kv head 0"


def pin_sharing_equals_private_copies(orc):
    dtype = gen.F16
    rng = np.random.default_rng(19)
    c = gen.random_decode_case(rng, num_seqs=4, num_q_heads=2, num_kv_heads=2, head_dim=32,
                               block_size=16, dtype=dtype, context_lens=[40, 50, 33, 64],
                               shared_prefix_blocks=2)
    assert len({tuple(c["block_tables"][s, :2]) for s in range(4)}) == 1
    shared = _decode(orc, dtype, c)
    # give every sequence private copies of the shared blocks
    NB = c["num_blocks"]
    extra = 4 * 2
    kc = np.concatenate([c["k_cache"], np.zeros((extra,) + c["k_cache"].shape[1:], np.uint16)])
    vc = np.concatenate([c["v_cache"], np.zeros((extra,) + c["v_cache"].shape[1:], np.uint16)])
    bt = c["block_tables"].copy()
    nxt = NB
    for s in range(4):
        for i in range(2):
            src = bt[s, i]
            kc[nxt] = kc[src]
            vc[nxt] = vc[src]
            bt[s, i] = nxt
            nxt += 1
    private = orc.decode(dtype, c["q"], kc, vc, bt, c["context_lens"], c["scale"])
    assert np.array_equal(shared, private), "shared blocks must read like private copies"


def pin_split_identity(orc):
    dtype = gen.BF16
    rng = np.random.default_rng(20)
    c = gen.random_decode_case(rng, num_seqs=4, num_q_heads=4, num_kv_heads=2, head_dim=64,
                               block_size=16, dtype=dtype, context_lens=[1, 511, 513, 1500])
    direct = _decode(orc, dtype, c)
    for pt in (1, 7, 16, 512, 4096):
        part = orc.decode_partitioned(dtype, c["q"], c["k_cache"], c["v_cache"],
                                      c["block_tables"], c["context_lens"], c["scale"], pt)
        err = np.abs(part - direct).max()     # outputs are O(1): absolute bound
        assert err <= 1e-13, f"partition {pt}: split-K merge differs by {err:.3e}"


def pin_stale_entries_are_not_read(orc):
    dtype = gen.F16
    c = _case(21, num_seqs=2, num_q_heads=2, num_kv_heads=1, head_dim=32, block_size=16,
              dtype=dtype, context_lens=[17, 3])
    bt = np.full((2, 6), 1 << 30, dtype=np.int32)
    bt[:, :c["block_tables"].shape[1]] = c["block_tables"]
    bt[0, 2:] = -1
    bt[1, 1:] = 123456789
    c["block_tables"] = bt
    out = _decode(orc, dtype, c)
    assert np.all(np.isfinite(out)), "a stale slot or table entry was read"


def pin_refuses_out_of_pool_entry(orc):
    import oracle

    c = _case(22, num_seqs=1, num_q_heads=1, num_kv_heads=1, head_dim=16, block_size=16,
              dtype=gen.F16, context_lens=[20])
    c["block_tables"][0, 1] = c["num_blocks"]
    try:
        _decode(orc, gen.F16, c)
    except oracle.OracleError:
        return
    raise AssertionError("an out-of-pool table entry below the context must be refused")


# ---------------------------------------------------------------- append / copy

def pin_append_matches_scatter(orc):
    rng = np.random.default_rng(23)
    NB, bs, Hkv, D = 9, 16, 3, 64
    kc = rng.integers(0, 1 << 16, size=(NB, bs, Hkv, D), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, size=(NB, bs, Hkv, D), dtype=np.uint16)
    T = 7
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int32)
    slots[2] = -1
    k = rng.integers(0, 1 << 16, size=(T, Hkv, D), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(T, Hkv, D), dtype=np.uint16)
    ek, ev = kc.copy(), vc.copy()
    keep = slots >= 0
    ek.reshape(NB * bs, Hkv, D)[slots[keep]] = k[keep]
    ev.reshape(NB * bs, Hkv, D)[slots[keep]] = v[keep]
    orc.cache_append(k, v, slots, kc, vc)
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev), "append differs from a scatter"


def pin_copy_matches_block_copy(orc):
    rng = np.random.default_rng(24)
    NB, bs, Hkv, D = 12, 16, 2, 64
    kc = rng.integers(0, 1 << 16, size=(NB, bs, Hkv, D), dtype=np.uint16)
    vc = rng.integers(0, 1 << 16, size=(NB, bs, Hkv, D), dtype=np.uint16)
    pairs = np.array([[3, 7], [3, 9], [0, 11], [5, 1]], dtype=np.int32)
    ek, ev = kc.copy(), vc.copy()
    for s, d in pairs:
        ek[d] = ek[s]
        ev[d] = ev[s]
    orc.copy_blocks(pairs, kc, vc)
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev), "copy differs from a block copy"




# ---------------------------------------------------------------- FP8 (E4M3) cache

def pin_e4m3_codes_match_torch(orc):
    """Every code widens as PyTorch's float8_e4m3fn (the OCP E4M3 format) does."""
    import torch

    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = np.array([orc.e4m3_to_f64(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2, "E4M3 NaN codes differ"
    assert np.array_equal(got[~nan], ref[~nan]), "E4M3 widening differs from PyTorch"
    assert np.signbit(got[0x80]) and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def pin_e4m3_rounding_matches_torch(orc):
    """Below the saturation point, the encoder rounds as PyTorch's fp32 -> e4m3fn."""
    import torch

    rng = np.random.default_rng(31)
    ys = np.concatenate([rng.uniform(-447.9, 447.9, 4000), rng.uniform(-0.02, 0.02, 4000),
                         rng.standard_normal(4000) * 3]).astype(np.float32)
    # exact midpoints between neighbouring codes, where ties decide
    vals = np.array([orc.e4m3_to_f64(c) for c in range(0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    ys = np.concatenate([ys, mids, -mids])
    ref = torch.from_numpy(ys).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_from_f32(float(y)) for y in ys], dtype=np.uint8)
    assert np.array_equal(got, ref), f"{int((got != ref).sum())} roundings differ from PyTorch"


def pin_e4m3_roundtrip_and_ties_to_even(orc):
    vals = [orc.e4m3_to_f64(c) for c in range(256)]
    for c in range(256):
        if not math.isnan(vals[c]):
            assert orc.e4m3_from_f32(vals[c]) == c, f"code {c:#x} does not round-trip"
    for c in range(0x7E):
        mid = (vals[c] + vals[c + 1]) / 2
        even = c if c % 2 == 0 else c + 1
        assert orc.e4m3_from_f32(mid) == even, f"tie between {c:#x} and {c + 1:#x}"
        assert orc.e4m3_from_f32(np.nextafter(np.float32(mid), np.float32(1e9))) == c + 1
        assert orc.e4m3_from_f32(np.nextafter(np.float32(mid), np.float32(-1e9))) == c


def pin_e4m3_saturates(orc):
    for y, code in [(448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (470.0, 0x7E), (479.0, 0x7E),
                    (1e30, 0x7E),
                    (float("inf"), 0x7E), (-1e30, 0xFE), (-449.0, 0xFE)]:
        assert orc.e4m3_from_f32(y) == code, f"{y} should saturate to {code:#x}"


def _exact_e4m3_case(orc, seed, dtype=gen.F16):
    """A small paged case whose K/V values are E4M3 codes that fp16 holds exactly."""
    rng = np.random.default_rng(seed)
    c = _case(seed, num_seqs=3, num_q_heads=4, num_kv_heads=2, head_dim=32, block_size=16,
              dtype=dtype, context_lens=[1, 20, 45], poison=False)
    shape = c["k_cache"].shape
    kcode = rng.integers(0, 256, size=shape).astype(np.uint8)
    vcode = rng.integers(0, 256, size=shape).astype(np.uint8)
    for a in (kcode, vcode):
        a[(a & 0x7F) == 0x7F] = 0x38   # no NaN codes
        a[(a & 0x78) >= 0x60] &= 0xC7  # keep |value| small enough for tame logits
    f = np.vectorize(orc.e4m3_to_f64)
    kf, vf = f(kcode).astype(np.float16), f(vcode).astype(np.float16)
    assert np.array_equal(kf.astype(np.float64), f(kcode)), "values not exact in fp16"
    return c, kcode, vcode, kf.view(np.uint16), vf.view(np.uint16)


def pin_fp8_decode_equals_16bit_decode(orc):
    c, kcode, vcode, kbits, vbits = _exact_e4m3_case(orc, 41)
    ones = np.ones(2, dtype=np.float32)
    got = orc.decode_fp8(gen.F16, c["q"], kcode, vcode, ones, ones, c["block_tables"],
                         c["context_lens"], c["scale"])
    ref = orc.decode(gen.F16, c["q"], kbits, vbits, c["block_tables"], c["context_lens"], c["scale"])
    assert np.max(np.abs(got - ref)) <= 1e-13, "FP8 decode differs from the fp16 decode of the same values"


def pin_fp8_scales(orc):
    c, kcode, vcode, _, _ = _exact_e4m3_case(orc, 42)
    ks = np.array([0.5, 2.0], dtype=np.float32)
    vs = np.array([0.25, 4.0], dtype=np.float32)
    a = orc.decode_fp8(gen.F16, c["q"], kcode, vcode, ks, vs, c["block_tables"], c["context_lens"],
                       c["scale"])
    b = orc.decode_fp8(gen.F16, c["q"], kcode, vcode, ks, 2 * vs, c["block_tables"],
                       c["context_lens"], c["scale"])
    assert np.array_equal(b, 2 * a), "the V scale must scale the output"
    d = orc.decode_fp8(gen.F16, c["q"], kcode, vcode, 2 * ks, vs, c["block_tables"],
                       c["context_lens"], c["scale"] / 2)
    assert np.array_equal(d, a), "the K scale must act as a factor of the logits"
    # kv head 1's scales must reach exactly the query heads of group 1
    e = orc.decode_fp8(gen.F16, c["q"], kcode, vcode, ks, np.array([0.25, 8.0], np.float32),
                       c["block_tables"], c["context_lens"], c["scale"])
    assert np.array_equal(e[:, :2], a[:, :2]) and np.array_equal(e[:, 2:], 2 * a[:, 2:])


def pin_fp8_large_logits_stay_finite(orc):
    """Logits near 1000 (exp overflows fp64 without the max subtracted)."""
    S, H, D, bs = 1, 1, 32, 16
    q = np.full((S, H, D), gen.to_bits(np.float32(1.0), gen.F16), dtype=np.uint16)
    kc = np.full((1, bs, H, D), 0x7D, dtype=np.uint8)   # 416
    kc[0, 3] = 0x7E                                        # 448: the dominant key
    vc = np.zeros((1, bs, H, D), dtype=np.uint8)
    vc[0, 3] = 0x38                                        # 1.0
    one = np.ones(H, dtype=np.float32)
    scale = 1000.0 / (D * 448.0)
    out = orc.decode_fp8(gen.F16, q, kc, vc, one, one, np.zeros((S, 1), np.int32),
                         np.array([bs], np.int32), scale)
    assert np.all(np.isfinite(out)), "large logits must not overflow"
    # the dominant key's weight is 1 / (1 + 15 e^(-1000 (448 - 416) / 448))
    w = 1.0 / (1.0 + 15.0 * math.exp(-1000.0 * 32.0 / 448.0))
    assert abs(out[0, 0, 0] - w) < 1e-12


def pin_fp8_append_encodes_each_element(orc):
    import torch

    rng = np.random.default_rng(43)
    NB, bs, Hkv, D, T = 6, 16, 2, 32, 9
    for dtype in (gen.F16, gen.BF16):
        kc = rng.integers(0, 256, size=(NB, bs, Hkv, D), dtype=np.uint8)
        vc = kc.copy()
        ek, ev = kc.copy(), vc.copy()
        slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int32)
        slots[4] = -1
        k = gen.normal_bits(rng, (T, Hkv, D), dtype)
        v = gen.normal_bits(rng, (T, Hkv, D), dtype)
        ks = np.array([0.012, 0.02], dtype=np.float32)
        vs = np.array([0.03, 0.015], dtype=np.float32)
        orc.cache_append_fp8(dtype, k, v, slots, ks, vs, kc, vc)
        for src, scales, exp in ((k, ks, ek), (v, vs, ev)):
            y = gen.bits_to_f32(src, dtype) / scales[None, :, None]   # fp32 division
            assert np.abs(y).max() < 448
            codes = torch.from_numpy(np.ascontiguousarray(y)).to(torch.float8_e4m3fn)
            codes = codes.view(torch.uint8).numpy()
            keep = slots >= 0
            exp.reshape(NB * bs, Hkv, D)[slots[keep]] = codes[keep]
        assert np.array_equal(kc, ek) and np.array_equal(vc, ev), "FP8 append differs"


# ---------------------------------------------------------------- several query tokens per sequence

def _multi_case(seed, Tq, dtype=gen.BF16, ctx=(40, 5, 3, 70)):
    rng = np.random.default_rng(seed)
    c = _case(seed, num_seqs=len(ctx), num_q_heads=4, num_kv_heads=2, head_dim=32, block_size=16,
              dtype=dtype, context_lens=list(ctx))
    q = gen.normal_bits(rng, (len(ctx), Tq, 4, 32), dtype)
    return c, q


def pin_multi_one_token_is_decode(orc):
    c, q = _multi_case(51, 1)
    got = orc.decode_multi(gen.BF16, q, c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"])
    ref = orc.decode(gen.BF16, q[:, 0], c["k_cache"], c["v_cache"], c["block_tables"],
                     c["context_lens"], c["scale"])
    assert np.max(np.abs(got[:, 0] - ref)) <= 1e-14


def pin_multi_token_t_is_decode_over_its_prefix(orc):
    """Query t of Tq equals a one-token decode whose context ends at its own token."""
    Tq = 4
    c, q = _multi_case(52, Tq)
    got = orc.decode_multi(gen.BF16, q, c["k_cache"], c["v_cache"], c["block_tables"],
                           c["context_lens"], c["scale"])
    for t in range(Tq):
        lens = np.maximum(c["context_lens"] - Tq + t + 1, 0).astype(np.int32)
        ref = orc.decode(gen.BF16, q[:, t], c["k_cache"], c["v_cache"], c["block_tables"], lens,
                         c["scale"])
        assert np.max(np.abs(got[:, t] - ref)) <= 1e-14, f"query token {t}"
    # a context shorter than Tq leaves the first queries without tokens: zero rows
    assert np.all(got[2, 0] == 0) and np.any(got[2, 3] != 0)


def pin_multi_is_causal(orc):
    """Tokens after a query's own position never reach it (they are NaN here)."""
    Tq = 3
    c, q = _multi_case(53, Tq, ctx=(33, 20))
    kc, vc = c["k_cache"].copy(), c["v_cache"].copy()
    nan = np.uint16(gen.NAN_BITS[gen.BF16])
    bs = 16
    for s, L in enumerate(c["context_lens"]):
        j = L - 1   # the last new token: only query Tq - 1 may see it
        slot = int(c["block_tables"][s, j // bs]) * bs + j % bs
        kc.reshape(-1, 2, 32)[slot] = nan
        vc.reshape(-1, 2, 32)[slot] = nan
    got = orc.decode_multi(gen.BF16, q, kc, vc, c["block_tables"], c["context_lens"], c["scale"])
    assert np.all(np.isfinite(got[:, :Tq - 1])), "an earlier query read a later token"
    assert np.all(np.isnan(got[:, Tq - 1])), "the last query must read every token"

# ---------------------------------------------------------------- block size 8, swap

def pin_block_size_8_equals_16(orc):
    """A pool of 16-token blocks read as twice as many 8-token blocks gives the same output."""
    c = _case(61, num_seqs=4, num_q_heads=4, num_kv_heads=2, head_dim=32, block_size=16,
              dtype=gen.F16, context_lens=[1, 9, 24, 47])
    NB = c["num_blocks"]
    k8 = c["k_cache"].reshape(NB * 2, 8, 2, 32)
    v8 = c["v_cache"].reshape(NB * 2, 8, 2, 32)
    t16 = c["block_tables"]
    t8 = np.empty((t16.shape[0], 2 * t16.shape[1]), dtype=np.int32)
    t8[:, 0::2] = np.where(t16 >= 0, 2 * t16, -1)
    t8[:, 1::2] = np.where(t16 >= 0, 2 * t16 + 1, -1)
    a = _decode(orc, gen.F16, c)
    b = orc.decode(gen.F16, c["q"], k8, v8, t8, c["context_lens"], c["scale"])
    assert np.array_equal(a, b), "8-token blocks must read the same tokens"


def pin_swap_matches_block_copy(orc):
    rng = np.random.default_rng(62)
    bs, Hkv, D = 16, 2, 32
    dev_k = rng.integers(0, 1 << 16, size=(10, bs, Hkv, D), dtype=np.uint16)
    dev_v = rng.integers(0, 1 << 16, size=(10, bs, Hkv, D), dtype=np.uint16)
    host_k = rng.integers(0, 1 << 16, size=(6, bs, Hkv, D), dtype=np.uint16)
    host_v = rng.integers(0, 1 << 16, size=(6, bs, Hkv, D), dtype=np.uint16)
    pairs = np.array([[7, 0], [2, 5], [9, 3]], dtype=np.int32)
    ek, ev = host_k.copy(), host_v.copy()
    for s, d in pairs:
        ek[d], ev[d] = dev_k[s], dev_v[s]
    orc.swap_blocks(pairs, dev_k, dev_v, host_k, host_v)
    assert np.array_equal(host_k, ek) and np.array_equal(host_v, ev), "swap differs from a block copy"
    try:
        orc.swap_blocks(np.array([[10, 0]], np.int32), dev_k, dev_v, host_k, host_v)
    except Exception:
        pass
    else:
        raise AssertionError("a source block outside the pool must be refused")


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
