"""Benchmark: paged decode attention on B200 through the C ABI of libpa.so.

One *step* is one pass of the whole hot path over one decode batch of the
workload: copy-on-write of shared blocks (pa_copy_blocks), append of each
sequence's new token (pa_cache_append), then decode attention over every
context (pa_decode).  Inputs are seeded synthetic data with the workload's
shapes (paged_kv_cache_458_b200.gen); the K/V pool and every step's inputs are
resident in HBM before the timed region starts.

The reported metric is the decode's K/V-read bandwidth: algorithmic bytes of
the decode (K and V rows of every context, q, out, block-table entries and
context lengths) divided by the device time of the whole step, plus decode
tokens/s per layer.  The K timed steps run between one pair of CUDA events
with nothing else on the stream.  The `roofline` object is the decode
kernels alone, timed with CUDA events around each step's decode in a second
pass over the same steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference]

With N > 1 (torchrun) every rank runs its own replica of the workload (its
own seed); there is no data exchange, only a max-over-ranks of the device
time.  `--impl reference` times the CPU oracle (fp64, all host cores) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_458_b200 import gen  # noqa: E402

METRIC = ("paged decode-attn KV-read GB/s (% of B200 HBM peak); decode tokens/s per layer")
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
VARIANTS = {"auto": 0, "cuda_cores": 1, "tensor_cores": 2}
# Timed beside the main workload, decode only, in the same run.
OTHER_WORKLOADS = ("llama2_7b", "qwen_7b_prefix", "llama2_70b_beam")


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=3000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--workload", default="mistral_7b_gqa", choices=sorted(gen.WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--partition-tokens", type=int, default=0)
    p.add_argument("--variant", default="auto", choices=sorted(VARIANTS),
                   help="decode kernel: auto, cuda_cores or tensor_cores")
    p.add_argument("--block-size", type=int, default=0,
                   help="re-block the workload's pool into blocks of this many tokens "
                        "(a divisor of its block size, e.g. 8); every token keeps its slot")
    p.add_argument("--swap", action="store_true",
                   help="also time pa_swap_blocks between the pool and pinned host memory")
    p.add_argument("--query-tokens", type=int, default=1,
                   help="query tokens per sequence (pa_decode_multi when > 1): the last ones "
                        "of each context, causal among themselves")
    p.add_argument("--kv-cache", default="dtype", choices=["dtype", "fp8"],
                   help="K/V cache elements: the workload's 16-bit dtype, or E4M3 codes with "
                        "per-kv-head scales (halves the K/V bytes)")
    p.add_argument("--shared-prefix", default="auto", choices=["auto", "on", "off"],
                   help="read blocks shared by consecutive sequences once per group; auto: on "
                        "when the workload's tables share their first block")
    p.add_argument("--cycle", type=int, default=64,
                   help="distinct precomputed steps; longer runs replay them in order")
    p.add_argument("--e2e-steps", type=int, default=500)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--per-workload", default=",".join(OTHER_WORKLOADS),
                   help="further workloads whose decode is timed beside the main line "
                        "(comma list; empty for none)")
    p.add_argument("--per-workload-steps", type=int, default=300)
    return p.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(x: float, dist, device=None) -> float:
    """Largest value of `x` over all ranks (a timing reduction, not data)."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, dist, device=None) -> float:
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# byte and flop accounting (per decode)


def decode_bytes(ctx: np.ndarray, num_q_heads, num_kv_heads, head_dim, block_size, elem=2,
                 kv_elem=None, query_tokens=1) -> int:
    """Algorithmic bytes of one decode: K+V rows (kv_elem bytes per element,
    default elem) once per sequence, q+out for each query token, table
    entries, lengths."""
    ctx = np.asarray(ctx, dtype=np.int64)
    S = ctx.shape[0]
    kv = int(2 * ctx.sum() * num_kv_heads * head_dim * (elem if kv_elem is None else kv_elem))
    qo = 2 * S * query_tokens * num_q_heads * head_dim * elem
    tables = int(4 * np.ceil(ctx / block_size).sum())
    return kv + qo + tables + 4 * S


def tables_share_blocks(tables: np.ndarray, ctx: np.ndarray) -> bool:
    """Whether two consecutive sequences start with the same physical block."""
    live = np.asarray(ctx) > 0
    first = np.asarray(tables)[:, 0]
    return bool(np.any(live[1:] & live[:-1] & (first[1:] == first[:-1])))


def unique_kv_bytes(tables: np.ndarray, ctx: np.ndarray, block_size, num_kv_heads, head_dim,
                    elem=2) -> int:
    """K+V bytes of the distinct slots a decode reads (shared blocks once)."""
    slots = []
    ar = np.arange(block_size, dtype=np.int64)
    for s in range(len(ctx)):
        L = int(ctx[s])
        if L <= 0:
            continue
        nb = -(-L // block_size)
        rows = (np.asarray(tables[s, :nb], dtype=np.int64)[:, None] * block_size + ar).reshape(-1)
        slots.append(rows[:L])
    n = len(np.unique(np.concatenate(slots))) if slots else 0
    return 2 * n * num_kv_heads * head_dim * elem


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read-only)


class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, uuid: str | None, period_s: float = 0.005):
        self.uuid, self.period = uuid, period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.error = None

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            # CUDA and NVML may number devices differently: match by UUID.
            self._h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:  # noqa: BLE001 - clocks are reported, never required
            self.error = repr(e)
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception as e:  # noqa: BLE001
                self.error = repr(e)
                return
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples),
                **({"error": self.error} if self.error else {})}


def device_uuid(torch) -> str:
    u = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    return u if u.startswith("GPU-") else "GPU-" + u


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(path: str) -> str:
    """First 16 hex digits of the SHA-256 of a kernel source without its
    blank lines and whole-line // comments: a comment edit keeps the digest,
    any change to code (trailing comments included) changes it."""
    with open(path, "rb") as f:
        lines = f.read().split(b"\n")
    kept = [ln for ln in lines if ln.strip() and not ln.strip().startswith(b"//")]
    return hashlib.sha256(b"\n".join(kept)).hexdigest()[:16]


def profiled_traffic(workload: str, variant: str, step_bytes: float):
    """DRAM bytes per decode launch from the committed ncu summary of this
    workload, if it was taken on the kernel that runs (same variant, same
    source digest); else None.  The capture is of one seeded step; its
    DRAM/algorithmic ratio is applied to this run's average step bytes."""
    path = os.path.join(ROOT, "profiles", f"pa_decode_{workload}.json")
    try:
        with open(path) as f:
            prof = json.load(f)
        digest = source_digest(os.path.join(ROOT, prof["source"]))
    except (OSError, ValueError, KeyError):
        return None
    if prof.get("variant") != variant or prof.get("source_sha256_16") != digest:
        return None
    return int(round(prof["traffic_over_algorithmic"] * step_bytes))


# ---------------------------------------------------------------------------
# the GPU arm


class DeviceWorkload:
    """The pool and a cycle of precomputed steps, resident on the device."""

    def __init__(self, case, torch, pa, partition_tokens: int, variant: int = 0,
                 shared_prefix: int = 0, fp8: bool = False, query_tokens: int = 1):
        self.case = case
        self.torch, self.pa = torch, pa
        dt = pa.torch_dtype(case.dtype)
        self.dt = dt

        def dev16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dt).cuda()

        def dev32(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()

        self.k_cache, self.v_cache = dev16(case.k_cache), dev16(case.v_cache)
        self.fp8 = fp8
        self.tq = query_tokens
        qrng = np.random.default_rng(case.seed + 77)
        self.steps = []
        for st in case.steps:
            q = st.q if query_tokens == 1 else gen.normal_bits(
                qrng, (case.num_seqs, query_tokens, case.num_q_heads, case.head_dim), case.dtype)
            self.steps.append(dict(
                pairs=dev32(st.pairs.reshape(-1, 2)) if len(st.pairs) else None,
                n_pairs=len(st.pairs), slots=dev32(st.slot_mapping), k_new=dev16(st.k_new),
                v_new=dev16(st.v_new), q=dev16(q), tables=dev32(st.block_tables),
                lens=dev32(st.context_lens), max_len=int(st.context_lens.max())))
        self.max_len = max(s["max_len"] for s in self.steps)
        self.shape = pa.make_shape(
            num_seqs=case.num_seqs, num_q_heads=case.num_q_heads, num_kv_heads=case.num_kv_heads,
            head_dim=case.head_dim, block_size=case.block_size, num_blocks=case.num_blocks,
            max_blocks_per_seq=case.max_blocks_per_seq, partition_tokens=partition_tokens,
            dtype=case.dtype, variant=variant, shared_prefix=shared_prefix,
            cache_format=pa.PA_CACHE_FP8_E4M3 if fp8 else pa.PA_CACHE_AS_DTYPE)
        if fp8:
            # E4M3 pools encoded from the 16-bit ones by the library's own
            # append over every slot, with per-kv-head scales amax / 448
            NB, bs, Hkv, D = case.k_cache.shape
            k16, v16 = self.k_cache, self.v_cache
            amax = lambda t: t.float().abs().reshape(-1, Hkv, D).amax(dim=(0, 2))  # noqa: E731
            self.k_scale = (amax(k16) / 448.0).clamp_min(1e-12).contiguous()
            self.v_scale = (amax(v16) / 448.0).clamp_min(1e-12).contiguous()
            self.k_cache = torch.empty((NB, bs, Hkv, D), dtype=torch.uint8, device="cuda")
            self.v_cache = torch.empty_like(self.k_cache)
            slots = torch.arange(NB * bs, dtype=torch.int32, device="cuda")
            pa.pa_cache_append_fp8(k16, v16, slots, NB * bs, self.k_cache, self.v_cache,
                                   self.k_scale, self.v_scale, self.shape)
            torch.cuda.synchronize()
            del k16, v16
        self.ws_bytes = (pa.pa_decode_workspace_bytes(self.shape, self.max_len) if self.tq == 1 else
                         pa.pa_decode_multi_workspace_bytes(self.shape, self.tq, self.max_len))
        self.ws = torch.empty(max(16, self.ws_bytes), dtype=torch.uint8, device="cuda")
        self.out = torch.empty((case.num_seqs, query_tokens, case.num_q_heads, case.head_dim)
                               if query_tokens > 1 else
                               (case.num_seqs, case.num_q_heads, case.head_dim), dtype=dt,
                               device="cuda")

    def step(self, i: int, stream, ev=None):
        """Enqueue step i (mod the cycle); ev = (start, mid, end) events or None."""
        self.enqueue(self.steps[i % len(self.steps)], stream, ev)

    def enqueue(self, st: dict, stream, ev=None, out=None):
        pa = self.pa
        out = self.out if out is None else out
        if ev:
            ev[0].record(stream)
        if st["n_pairs"]:
            pa.pa_copy_blocks(st["pairs"], st["n_pairs"], self.k_cache, self.v_cache, self.shape,
                              stream.cuda_stream)
        if self.fp8:
            pa.pa_cache_append_fp8(st["k_new"], st["v_new"], st["slots"], self.case.num_seqs,
                                   self.k_cache, self.v_cache, self.k_scale, self.v_scale,
                                   self.shape, stream.cuda_stream)
        else:
            pa.pa_cache_append(st["k_new"], st["v_new"], st["slots"], self.case.num_seqs,
                               self.k_cache, self.v_cache, self.shape, stream.cuda_stream)
        if ev:
            ev[1].record(stream)
        if self.fp8:
            pa.pa_decode_fp8(st["q"], self.k_cache, self.v_cache, self.k_scale, self.v_scale,
                             st["tables"], st["lens"], self.case.scale, out, self.shape,
                             st["max_len"], self.ws, self.ws_bytes, stream.cuda_stream)
        elif self.tq > 1:
            pa.pa_decode_multi(st["q"], self.k_cache, self.v_cache, st["tables"], st["lens"],
                               self.case.scale, out, self.shape, self.tq, st["max_len"], self.ws,
                               self.ws_bytes, stream.cuda_stream)
        else:
            pa.pa_decode(st["q"], self.k_cache, self.v_cache, st["tables"], st["lens"],
                         self.case.scale, out, self.shape, st["max_len"], self.ws,
                         self.ws_bytes, stream.cuda_stream)
        if ev:
            ev[2].record(stream)


def split_blocks(case, factor: int):
    """The same case over blocks `factor` times smaller: each block b becomes
    blocks factor*b .. factor*b + factor-1, so every token keeps its slot."""
    import dataclasses

    if factor == 1:
        return case
    NB, bs, Hkv, D = case.k_cache.shape
    nbs = bs // factor

    def tables(t):
        out = np.full((t.shape[0], t.shape[1] * factor), -1, dtype=np.int32)
        for i in range(factor):
            out[:, i::factor] = np.where(t >= 0, factor * t + i, -1)
        return out

    def pairs(p):
        p = np.asarray(p, dtype=np.int32).reshape(-1, 2)
        return np.concatenate([factor * p + i for i in range(factor)]) if len(p) else p

    steps = [dataclasses.replace(st, block_tables=tables(st.block_tables), pairs=pairs(st.pairs))
             for st in case.steps]
    return dataclasses.replace(
        case, block_size=nbs, num_blocks=NB * factor, max_blocks_per_seq=case.max_blocks_per_seq * factor,
        k_cache=case.k_cache.reshape(NB * factor, nbs, Hkv, D),
        v_cache=case.v_cache.reshape(NB * factor, nbs, Hkv, D),
        block_tables=tables(case.block_tables), steps=steps)


def swap_bandwidth(w, torch, pa, n_blocks: int = 256, reps: int = 5):
    """pa_swap_blocks out to pinned host memory and back in, GB/s each way."""
    NB = w.case.num_blocks
    n = min(n_blocks, NB)
    hk = torch.empty((n,) + tuple(w.k_cache.shape[1:]), dtype=w.k_cache.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.tensor([[b, i] for i, b in enumerate(range(NB - n, NB))], dtype=torch.int32,
                             device="cuda")
    in_pairs = out_pairs.flip(1).contiguous()
    nbytes = 2 * hk.numel() * hk.element_size()
    res = {}
    for name, args in (("out", (out_pairs, n, w.k_cache, w.v_cache, NB, hk, hv, n)),
                       ("in", (in_pairs, n, hk, hv, n, w.k_cache, w.v_cache, NB))):
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            pa.pa_swap_blocks(*args, w.shape)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        res[f"{name}_gbs"] = round(nbytes / (sorted(ts)[len(ts) // 2] * 1e-3) / 1e9, 2)
    res["blocks"] = n
    res["bytes_each_way"] = nbytes
    return res


def time_other_workload(name, args, rank, torch, pa, stream, peak):
    """Decode of another workload in the same run: automatic variant (shared
    prefixes on where the tables share blocks), W warm-up steps, then K steps
    timed as one stretch and again with events around each decode.  Returns
    the decode GB/s and its roofline fraction; for workloads whose tables
    share blocks, also the GB/s of the distinct K/V slots read."""
    steps = max(1, args.per_workload_steps)
    warm = max(3, args.warmup)
    n_cycle = max(1, min(args.cycle, steps + warm))
    case = gen.make_case(name, n_steps=n_cycle, poison=False,
                         seed=gen.SEED_BASE + gen.WORKLOADS[name].number + 1000 * rank)
    shared = int(tables_share_blocks(case.steps[0].block_tables, case.steps[0].context_lens))
    w = DeviceWorkload(case, torch, pa, case.workload.partition_tokens, 0, shared)
    bytes_per = [decode_bytes(s.context_lens, case.num_q_heads, case.num_kv_heads, case.head_dim,
                              case.block_size) for s in case.steps]
    with torch.cuda.stream(stream):
        for i in range(warm):
            w.step(i, stream)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(device_uuid(torch)) as clocks:
            t0.record(stream)
            for i in range(steps):
                w.step(warm + i, stream)
            t1.record(stream)
            torch.cuda.synchronize()
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
        for i in range(steps):
            w.step(warm + i, stream, evs[i])
        torch.cuda.synchronize()
    status, bits = pa.pa_last_device_error(stream.cuda_stream)
    if status != pa.PA_OK:
        raise RuntimeError(f"device check in {name}: {bits:#x}")
    step_bytes = sum(bytes_per[(warm + i) % n_cycle] for i in range(steps))
    dec_ms = sum(evs[i][1].elapsed_time(evs[i][2]) for i in range(steps))
    dec_gbs = step_bytes / (dec_ms * 1e-3) / 1e9
    resolved = {1: "cuda_cores", 2: "tensor_cores",
                3: "shared_prefix"}[pa.pa_decode_resolved_variant(w.shape)]
    res = {
        "decode_variant": resolved,
        "steps": steps, "warmup": warm,
        "step_gbs": round(step_bytes / (t0.elapsed_time(t1) * 1e-3) / 1e9, 2),
        "decode_gbs": round(dec_gbs, 2),
        "decode_ms_per_step": round(dec_ms / steps, 5),
        "decode_bytes_per_step": int(step_bytes / steps),
        "frac": round(dec_gbs / peak, 4),
        "traffic": profiled_traffic(name, resolved, step_bytes / steps),
        "tokens_per_s_per_layer": round(case.num_seqs * steps / (dec_ms * 1e-3), 1),
        "clocks": clocks.summary(),
    }
    if shared:
        # unique bytes of the timed steps: distinct K/V slots (shared blocks
        # once) plus the same q, out, table and length bytes
        per_cycle = {}
        uniq = 0
        for i in range(steps):
            j = (warm + i) % n_cycle
            if j not in per_cycle:
                st = case.steps[j]
                kv_logical = 2 * int(st.context_lens.sum()) * case.num_kv_heads * case.head_dim * 2
                per_cycle[j] = bytes_per[j] - kv_logical + unique_kv_bytes(
                    st.block_tables, st.context_lens, case.block_size, case.num_kv_heads,
                    case.head_dim)
            uniq += per_cycle[j]
        res["unique_bytes_per_step"] = int(uniq / steps)
        res["unique_gbs"] = round(uniq / (dec_ms * 1e-3) / 1e9, 2)
        res["unique_frac"] = round(res["unique_gbs"] / peak, 4)
    del w
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local, dist):
    import torch

    from paged_kv_cache_458_b200 import pa

    torch.cuda.set_device(local)
    stream = torch.cuda.Stream()
    n_cycle = max(1, min(args.cycle, args.steps + args.warmup))
    case = gen.make_case(args.workload, n_steps=n_cycle, poison=False,
                         seed=gen.SEED_BASE + gen.WORKLOADS[args.workload].number + 1000 * rank)
    if args.block_size:
        if case.block_size % args.block_size:
            raise SystemExit(f"--block-size must divide the workload's {case.block_size}")
        case = split_blocks(case, case.block_size // args.block_size)
    shared = {"on": 1, "off": 0}.get(args.shared_prefix)
    if shared is None:
        shared = int(args.variant == "auto" and
                     tables_share_blocks(case.steps[0].block_tables, case.steps[0].context_lens))
    fp8 = args.kv_cache == "fp8"
    partition = args.partition_tokens or case.workload.partition_tokens
    if args.query_tokens > 1 and fp8:
        raise SystemExit("--query-tokens > 1 reads a 16-bit cache")
    w = DeviceWorkload(case, torch, pa, partition, VARIANTS[args.variant], shared, fp8,
                       args.query_tokens)
    kv_elem = 1 if fp8 else 2
    bytes_per = [decode_bytes(s.context_lens, case.num_q_heads, case.num_kv_heads, case.head_dim,
                              case.block_size, kv_elem=kv_elem, query_tokens=args.query_tokens)
                 for s in case.steps]
    pool_bytes = 2 * case.k_cache.nbytes * kv_elem // 2
    kv_step0 = 2 * int(case.steps[0].context_lens.sum()) * case.num_kv_heads * case.head_dim * kv_elem

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            w.step(i, stream)
        torch.cuda.synchronize()
        st0, bits = pa.pa_last_device_error(stream.cuda_stream)
        if st0 != pa.PA_OK:
            raise RuntimeError(f"device check during warm-up: {bits:#x}")

        # The timed region: K steps between one pair of events, nothing else
        # on the stream, so consecutive kernels overlap as they do in use.
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        launches0 = pa.pa_kernel_launches()
        with ClockSampler(device_uuid(torch)) as clocks:
            t0.record(stream)
            for i in range(args.steps):
                w.step(args.warmup + i, stream)
            t1.record(stream)
            torch.cuda.synchronize()
        launches = pa.pa_kernel_launches() - launches0
        if dist is not None:
            dist.barrier()
        st1, bits = pa.pa_last_device_error(stream.cuda_stream)
        if st1 != pa.PA_OK:
            raise RuntimeError(f"device check during the timed steps: {bits:#x}")
        # Then the same K steps again with events around each step's decode,
        # for the decode kernels' own time (the roofline): events between
        # kernels keep them from overlapping, so this pass is not the value.
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
               for _ in range(args.steps)]
        for i in range(args.steps):
            w.step(args.warmup + i, stream, evs[i])
        torch.cuda.synchronize()

    total_ms = t0.elapsed_time(t1)
    dec_ms = [evs[i][1].elapsed_time(evs[i][2]) for i in range(args.steps)]
    dec_total_ms = sum(dec_ms)
    step_bytes = sum(bytes_per[(args.warmup + i) % n_cycle] for i in range(args.steps))
    max_ms = max_over_ranks(total_ms, dist, "cuda")
    all_bytes = sum_over_ranks(float(step_bytes), dist, "cuda")
    value = all_bytes / (max_ms * 1e-3) / 1e9

    peak, peak_kind = measured_peak()
    achieved = step_bytes / (dec_total_ms * 1e-3) / 1e9
    resolved = {1: "cuda_cores", 2: "tensor_cores",
                3: "shared_prefix"}[pa.pa_decode_resolved_variant(w.shape)]
    if args.query_tokens > 1:
        resolved = "multi_query"
    traffic = (None if fp8 or args.query_tokens > 1 or args.block_size else
               profiled_traffic(args.workload, resolved, step_bytes / args.steps))
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(max_ms / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if fp8 else gen.DTYPE_NAMES[case.dtype], "accum_dtype": "f32",
        "data": "synthetic (seeded N(0,1) values, shapes and block structure of the workload)",
        "config": {
            **workload_config(args, case, world, fp8),
            "partition_tokens": pa.pa_decode_partition_tokens(w.shape),
            "decode_variant": f"{args.variant} -> {resolved}",
            "shared_prefix": bool(shared),
            "steps_cycle": n_cycle,
            "l2": (f"inputs larger than L2: {kv_step0 / 1e6:.0f} MB of K/V read per decode, "
                   f"{pool_bytes / 1e6:.0f} MB pool, L2 126 MB; no flush"),
        },
        "tokens_per_s_per_layer": round(case.num_seqs * args.query_tokens * args.steps * world /
                                        (max_ms * 1e-3), 1),
        "decode_ms_per_step": round(dec_total_ms / args.steps, 5),
        "decode_bytes_per_step": int(step_bytes / args.steps),
        "pct_of_8tbps": round(100 * value / 8000.0, 2),
        "roofline": {
            "bound": "hbm",
            "kernel": (f"pa_decode ({resolved} partition kernel + split-K merge kernel)"
                       if resolved != "shared_prefix" else
                       "pa_decode (plan + tensor-core kernel over every group's row list "
                       "+ split-K merge)"),
            "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
        },
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
    }
    if case.workload.name in ("qwen_7b_prefix", "llama2_70b_beam"):
        st = case.steps[0]
        result["unique_kv_bytes_step0"] = unique_kv_bytes(
            st.block_tables, st.context_lens, case.block_size, case.num_kv_heads, case.head_dim,
            elem=kv_elem)
        # the same decode counted in distinct K/V slots (shared blocks once)
        result["unique_kv_gbs_step0_est"] = round(
            result["unique_kv_bytes_step0"] / (dec_total_ms / args.steps * 1e-3) / 1e9, 2)
    if args.swap:
        result["swap"] = swap_bandwidth(w, torch, pa)
    if not args.no_e2e:
        result["e2e"] = run_e2e(args, w, stream, bytes_per, n_cycle, dist)
    others = [n for n in args.per_workload.split(",") if n and n != args.workload]
    unknown = [n for n in others if n not in gen.WORKLOADS]
    if unknown:
        raise SystemExit(f"--per-workload: unknown workloads {unknown}")
    if others:
        del w
        torch.cuda.empty_cache()
        result["per_workload"] = {n: time_other_workload(n, args, rank, torch, pa, stream, peak)
                                  for n in others}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(case, args.cpu_seconds, case.steps[0])
    return result


def run_e2e(args, w, stream, bytes_per, n_cycle, dist):
    """Same metric through the public calls with host buffers: every step
    copies its inputs from pinned host memory and reads its output back.
    As a serving loop would, the copies run on their own streams: step i+1's
    inputs go up while step i computes, and step i's output comes back while
    step i+1 computes (two output buffers)."""
    import torch

    case = w.case
    host = []
    for i, st in enumerate(case.steps):
        def pin16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(w.dt).pin_memory()

        def pin32(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).pin_memory()

        host.append(dict(pairs=pin32(st.pairs.reshape(-1, 2)) if len(st.pairs) else None,
                         n_pairs=len(st.pairs), slots=pin32(st.slot_mapping), k_new=pin16(st.k_new),
                         v_new=pin16(st.v_new), q=w.steps[i]["q"].cpu().pin_memory(),
                         tables=pin32(st.block_tables),
                         lens=pin32(st.context_lens), max_len=int(st.context_lens.max())))
    outs = [w.out, torch.empty_like(w.out)]
    out_host = [torch.empty(w.out.shape, dtype=w.dt).pin_memory() for _ in range(2)]
    dev = [dict((k, (torch.empty_like(v, device="cuda") if isinstance(v, torch.Tensor) else v))
                for k, v in h.items()) for h in host]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    free = [None] * len(dev)      # compute done with dev[j]
    fetched = [None, None]        # output buffer b read back
    h2d = 0
    steps = min(args.e2e_steps, args.steps)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    up.wait_event(ev0)
    down.wait_event(ev0)
    for i in range(steps):
        j = (args.warmup + i) % n_cycle
        b = i % 2
        h, d = host[j], dev[j]
        with torch.cuda.stream(up):
            if free[j] is not None:
                up.wait_event(free[j])
            for k, v in h.items():
                if isinstance(v, torch.Tensor):
                    d[k].copy_(v, non_blocking=True)
                    h2d += v.numel() * v.element_size()
            ready = torch.cuda.Event()
            ready.record(up)
        stream.wait_event(ready)
        if fetched[b] is not None:
            stream.wait_event(fetched[b])
        with torch.cuda.stream(stream):
            w.enqueue(d, stream, out=outs[b])
        done = torch.cuda.Event()
        done.record(stream)
        free[j] = done
        with torch.cuda.stream(down):
            down.wait_event(done)
            out_host[b].copy_(outs[b], non_blocking=True)
            fetched[b] = torch.cuda.Event()
            fetched[b].record(down)
    for e in fetched:
        if e is not None:
            stream.wait_event(e)
    ev1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), dist, "cuda")
    all_bytes = sum_over_ranks(float(sum(bytes_per[(args.warmup + i) % n_cycle]
                                         for i in range(steps))), dist, "cuda")
    return {"value": round(all_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "steps": steps, "ms_per_step": round(ms / steps, 5),
            "h2d_bytes_per_step": int(h2d // steps),
            "d2h_bytes_per_step": int(out_host[0].numel() * out_host[0].element_size()),
            "copies": "inputs up and outputs back on their own streams, overlapping the "
                      "neighbouring steps' kernels"}


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)


def _oracle_sample(case, st, n_seqs, orc, threads):
    sl = slice(0, n_seqs)
    t0 = time.perf_counter()
    orc.decode(case.dtype, st.q[sl], case.k_cache, case.v_cache, st.block_tables[sl],
               st.context_lens[sl], case.scale, num_threads=threads)
    dt = time.perf_counter() - t0
    nbytes = decode_bytes(st.context_lens[sl], case.num_q_heads, case.num_kv_heads, case.head_dim,
                          case.block_size)
    return dt, nbytes


def _timed_oracle(case, st, orc, threads, seconds):
    """Decode the first sequences of the batch, as many as about `seconds`
    of work on `threads` threads (the whole batch again while under half of
    it); returns (seconds, algorithmic bytes, sequences, repetitions)."""
    dt1, _ = _oracle_sample(case, st, 1, orc, threads)
    n = int(max(1, min(case.num_seqs, seconds / max(dt1, 1e-6))))
    dt, nbytes = _oracle_sample(case, st, n, orc, threads)
    reps = 1
    while dt < 0.5 * seconds:  # the whole batch took less: decode it again
        d, b = _oracle_sample(case, st, n, orc, threads)
        dt, nbytes, reps = dt + d, nbytes + b, reps + 1
    return dt, nbytes, n, reps


def cpu_baseline(case, seconds: float, st):
    """The fp64 oracle on the host cores, on the first sequences of the batch
    (sized to about `seconds` of work on all cores, and a third of that on one
    thread); reported as GB/s of algorithmic bytes."""
    import oracle

    orc = oracle.load()
    cores = len(os.sched_getaffinity(0))
    threads = orc.num_threads(cores)
    dt, nbytes, n, reps = _timed_oracle(case, st, orc, threads, seconds)
    dt_1, nbytes_1, n_1, reps_1 = _timed_oracle(case, st, orc, 1, seconds / 3)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"fp64 C oracle, decode of the first {n} of {case.num_seqs} sequences of step 0, "
                      f"{reps} time(s) ({nbytes / 1e6:.1f} MB algorithmic), {dt:.2f} s wall, "
                      f"{threads} threads",
            "single_thread": {
                "value": round(nbytes_1 / dt_1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                "sample": f"the first {n_1} sequences, {reps_1} time(s) "
                          f"({nbytes_1 / 1e6:.1f} MB), {dt_1:.2f} s wall, 1 thread"},
            "affinity_cores": cores}


def workload_config(args, case, world, fp8):
    """The keys of a result's config that name the workload (both arms)."""
    return {
        "workload": f"{args.workload}: {case.workload.description}",
        "num_seqs": case.num_seqs, "num_q_heads": case.num_q_heads,
        "num_kv_heads": case.num_kv_heads, "head_dim": case.head_dim,
        "block_size": case.block_size, "storage_dtype": gen.DTYPE_NAMES[case.dtype],
        "query_tokens": args.query_tokens,
        "kv_cache": "e4m3 codes + per-kv-head fp32 scales" if fp8 else gen.DTYPE_NAMES[case.dtype],
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
    }


def run_reference(args, rank, world):
    """The oracle as the reference arm: each step decodes a bounded sample."""
    import oracle

    case = gen.make_case(args.workload, n_steps=1, poison=False)
    st = case.steps[0]
    orc = oracle.load()
    cores = len(os.sched_getaffinity(0))
    threads = orc.num_threads(cores)
    budget = 120.0 / max(1, args.steps + args.warmup)
    dt1, _ = _oracle_sample(case, st, 1, orc, threads)
    n = int(max(1, min(case.num_seqs, budget / max(dt1, 1e-6))))
    for _ in range(args.warmup):
        _oracle_sample(case, st, n, orc, threads)
    tot_t, tot_b = 0.0, 0
    for _ in range(args.steps):
        dt, nb = _oracle_sample(case, st, n, orc, threads)
        tot_t += dt
        tot_b += nb
    value = tot_b / tot_t / 1e9
    sample = (f"fp64 C oracle, each step decodes the first {n} of {case.num_seqs} sequences "
              f"of step 0 on {threads} threads")
    return {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * tot_t / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args, case, world, False),
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0
    dist = init_dist(world, "nccl")
    try:
        res = run_ours(args, rank, world, local, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
