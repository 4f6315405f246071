"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

With N GPUs every rank runs its own replica of the workload (no data
exchange); the only collectives are the max of the device time and the sum
of processed bytes over ranks.  These run here on gloo.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from paged_kv_cache_458_b200 import gen

    r, w, local = bench.dist_env()
    d = bench.init_dist(w, "gloo")
    mx = bench.max_over_ranks(10.0 + r, d)
    sm = bench.sum_over_ranks(1.5 * (r + 1), d)
    seed = gen.SEED_BASE + gen.WORKLOADS["tiny"].number + 1000 * r
    case = gen.make_case("tiny", n_steps=0, seed=seed)
    d.barrier()
    d.destroy_process_group()
    q.put((r, w, mx, sm, int(case.q.astype("int64").sum())))


def test_two_ranks_reduce_timing_and_use_distinct_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == 11.0 for r in res), "max over ranks"
    assert all(r[3] == 1.5 + 3.0 for r in res), "sum over ranks"
    assert res[0][4] != res[1][4], "each rank runs its own seeded replica"


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0"]) == 0
    assert capsys.readouterr().out == ""
