"""Host logic of the multi-GPU benchmark path, run as world-size-2 gloo ranks
on the CPU: the slowest rank sets the job's step time, the job throughput
counts every rank's replica, the barrier releases all ranks together, and
the reference arm prints from rank 0 only."""
import io
import os
import socket
import sys
import contextlib

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    dev = torch.device("cpu")
    local_ms = [2.0, 3.5][rank]
    bench._barrier(dist, dev)
    job_ms = bench._max_over_ranks(dist, local_ms, dev)
    value = bench.job_throughput(world, 1e12, job_ms)
    bench._barrier(dist, dev)
    q.put((rank, job_ms, value))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, job_ms, value in res:
        assert job_ms == 3.5                       # max over ranks, on every rank
        assert abs(value - 2 * 1e12 / 3.5e-3 / 1e12) < 1e-9   # both replicas counted


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"steps": 3, "warmup": 3})()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""


def _sharded_worker(rank, world, port, method, q):
    try:
        sys.path.insert(0, ROOT)
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        import bench
        import oracle
        from test_dist_gloo import OracleOps
        args = type("A", (), {"steps": 2, "warmup": 3, "workload": "tiny_ring_f32",
                              "method": method, "gpus": world})()
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            line = bench.run_sharded(args, ops=OracleOps(oracle), device=torch.device("cpu"))
        q.put((rank, line, buf.getvalue()))
        dist.destroy_process_group()
    except Exception:
        import traceback
        q.put((rank, "crash", traceback.format_exc()))


@pytest.mark.parametrize("method,world", [("ring", 2), ("ulysses", 2), ("usp", 4)])
def test_sharded_mode_host_logic(method, world):
    """bench.py --mode sharded on gloo ranks (kernels answered by the oracle):
    the sequence is split over the ranks, only rank 0 prints, the value is
    the whole sequence's FLOPs over the slowest rank, and every rank's
    exchange bytes are reported."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    from context_attention_dits_cp_b200 import workloads as wl
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, method, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
    assert all(r[1] != "crash" for r in res), res
    line, printed = res[0][1], res[0][2]
    assert all(r[1] is None and r[2] == "" for r in res[1:])
    assert json.loads(printed) == line
    w = wl.workload("tiny_ring_f32")
    assert line["scaling"] == "strong" and line["n_gpus"] == world
    assert abs(line["value"] - w.flops / (line["ms_per_step"] * 1e-3) / 1e12) < 1e-9 * line["value"]
    assert sum(line["config"]["shard_lengths"]) == w.S
    plans = [bench.sharded_plan(w, world, r, method) for r in range(world)]
    assert [p["tokens"][1] - p["tokens"][0] for p in plans] == line["config"]["shard_lengths"]
    assert line["exchange_bytes_per_rank"] == [{"send": p["send"], "recv": p["recv"]}
                                               for p in plans]
    # what the ranks send is what they receive
    assert sum(p["send"] for p in plans) <= sum(p["recv"] for p in plans) * world
    if method == "ulysses":
        assert sum(p["send"] for p in plans) == sum(p["recv"] for p in plans)
