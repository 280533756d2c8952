"""The multi-rank plumbing of bench.py on CPU: two gloo ranks (127.0.0.1) take the barrier,
agree on the maximum of their timings, and the whole-job figure divides all ranks' layers
by the slowest rank's time; the reference arm prints from rank 0 only."""
import importlib.util
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _rank_main(rank, port, q):
    import torch.distributed as dist
    b = _bench()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=2)
    try:
        b.barrier(2)
        ms = [3.0, 5.0][rank]  # rank 1 is the slow one
        top = b.max_over_ranks(2, ms, device="cpu")
        q.put((rank, top, b.us_per_layer(top, steps=4, layers_per_step=24, ws=2)))
        b.barrier(2)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_agree_on_the_max():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[1] for g in got] == [5.0, 5.0]
    # 2 ranks x 4 steps x 24 layers in 5 ms
    assert got[0][2] == pytest.approx(5.0e3 / (4 * 24 * 2))


def test_reference_arm_prints_from_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_replica_division():
    b = _bench()
    assert b.us_per_layer(10.0, 2, 5, 1) == pytest.approx(1000.0)
    assert b.us_per_layer(10.0, 2, 5, 4) == pytest.approx(250.0)
    assert json.loads(json.dumps({"v": b.us_per_layer(1.0, 1, 1, 1)}))["v"] == 1000.0
