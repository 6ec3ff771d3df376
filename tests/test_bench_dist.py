"""The N > 1 timing path of bench.py on CPU: two gloo ranks, one process each.

Each rank reports a different step time; both must see the maximum, and the
whole-job rate must count every rank's units over that slowest time (weak
scaling, replicas with no data exchange).  The reference arm's non-zero
ranks exit without work."""
import importlib.util
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    bench = _load_bench()
    d = bench.Dist(backend="gloo", device="cpu")
    d.init(torch)
    d.barrier(torch)
    ms = d.max(torch, 2.0 + rank)        # rank r "took" 2 + r ms
    rate = bench.whole_job_rate(1000.0, ms, d.world)
    d.barrier(torch)
    d.close()
    out.put((rank, d.world, ms, rate))


def test_max_over_ranks_and_whole_job_rate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, world, ms, rate in res:
        assert world == 2
        assert ms == pytest.approx(3.0)                      # the slower rank's time
        assert rate == pytest.approx(2 * 1000.0 / 3.0e-3)   # both ranks' units / max time


def test_single_process_needs_no_group():
    bench = _load_bench()
    d = bench.Dist()
    if d.world != 1:
        pytest.skip("launched under a multi-process launcher")
    assert d.max(None, 1.5) == 1.5
    assert bench.whole_job_rate(10.0, 2.0, 1) == pytest.approx(5000.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
