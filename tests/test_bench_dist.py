"""The multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

`bench.py --gpus N` runs one process per GPU under torchrun. Every rank times its own requests
(weak scaling, no data-path collective), and the reported time is the max over ranks. The pieces
that do this are exercised here with a world-size-2 gloo process group: the rank environment, the
disjoint request ranges, the max over ranks, and the barrier. The reference arm's ranks other than
0 exit without work and print nothing.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench

    r, w, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        batch = 70
        lo = bench.request_offset(r, batch)
        # a rank-dependent "timed region": the reduction must return the slowest rank's time on every rank
        ms = 10.0 + 5.0 * r
        worst = bench.reduce_max(ms)
        bench.barrier(None)
        out.put((r, w, local, lo, lo + batch, worst))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks_disjoint_requests_and_max_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=10) for _ in range(2))
    (r0, w0, l0, a0, b0, m0), (r1, w1, l1, a1, b1, m1) = res
    assert (r0, w0, l0) == (0, 2, 0) and (r1, w1, l1) == (1, 2, 1)
    assert b0 <= a1, "the ranks' request ranges overlap"
    assert (a0, b0, a1, b1) == (0, 70, 70, 140)
    assert m0 == m1 == 15.0, "the reported time is the max over ranks on every rank"


def test_single_process_reduction_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max(3.25) == 3.25
    bench.barrier(None)  # no process group: a no-op


def test_reference_arm_other_ranks_exit_without_output():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                           "--steps", "1", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=120)
    assert proc.returncode == 0, proc.stderr
    assert proc.stdout.strip() == ""


def test_step_traffic_only_for_the_profiled_step():
    """The bench line carries the committed DRAM capture only for the configuration it was taken
    on (and only while the decode source is the captured one)."""
    import argparse

    import bench

    base = dict(workload=bench.DEFAULT_WORKLOAD, batch=0, scale_dtype="f32", fit_rounds=0)
    assert bench.step_traffic(argparse.Namespace(**base)) == bench.profiled_traffic()
    for change in (dict(batch=32), dict(scale_dtype="bf16"), dict(fit_rounds=1), dict(workload="layer48_b8_4bit")):
        assert bench.step_traffic(argparse.Namespace(**{**base, **change})) is None, change
