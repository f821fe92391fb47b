"""Host-side multi-rank plumbing on CPU (gloo, world size 2): the benchmark
runs one process per GPU with no collective on the data path; ranks only
meet at barriers and take the max of their step times.  These tests run
that plumbing in two CPU processes, and the reference arm under torchrun,
where rank 0 alone works and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    got = d.max(1.5 + rank)           # each rank's step time
    d.barrier()
    out.put((rank, d.world, got))
    d.close()


def test_dist_max_and_barrier_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2, 2.5), (1, 2, 2.5)]   # both ranks see the max


def test_single_process_dist_is_a_no_op():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ["WORLD_SIZE", "RANK", "LOCAL_RANK"] if k in os.environ}
    try:
        d = bench.Dist()
        d.init("gloo")
        assert d.world == 1 and d.rank == 0 and d.pg is None
        d.barrier()
        assert d.max(3.25) == 3.25
        d.close()
    finally:
        os.environ.update(env)


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "linear_6of8_int8_m16", "--gpus", "2", "--steps", "1",
           "--warmup", "1", "--ref-budget", "0.2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=540)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
