"""The benchmark's multi-process path (one process per GPU under torchrun) on the CPU: two gloo
ranks exercise the process-group setup, the timing barrier and the max-over-ranks reduction, and
the reference arm's rank gating (rank 0 alone runs and prints)."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, local = bench.dist_init(world, backend="gloo")
    assert (w, r, local) == (world, rank, rank)
    bench.barrier(w)
    # each rank's "device time" differs; every rank must see the maximum
    got = bench.max_over_ranks(1.5 + rank, w)
    out.put((rank, got))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_barrier_and_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 2.5, 1: 2.5}


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_reference_arm_rank_gating():
    """Under torchrun only rank 0 runs the reference arm (the float64 oracle) and prints its one
    JSON line; the other ranks exit 0 without work."""
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r1 = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                         "--warmup", "0", "--cpu-rows", "8"], cwd=ROOT, env=env, capture_output=True, text=True,
                        timeout=300)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    env.update(RANK="0", LOCAL_RANK="0")
    r0 = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
                         "--warmup", "0", "--cpu-rows", "8"], cwd=ROOT, env=env, capture_output=True, text=True,
                        timeout=300)
    assert r0.returncode == 0, r0.stderr[-2000:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["rows_per_s"] > 0 and line["cpu_baseline"]["extrapolated_full_config_s"] > 0
