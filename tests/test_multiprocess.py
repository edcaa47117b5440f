"""The N > 1 path on the CPU: two ranks over gloo.  The layer shards into independent replicas, so
the only collectives are the bench's barrier and the max-over-ranks of its timings; these tests run
them, and the reference arm under torchrun (rank 0 alone works and prints), without a GPU."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    bench.init_dist(world, "gloo")
    bench.barrier(world)
    # each rank reports its own time; every rank must see the slowest
    got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
    bench.barrier(world)
    q.put((rank, got, bench.dist_env()))
    dist.destroy_process_group()


def test_bench_collectives_over_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2.5 for r in res)  # max over ranks
    assert res[1][2] == (1, 2, 1)  # RANK, WORLD_SIZE, LOCAL_RANK as torchrun sets them


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference` launched the way the driver launches N > 1: rank 0 alone times the
    oracle and prints one JSON line; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--ref-sample-tokens", "128"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    ln = lines[0]
    assert ln["impl"] == "reference" and ln["n_gpus"] == 2 and ln["value"] > 0
    assert ln["cpu_baseline"]["kind"] == "oracle" and ln["e2e"]["h2d_bytes_per_step"] == 0
