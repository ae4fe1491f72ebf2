"""bench.py's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1.

The N > 1 path of bench.py (one process per GPU, max over ranks of the
timed region, rank 0 alone prints; the reference arm runs on rank 0 only)
is covered here with the gloo backend and no GPU.
"""
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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, local = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    # the timed region's max over ranks: every rank gets the slowest time
    v = bench.max_over_ranks(0.25 + rank, w)
    bench.barrier(w)
    # weak scaling: whole-job value = units of all ranks / the max time
    value = w * 100.0 / v
    results.put((rank, v, value))
    dist.destroy_process_group()


def test_max_over_ranks_and_barrier_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(2))
    assert [g[1] for g in got] == [1.25, 1.25]       # max over ranks
    assert [g[2] for g in got] == [160.0, 160.0]     # 2 ranks x 100 units / 1.25 s


def test_reference_arm_under_torchrun_prints_once_on_rank_0():
    """`--impl reference` launched as a two-GPU run is (torchrun, two ranks): rank 0 times the
    CPU oracle and prints one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-seconds", "2"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
