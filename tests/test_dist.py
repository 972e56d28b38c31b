"""Multi-rank host logic of the benchmark, on CPU with the gloo backend.

The (sequence, head) units of the method are independent, so a run on N GPUs
is N replicas with no data-path collective; the only cross-rank step is the
max over ranks of the step time.  Two gloo ranks check that reduction, the
whole-job throughput and the barrier."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    try:
        ms_local = 2.0 if rank == 0 else 3.0  # rank 1 is the slow one
        value, ms = bench.aggregate(16384, ms_local, world)
        bench.barrier(world)
        q.put((rank, value, ms, bench.max_over_ranks(float(rank), world)))
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, ms, mx in res:
        assert ms == 3.0                                # max over ranks
        assert abs(value - 16384 * 2 / 3.0e-3) < 1e-6   # all ranks' tokens / slowest time
        assert mx == 1.0


def test_single_rank_aggregation_is_local():
    import bench
    value, ms = bench.aggregate(1000, 4.0, 1)
    assert ms == 4.0 and abs(value - 250000.0) < 1e-9


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference --gpus 2` launched the way the multi-GPU runs
    are (torchrun, one process per rank, gloo here): rank 0 alone times the
    oracle and prints one JSON line, the other rank exits 0 without work."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--ref-budget-s", "2"]
    r = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
