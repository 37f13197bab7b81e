"""The multi-rank bench path on CPU: world size 2 over gloo.  Each rank
reports its own step time and executed FLOPs; the job's throughput is the
sum of FLOPs over the slowest rank's time."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup("gloo")
    assert (w, r) == (world, rank)
    local_ms = [10.0, 14.0][rank]
    local_flops = [3e12, 5e12][rank]
    value, ms, flops = bench.job_throughput(local_ms, local_flops, w)
    bench.barrier(w)
    q.put((rank, value, ms, flops))
    dist.destroy_process_group()


def test_job_throughput_two_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, ms, flops in res:
        assert ms == 14.0                 # the slowest rank's time
        assert flops == 8e12              # every rank's work
        assert value == pytest.approx(8e12 / 14e-3 / 1e12)


def test_reference_arm_two_ranks_only_rank0_prints(tmp_path):
    """`bench.py --impl reference` under torchrun: rank 0 prints one JSON line,
    the other rank exits 0 without work (no GPU needed)."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--workload", "tiny-f32", "--steps", "2", "--warmup", "1",
           "--cpu-seconds", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    import json
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["e2e"]["h2d_bytes_per_step"] == 0
