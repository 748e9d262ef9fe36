"""The N > 1 path of bench.py on CPU ranks (gloo, world size 2): the reduction that reports the
slowest rank's time, the barrier, the per-rank inputs, and the reference arm under torchrun
(rank 0 alone works and prints the one JSON line; the other rank exits 0 without output)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import hga_inputs as HI
    import torch.distributed as dist
    w_, r_, _ = bench.dist_setup()
    assert (w_, r_) == (world, rank) and dist.get_backend() == "gloo"
    # slowest rank's time
    m = bench.all_max(1.0 + rank, world, "cpu")
    bench.barrier(world)
    # every rank draws its own layer (seed + rank): the inputs differ between ranks
    w = HI.WORKLOADS["tiny_f32"]
    x = HI.make_inputs(w, 7 + rank)
    gathered = [torch.zeros(4) for _ in range(world)]
    dist.all_gather(gathered, x["q"].flatten()[:4].contiguous())
    distinct = not torch.equal(gathered[0], gathered[1])
    dist.destroy_process_group()
    q.put((rank, m, distinct))


def test_max_over_ranks_barrier_and_rank_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    out = sorted(q.get(timeout=5) for _ in range(2))
    assert [o[1] for o in out] == [2.0, 2.0]          # both ranks report the slower rank's value
    assert all(o[2] for o in out)


@pytest.mark.timeout(300)
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny_f32"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=280)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
