"""The multi-process path of bench.py on the CPU (world size 2, gloo): one
process per GPU under torchrun, each timing its own replica (the layer has
no exchange step), the job's time the slowest rank's, one JSON line from
rank 0."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        got = bench.max_over_ranks(1.5 + rank, world, "cpu")
        dist.barrier()
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gives_every_rank_the_slowest():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_process_needs_no_collective():
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25


def _run(args, env=None, timeout=600):
    return subprocess.run([sys.executable, *args], cwd=ROOT, capture_output=True, text=True, timeout=timeout,
                          env={**os.environ, **(env or {})})


def test_reference_arm_under_torchrun_prints_one_line_from_rank_0():
    port = _free_port()
    r = _run(["-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
              "--master-port", str(port), "bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1",
              "--warmup", "0"], env={"OMP_NUM_THREADS": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def test_several_gpus_without_torchrun_is_refused():
    r = _run(["bench.py", "--gpus", "2"], env={"WORLD_SIZE": "1", "RANK": "0"}, timeout=300)
    assert r.returncode == 2
    assert "torchrun" in json.loads(r.stdout.strip().splitlines()[-1])["error"]
