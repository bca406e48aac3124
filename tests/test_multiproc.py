"""The N>1 benchmark path on CPU with world_size 2 over gloo.

Each rank runs its own replica (no data-path exchange); the only collective
is the max-over-ranks of the timing, and the whole-job value is all ranks'
bytes over the slowest rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        assert bench.dist_env() == (rank, world, rank)
        slowest = bench.reduce_max(10.0 + 5.0 * rank)
        bench.barrier()
        value = bench.weak_scaling_value(1_000_000_000, world, 4, slowest)
        # the reference arm runs on rank 0 only; other ranks return at once
        rc = None
        if rank == 1:
            rc = bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"])
        q.put((rank, slowest, value, rc))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value, rc in got:
        assert slowest == 15.0                          # max over ranks
        assert value == pytest.approx(2 * 4 * 1.0 / 15e-3)  # 2 ranks x 4 steps x 1 GB / 15 ms
    assert got[1][3] == 0


def test_gpus_flag_launches_one_process_per_rank():
    # `bench.py --gpus 2` outside a launcher starts two ranks itself; the
    # reference arm (host only) runs on rank 0 and reports both ranks
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--impl", "reference",
                        "--workload", "tiny", "--steps", "3", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
