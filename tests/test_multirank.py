"""The N > 1 host logic of bench.py on CPU ranks (gloo, world size 2).

Rows of a batch are independent, so each rank runs its own batch against its
own weight replica with no collective on the data path.  What needs checking
is the job-level arithmetic: units are summed over ranks and the job time is
the maximum over ranks, and the reference arm prints only on rank 0.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench
    units, ms = bench.aggregate(1000.0 * (rank + 1), 10.0 + 5.0 * rank, world, "cpu")
    mx = bench.max_over_ranks(3.0 - rank, world, "cpu")
    bench.barrier(world)
    q.put((rank, units, ms, mx))
    dist.destroy_process_group()


def test_aggregate_sums_units_and_takes_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, units, ms, mx in out:
        assert units == 3000.0        # 1000 + 2000
        assert ms == 15.0             # max(10, 15)
        assert mx == 3.0              # max(3, 2)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "2", "--warmup", "0", "--workload", "tiny"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        assert len(lines) == 1
        rec = json.loads(lines[0])
        assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
        assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
    else:
        assert lines == []
