"""The multi-rank path of bench.py on CPU: world size 2 over gloo (127.0.0.1).

Each rank decodes its own batch (weak scaling, no collective on the data
path): the ranks' workloads are independent draws, the step time is the
slowest rank's (one MAX all-reduce), the job's throughput counts every
rank's batch, and the reference arm runs on rank 0 alone.
"""

import contextlib
import io
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with contextlib.closing(socket.socket(socket.AF_INET, socket.SOCK_STREAM)) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import torch

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        small = synth.get_config("c1").scaled(ctx_len=1024, K_b=8, k=128)
        c, qb, K, V, lab = bench.workload(small, rank)
        # independent batches: every rank draws its own K (checksums gathered)
        mine = torch.tensor([float(np.asarray(K, dtype=np.float64).sum()), float(c.seed)], dtype=torch.float64)
        got = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got, mine)
        # the slowest rank sets each timing
        times = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], world)
        value = bench.job_tokens_per_s(world, c.batch, times[0])
        # the reference arm: rank 0 prints one line, the others return silently
        out = io.StringIO()

        class Args:
            steps, warmup, cpu_seconds, gpus = 1, 0, 0.2, world

        with contextlib.redirect_stdout(out):
            bench.run_reference(Args, small)
        q.put((rank, [g.tolist() for g in got], times, value, out.getvalue()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_over_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, got, times, value, printed = q.get(timeout=300)
        res[rank] = (got, times, value, printed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got0 = res[0][0]
    assert got0 == res[1][0], "all_gather disagrees between ranks"
    assert got0[0][0] != got0[1][0] and got0[0][1] != got0[1][1], "ranks drew the same workload"
    for r in range(world):
        assert res[r][1] == [2.0, 10.0, 3.0], "timings are not the max over ranks"
        assert abs(res[r][2] - 2 * 1 / (2.0 / 1e3)) < 1e-6, "job throughput does not count every rank's batch"
    lines = [ln for ln in res[0][3].splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and '"impl": "reference"' in lines[0]
    assert res[1][3] == "", "rank 1 printed in the reference arm"
