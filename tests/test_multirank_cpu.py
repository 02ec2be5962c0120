"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, as torchrun
would start them for `bench.py --gpus 2` (every rank times an independent
layer; the job time is the slowest rank's; no collective on the data path)."""

import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank                    # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, dist)
        first = bench.max_over_ranks(-rank, dist)       # collectives stay in step across calls
        mine = bench.head_partition(40, rank, world)   # --partition heads: this rank's heads of one call
        parts = [None] * world
        dist.all_gather_object(parts, mine)
        out.put((rank, job_ms, first, bench.rank_seed(2000, rank),
                 bench.aggregate_tflops(2.0e12, world, job_ms), parts))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_is_max_over_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]
    assert [r[2] for r in res] == [0.0, 0.0]
    assert res[0][3] != res[1][3]                       # independent inputs per rank
    # whole-job throughput: both ranks' work over the slowest rank's time
    assert res[0][4] == pytest.approx(2 * 2.0e12 / 15e-3 / 1e12)
    # --partition heads: the ranks' head lists cover the 40 heads of the call
    # exactly once, and every rank sees the same partition
    parts = res[0][5]
    assert parts == res[1][5]
    assert sorted(h for p in parts for h in p) == list(range(40))
    assert all(len(p) == 20 for p in parts)


@pytest.mark.parametrize("heads,world", [(40, 3), (40, 8), (12, 5), (3, 4)])
def test_head_partition_covers_every_head_once(heads, world):
    sys.path.insert(0, ROOT)
    import bench

    parts = [bench.head_partition(heads, r, world) for r in range(world)]
    assert sorted(h for p in parts for h in p) == list(range(heads))
    assert max(map(len, parts)) - min(map(len, parts)) <= 1


def test_single_process_and_reference_arm_off_rank_zero():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5) == 3.5             # no process group: identity
    assert bench.run_reference(None, 1, 2) is None      # ranks > 0 of the reference arm do no work
