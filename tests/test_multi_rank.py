"""The bench's multi-rank logic on CPU with the gloo backend (world size 2): the
max-over-ranks time, the barrier, replica seeds, and the balanced matrix partition used for
strong scaling. No GPU and no collective on the data path are involved."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from calibration_free_weight_hqq_b200 import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        local_ms = 10.0 * (rank + 1)
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        dist.barrier()
        q.put((rank, m, bench.replica_seed_offset(rank)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [m for _, m, _ in got] == [20.0, 20.0]          # every rank sees the max
    assert len({off for _, _, off in got}) == world         # distinct replica seeds


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_partition_covers_every_matrix_once_and_balances(world):
    sizes = [m.numel for m in workloads.llama7b_model_4b().matrices]
    parts = bench.partition_by_weight(sizes, world)
    flat = sorted(i for p in parts for i in p)
    assert flat == list(range(len(sizes)))
    loads = [sum(sizes[i] for i in p) for p in parts]
    assert max(loads) - min(loads) <= max(sizes)            # greedy bound
    assert max(loads) <= sum(sizes) / world * 1.02
