"""The multi-GPU host logic (one process per GPU, independent replicas,
timings reduced as the maximum over ranks) on world_size-2 gloo ranks, CPU only."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    from learned_product_hash_proj_b200 import dist
    r, local, w = dist.init("gloo", timeout_s=60)
    mx = dist.reduce_max([1.0 + r, 10.0 - r])
    sm = dist.reduce_sum([r + 1])
    tput = dist.throughput([1000.0], [0.5 + r])          # slowest rank takes 1.5 s
    seeds = dist.reduce_sum([dist.replica_seed(0, r) * 10 ** (3 * r)])
    dist.barrier()
    dist.finalize()
    q.put((r, local, w, mx, sm, tput, seeds))


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, local, world, mx, sm, tput, seeds) in enumerate(out):
        assert (rank, local, world) == (r, r, 2)
        assert mx == [2.0, 10.0]
        assert sm == [3.0]
        assert tput == pytest.approx(2000.0 / 1.5)
        assert seeds == [0 + 1 * 1000]          # replicas draw distinct seeds (0 and 1)


def test_single_process_defaults():
    from learned_product_hash_proj_b200 import dist
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        os.environ.pop(k, None)
    assert dist.env_rank() == (0, 0, 1)
    assert dist.reduce_max([3.0]) == [3.0]
    assert dist.throughput([10.0], [2.0]) == 5.0
