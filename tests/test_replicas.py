"""Multi-rank host logic (no GPU): pair sharding and the whole-job reductions,
run as two gloo ranks on the CPU."""
import os
import socket
import tempfile

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from retnet_retention_chunkwise_b200 import replicas


@pytest.mark.parametrize("n,world", [(32, 1), (32, 2), (7, 3), (1024, 8), (3, 8), (0, 4)])
def test_shard_pairs_partition(n, world):
    seen = []
    sizes = []
    for r in range(world):
        b, e = replicas.shard_pairs(n, r, world)
        assert 0 <= b <= e <= n
        seen.extend(range(b, e))
        sizes.append(e - b)
    assert seen == list(range(n))
    assert max(sizes) - min(sizes) <= 1


def test_shard_pairs_rejects_bad_rank():
    with pytest.raises(ValueError):
        replicas.shard_pairs(4, 2, 2)


def test_single_process_reductions_are_identity():
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.sum_over_ranks(2.0) == 2.0
    v, tot, t = replicas.job_throughput(10.0, 2.0)
    assert (v, tot, t) == (5.0, 10.0, 2.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # each rank processes its own pairs; rank r takes (r + 1) * 0.1 s
        b, e = replicas.shard_pairs(10, rank, world)
        units = float(e - b)
        rate, total, t = replicas.job_throughput(units, 0.1 * (rank + 1))
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{rate} {total} {t}")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_job_throughput():
    out = tempfile.mkdtemp()
    mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    for r in range(2):
        rate, total, t = (float(x) for x in open(os.path.join(out, f"r{r}.txt")).read().split())
        assert total == 10.0 and abs(t - 0.2) < 1e-12 and abs(rate - 50.0) < 1e-9
