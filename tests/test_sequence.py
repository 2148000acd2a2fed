"""A sequence cut across ranks (no GPU): the run split, and the exchange of
retnet_retention_chunkwise_b200.sequence run as gloo ranks on the CPU with the
four compute steps taken from the oracle."""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from retnet_retention_chunkwise_b200 import sequence


@pytest.mark.parametrize("L,chunk,world", [(1000, 64, 2), (1000, 64, 3), (64, 64, 4), (0, 16, 2), (4097, 128, 8)])
def test_split_runs_partition(L, chunk, world):
    runs = [sequence.split_runs(L, chunk, r, world) for r in range(world)]
    assert runs[0][0] == 0 and runs[-1][1] == L
    for (b0, e0), (b1, _) in zip(runs, runs[1:]):
        assert e0 == b1
    blocks = [(e - b + chunk - 1) // chunk for b, e in runs]
    assert max(blocks) - min(blocks) <= 1
    for b, e in runs[:-1]:
        assert b % chunk == 0 and (e == L or e % chunk == 0)


class OracleOps:
    """The four steps in fp64 on the CPU: the oracle for the run sums and the
    runs, the fold written out from the recurrence."""

    def run_state(self, k, v, gamma, chunk):
        return torch.from_numpy(oracle.recurrent(k, k, v, gamma)[1])

    def fold(self, parts, lens, gamma, state_in):
        g = np.asarray(gamma, dtype=np.float64)[None, :, None, None]
        s = np.zeros(parts.shape[1:]) if state_in is None else state_in.numpy().copy()
        for i, n in enumerate(lens):
            s = g ** n * s + parts[i].numpy()
        return torch.from_numpy(s)

    def chunkwise(self, q, k, v, gamma, chunk, state_in):
        y, s = oracle.chunkwise(q, k, v, gamma, chunk, None if state_in is None else state_in.numpy())
        return torch.from_numpy(y), torch.from_numpy(s)


def _inputs(B, H, L, dk, dv, seed):
    rng = np.random.default_rng(seed)
    q, k = (torch.from_numpy(rng.standard_normal((B, H, L, dk)) / np.sqrt(dk)) for _ in range(2))
    v = torch.from_numpy(rng.standard_normal((B, H, L, dv)))
    s_in = torch.from_numpy(rng.standard_normal((B, H, dk, dv)) * 0.5)
    return q, k, v, s_in


def _worker(rank, world, port, out_dir, L, chunk, uneven, known_lens=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, s_in = _inputs(1, 2, L, 3, 4, 5)
        gamma = np.array([0.9, 0.6])
        if uneven:  # runs of arbitrary lengths, not block-aligned
            cuts = [0, 5, 6, 17, L][: world] + [L]
        else:
            cuts = [sequence.split_runs(L, chunk, r, world)[0] for r in range(world)] + [L]
        b, e = cuts[rank], cuts[rank + 1]
        # the caller's own run lengths (no length exchange), or None (exchanged)
        lens = [cuts[r + 1] - cuts[r] for r in range(world)] if known_lens else None
        run = lambda t: t[:, :, b:e].contiguous()  # noqa: E731
        y, s = sequence.chunkwise_sequence_sharded(run(q), run(k), run(v), gamma, chunk, state_in=s_in,
                                                   ops=OracleOps(), lens=lens)
        torch.save({"y": y, "s": s, "b": b, "e": e}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,L,chunk,uneven,known_lens", [(2, 40, 8, False, False), (3, 37, 4, False, False),
                                                             (3, 23, 4, True, False), (4, 50, 4, True, False),
                                                             (2, 40, 8, False, True), (3, 23, 4, True, True)])
def test_sequence_sharded_exchange_gloo(world, L, chunk, uneven, known_lens):
    with tempfile.TemporaryDirectory() as out_dir:
        mp.start_processes(_worker, args=(world, _free_port(), out_dir, L, chunk, uneven, known_lens), nprocs=world,
                           join=True, start_method="spawn")
        res = [torch.load(os.path.join(out_dir, f"r{r}.pt")) for r in range(world)]
    q, k, v, s_in = _inputs(1, 2, L, 3, 4, 5)
    y_ref, s_ref = oracle.recurrent(q, k, v, np.array([0.9, 0.6]), s_in.numpy())
    assert [r["b"] for r in res] == [0] + [r["e"] for r in res[:-1]] and res[-1]["e"] == L
    y = torch.cat([r["y"] for r in res], dim=2).numpy()
    assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(res[-1]["s"].numpy(), s_ref, rtol=1e-12, atol=1e-12)
