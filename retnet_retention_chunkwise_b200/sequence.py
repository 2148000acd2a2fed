"""One sequence cut across ranks (one process per GPU).

Rank r holds the run of tokens [begin_r, end_r) of every (b, h).  The run's
outputs need the state at begin_r, which depends on every earlier token.  The
recurrence between blocks (page "Retentive Networks -- Microsoft ...",
section "Il meccanismo") gives that state from the earlier runs' own sums: with
D_i the state of run i from a zero state and len_i its length,
S_0 = state_in and S_(i+1) = gamma^len_i S_i + D_i.  So each rank

  1. sums its run from a zero state      (retention_chunkwise_state: k, v only),
  2. all-gathers the sums and lengths    (the one exchange: B*H*dk*dv fp32 each),
  3. folds the sums of the ranks before it onto state_in (retention_state_fold),
  4. runs the chunkwise form on its run from that state (retention_chunkwise).

The last rank's state_out is the state after the whole sequence.  Compute runs
in the library's kernels; this module only moves tensors and calls the
collective.  The compute steps are passed in as ``ops`` so the exchange can be
tested on the CPU with other implementations of the same four calls.
"""
from __future__ import annotations

import torch


def split_runs(L: int, chunk: int, rank: int, world: int):
    """[begin, end) tokens of `rank`: whole blocks of `chunk` tokens spread as
    evenly as possible (block counts differ by at most one), the ragged last
    block on the last non-empty rank."""
    if world < 1 or not (0 <= rank < world) or chunk < 1 or L < 0:
        raise ValueError("bad split arguments")
    n_blocks = (L + chunk - 1) // chunk
    base, extra = divmod(n_blocks, world)
    b0 = rank * base + min(rank, extra)
    b1 = b0 + base + (1 if rank < extra else 0)
    return min(b0 * chunk, L), min(b1 * chunk, L)


class CudaOps:
    """The four compute steps on this library's kernels."""

    def __init__(self):
        from retnet_retention_chunkwise_b200 import chunkwise, chunkwise_state, state_fold
        self._chunkwise, self._state, self._fold = chunkwise, chunkwise_state, state_fold

    def run_state(self, k, v, gamma, chunk):
        return self._state(k, v, gamma, chunk)

    def fold(self, parts, lens, gamma, state_in):
        return self._fold(parts, lens, gamma, state_in=state_in)

    def chunkwise(self, q, k, v, gamma, chunk, state_in):
        return self._chunkwise(q, k, v, gamma, chunk, state_in=state_in)


def chunkwise_sequence_sharded(q, k, v, gamma, chunk: int, *, state_in=None, group=None, ops=None, lens=None):
    """This rank's run of a sequence cut across the ranks of `group`.

    q, k, v: the run, [B,H,L_r,d] on this rank's device (runs in rank order make
    the sequence; lengths may differ).  state_in: the state before the whole
    sequence, fp32 [B,H,dk,dv], the same on every rank, or None (zero).
    lens: the run length of every rank, in rank order, when the caller knows
    them (e.g. from split_runs); then they are not exchanged and nothing waits
    on the device between the collective and the fold.  None: they are
    all-gathered with the sums and read back to the host.
    Returns (y_r, state after this run); on the last rank the latter is the
    state after the whole sequence."""
    import torch.distributed as dist
    ops = ops or CudaOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if lens is not None:
        lens = [int(n) for n in lens]
        if len(lens) != world or lens[rank] != q.shape[2] or min(lens) < 0:
            raise ValueError("lens must hold every rank's run length, this rank's equal to q.shape[2]")
    d = ops.run_state(k, v, gamma, chunk)                      # 1. the run's own sum
    # 2. the exchange: rank i's sum lands in rows [i*B, (i+1)*B) of one tensor
    parts = torch.empty((world * d.shape[0],) + tuple(d.shape[1:]), dtype=d.dtype, device=d.device)
    dist.all_gather_into_tensor(parts, d.contiguous(), group=group)
    parts = parts.view((world,) + tuple(d.shape))
    if lens is None:
        n = torch.empty(world, dtype=torch.int64, device=d.device)
        dist.all_gather_into_tensor(n, torch.tensor([q.shape[2]], dtype=torch.int64, device=d.device), group=group)
        lens = n.tolist()
    s_r = ops.fold(parts[:rank], lens[:rank], gamma, state_in)  # 3. the state at begin_r
    return ops.chunkwise(q, k, v, gamma, chunk, s_r)           # 4. the run itself
