"""GPU parity of the state-only call, the state fold and a sequence cut into
runs (one GPU; the runs emulate ranks, and a one-rank NCCL group drives the
real exchange), against the fp64 oracle.

Metric: max |gpu - oracle| / max |oracle|, over each tensor and over each of
its (b, h) slices (tests/parity.py); 1e-4 for fp32 inputs, 2e-2 for bf16
inputs."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import retnet_retention_chunkwise_b200 as ret
from retnet_retention_chunkwise_b200 import inputs, sequence
from tests.parity import rel

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}




@pytest.mark.parametrize("dt,B,H,L,dk,dv,C", [
    (torch.bfloat16, 1, 2, 8192, 256, 512, 128),   # many segments, four dv slices
    (torch.bfloat16, 2, 3, 1000, 128, 256, 64),    # ragged tail
    (torch.bfloat16, 1, 2, 777, 64, 128, 256),     # 256-row blocks
    (torch.bfloat16, 1, 1, 100, 128, 128, 128),    # one block
    (torch.bfloat16, 1, 2, 500, 64, 256, 64),      # dk = 64, two dv slices per CTA
    (torch.float32, 1, 2, 300, 64, 48, 32),
])
def test_chunkwise_state_matches_state_out(dt, B, H, L, dk, dv, C):
    q, k, v = inputs.qkv(B, H, L, dk, dv, dt, seed=L + dk)
    gam = inputs.multiscale_gammas(H)
    s_in = inputs.state(B, H, dk, dv, seed=4, scale=0.5)
    _, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    kd, vd, sd = k.cuda(), v.cuda(), s_in.cuda()
    got = ret.chunkwise_state(kd, vd, gam, C, state_in=sd)
    assert rel(got, s_ref) <= TOL[dt]
    # from zero
    _, z_ref = oracle.recurrent(q, k, v, gam)
    assert rel(ret.chunkwise_state(kd, vd, gam, C), z_ref) <= TOL[dt]
    # in place over state_in
    ret.chunkwise_state(kd, vd, gam, C, state_in=sd, out=sd)
    assert torch.equal(sd, got)
    assert ret.device_status() == 0


def test_chunkwise_state_small_workspace_and_empty():
    B, H, L, dk, dv, C = 1, 2, 4096, 128, 128, 128
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=3)
    gam = inputs.multiscale_gammas(H)
    _, s_ref = oracle.recurrent(q, k, v, gam)
    kd, vd = k.cuda(), v.cuda()
    full = ret.chunkwise_state(kd, vd, gam, C)
    two = torch.empty(2 * B * H * dk * dv, dtype=torch.float32, device="cuda")  # room for one segment
    one_seg = ret.chunkwise_state(kd, vd, gam, C, workspace=two)
    assert rel(full, s_ref) <= 2e-2 and rel(one_seg, s_ref) <= 2e-2
    s_in = inputs.state(B, H, dk, dv, seed=5).cuda()
    e = torch.empty((B, H, 0, dk), dtype=torch.bfloat16, device="cuda")
    ev = torch.empty((B, H, 0, dv), dtype=torch.bfloat16, device="cuda")
    assert torch.equal(ret.chunkwise_state(e, ev, gam, C, state_in=s_in), s_in)
    assert torch.count_nonzero(ret.chunkwise_state(e, ev, gam, C)) == 0
    assert ret.device_status() == 0


def test_state_fold_against_runs():
    # the state after three runs, folded from the runs' own sums, against the
    # oracle's state after the whole sequence
    B, H, dk, dv = 2, 3, 64, 128
    lens = [70, 1, 130]
    q, k, v = inputs.qkv(B, H, sum(lens), dk, dv, torch.float32, seed=8)
    gam = np.array([0.0, 0.9, 1.0])  # gamma 0 and 1 included
    s_in = inputs.state(B, H, dk, dv, seed=6, scale=0.5)
    cuts = np.cumsum([0] + lens)
    parts = np.stack([oracle.recurrent(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], gam)[1]
                      for a, b in zip(cuts, cuts[1:])])
    _, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    pd = torch.from_numpy(parts).float().cuda()
    got = ret.state_fold(pd, lens, torch.from_numpy(gam).float(), state_in=s_in.cuda())
    assert rel(got, s_ref) <= 1e-4
    # no parts: the state passes through; in place over state_in
    sd = s_in.cuda()
    assert torch.equal(ret.state_fold(pd[:0], [], torch.from_numpy(gam).float(), state_in=sd), sd)
    ret.state_fold(pd, lens, torch.from_numpy(gam).float(), state_in=sd, out=sd)
    assert torch.equal(sd, got)
    assert ret.device_status() == 0


@pytest.mark.parametrize("dt,world,L,dk,dv,C", [
    (torch.bfloat16, 4, 3000, 256, 512, 128),
    (torch.bfloat16, 3, 1000, 128, 256, 64),
    (torch.float32, 3, 200, 64, 64, 32),
])
def test_sequence_cut_into_runs(dt, world, L, dk, dv, C):
    # each "rank" r: its run's sum, the fold of the sums before it, its run
    B, H = 1, 2
    q, k, v = inputs.qkv(B, H, L, dk, dv, dt, seed=world + L)
    gam = inputs.multiscale_gammas(H)
    s_in = inputs.state(B, H, dk, dv, seed=7, scale=0.5)
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    qd, kd, vd, sd = q.cuda(), k.cuda(), v.cuda(), s_in.cuda()
    runs = [sequence.split_runs(L, C, r, world) for r in range(world)]
    sub = lambda t, b, e: t[:, :, b:e].contiguous()  # noqa: E731
    sums = torch.stack([ret.chunkwise_state(sub(kd, b, e), sub(vd, b, e), gam, C) for b, e in runs])
    ys, s_last = [], None
    for r, (b, e) in enumerate(runs):
        s_r = ret.state_fold(sums[:r], [e1 - b1 for b1, e1 in runs[:r]], gam, state_in=sd)
        y_r, s_last = ret.chunkwise(sub(qd, b, e), sub(kd, b, e), sub(vd, b, e), gam, C, state_in=s_r)
        ys.append(y_r)
    assert rel(torch.cat(ys, dim=2), y_ref) <= TOL[dt]
    assert rel(s_last, s_ref) <= TOL[dt]
    assert ret.device_status() == 0


def test_sequence_sharded_one_rank_nccl():
    # the module's own path, NCCL collectives included, on a one-rank group
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        B, H, L, dk, dv, C = 1, 2, 700, 128, 256, 128
        q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=12)
        gam = inputs.multiscale_gammas(H)
        s_in = inputs.state(B, H, dk, dv, seed=9, scale=0.5)
        y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
        y, s_out = sequence.chunkwise_sequence_sharded(q.cuda(), k.cuda(), v.cuda(), gam, C, state_in=s_in.cuda())
        torch.cuda.synchronize()
        assert rel(y, y_ref) <= 2e-2 and rel(s_out, s_ref) <= 2e-2
    finally:
        dist.destroy_process_group()
    assert ret.device_status() == 0


def test_decode_graph_matches_eager_steps():
    from retnet_retention_chunkwise_b200.graphs import DecodeGraph
    B, H, dk, dv, n = 2, 4, 128, 256, 16
    gam = inputs.multiscale_gammas(H)
    s0 = inputs.state(B, H, dk, dv, seed=3, scale=0.5).cuda()
    tq, tk, tv = inputs.qkv(2 * n, B * H, 1, dk, dv, torch.bfloat16, seed=21)
    tq, tk, tv = (t.view(2 * n, B, H, 1, -1).cuda() for t in (tq, tk, tv))
    # eager: 2n steps
    s_eager = s0.clone()
    y_eager = torch.stack([ret.recurrent_step(tq[i], tk[i], tv[i], gam, s_eager) for i in range(2 * n)])
    # graph: n steps captured once, replayed twice with new inputs
    s_graph = s0.clone()
    g = DecodeGraph(s_graph, gam, n)
    ys = []
    for r in range(2):
        g.q.copy_(tq[r * n:(r + 1) * n])
        g.k.copy_(tk[r * n:(r + 1) * n])
        g.v.copy_(tv[r * n:(r + 1) * n])
        ys.append(g.replay().clone())
    torch.cuda.synchronize()
    assert ret.device_status() == 0
    assert torch.equal(torch.cat(ys), y_eager) and torch.equal(s_graph, s_eager)
    # and the oracle on the whole run of 2n tokens
    q_all = tq.reshape(2 * n, B, H, -1).permute(1, 2, 0, 3).cpu()
    k_all = tk.reshape(2 * n, B, H, -1).permute(1, 2, 0, 3).cpu()
    v_all = tv.reshape(2 * n, B, H, -1).permute(1, 2, 0, 3).cpu()
    y_ref, s_ref = oracle.recurrent(q_all, k_all, v_all, gam, s0.cpu())
    assert rel(torch.cat(ys).reshape(2 * n, B, H, dv).permute(1, 2, 0, 3), y_ref) <= 2e-2
    assert rel(s_graph, s_ref) <= 2e-2
