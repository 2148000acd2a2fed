"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times, on EVERY (b, h) of every workload: the oracle runs each batch row (or a
group of heads) over its whole sequence, and each head is held to the bound on
its own scale as well as over the whole tensor (tests/parity.py).

Bound: max |gpu - oracle| / max |oracle| <= 2e-2 (bf16 inputs, fp32
accumulation and state).  The oracle's C functions release the GIL, so the
single-threaded ones run in a thread pool over heads."""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import oracle
import retnet_retention_chunkwise_b200 as ret
from retnet_retention_chunkwise_b200 import inputs
from tests.parity import rel

pytestmark = pytest.mark.gpu
TOL = 2e-2
NCPU = os.cpu_count() or 4


def _map(fn, items):
    oracle.load()  # built and loaded once, before the threads share it
    with cf.ThreadPoolExecutor(max_workers=NCPU) as ex:
        return list(ex.map(fn, items))


@pytest.fixture(scope="module")
def headline():
    """The headline chunkwise call and the state-only call, with the oracle's
    y and state_out for all 32 heads (one oracle call per batch row)."""
    w = inputs.WORKLOADS["retnet1p3b_layer_bf16"]  # B4 H8 L8192 dk256 dv512, C128
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    y, s = ret.chunkwise(q, k, v, gam, w.chunk)
    s_only = ret.chunkwise_state(k, v, gam, w.chunk)
    assert ret.device_status() == 0
    y_ref = np.empty((w.B, w.H, w.L, w.dv))
    s_ref = np.empty((w.B, w.H, w.dk, w.dv))
    for b in range(w.B):
        yb, sb = oracle.recurrent(q[b:b + 1].cpu(), k[b:b + 1].cpu(), v[b:b + 1].cpu(), gam)
        y_ref[b], s_ref[b] = yb[0], sb[0]
    return {"y": y.cpu(), "s": s.cpu(), "s_only": s_only.cpu(), "y_ref": y_ref, "s_ref": s_ref}


def test_retnet1p3b_layer_every_head(headline):
    assert rel(headline["y"], headline["y_ref"]) <= TOL
    assert rel(headline["s"], headline["s_ref"]) <= TOL


def test_state_only_headline_every_head(headline):
    # the state-only call at the shape bench.py times it
    assert rel(headline["s_only"], headline["s_ref"]) <= TOL


def test_decode_6p7b_every_head():
    w = inputs.WORKLOADS["decode_6p7b_bf16"]  # B64 H16 dk256 dv512; 512-token prefill, C128
    steps = inputs.DECODE_STEPS
    gam = w.gammas()
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, 0)
    state = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    y_pre, _ = ret.chunkwise(q, k, v, gam, w.chunk, state_out=state)
    tq, tk, tv = inputs.qkv_cuda(steps, w.B * w.H, 1, w.dk, w.dv, w.dtype, 1)
    tq, tk, tv = (t.view(steps, w.B, w.H, 1, -1) for t in (tq, tk, tv))
    y_dec = torch.empty((steps, w.B, w.H, 1, w.dv), dtype=w.dtype, device="cuda")
    for n in range(steps):
        ret.recurrent_step(tq[n], tk[n], tv[n], gam, state, out=y_dec[n])
    assert ret.device_status() == 0
    for b in range(w.B):  # the oracle over prefill + steps, one batch row (16 heads) at a time
        cat = lambda a, t: torch.cat([a[b], t[:, b, :, 0].transpose(0, 1)], dim=1).unsqueeze(0).cpu()  # noqa: E731
        y_ref, s_ref = oracle.recurrent(cat(q, tq), cat(k, tk), cat(v, tv), gam)
        assert rel(y_pre[b:b + 1], y_ref[:, :, :w.L]) <= TOL, b
        assert rel(y_dec[:, b, :, 0].transpose(0, 1).unsqueeze(0), y_ref[:, :, w.L:]) <= TOL, b
        assert rel(state[b:b + 1], s_ref) <= TOL, b


def test_long_context_every_head_all_chunks():
    # C in {64, 128, 256}: one 65536-token call and four 16384-token calls with
    # the state carried; every head of all six results against one oracle run
    w = inputs.WORKLOADS["long_context_bf16"]  # B1 H16 L65536 dk128 dv256
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    seg = w.L // inputs.LONG_CONTEXT_CALLS
    got = {}
    for C in (64, 128, 256):
        y_full, s_full = ret.chunkwise(q, k, v, gam, C)
        state = torch.zeros((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
        parts = []
        for i in range(0, w.L, seg):
            y, _ = ret.chunkwise(q[:, :, i:i + seg].contiguous(), k[:, :, i:i + seg].contiguous(),
                                 v[:, :, i:i + seg].contiguous(), gam, C, state_in=state, state_out=state)
            parts.append(y)
        got[C] = (y_full, s_full, torch.cat(parts, dim=2), state)
    assert ret.device_status() == 0
    G = 4  # heads per oracle call
    for h0 in range(0, w.H, G):
        sl = slice(h0, h0 + G)
        y_ref, s_ref = oracle.recurrent(q[:, sl].cpu(), k[:, sl].cpu(), v[:, sl].cpu(), gam[sl])
        for C, (y_full, s_full, y_split, s_split) in got.items():
            assert rel(y_full[:, sl], y_ref) <= TOL, (C, "one call", h0)
            assert rel(y_split[:, sl], y_ref) <= TOL, (C, "four calls", h0)
            assert rel(s_full[:, sl], s_ref) <= TOL and rel(s_split[:, sl], s_ref) <= TOL, (C, h0)


@pytest.mark.parametrize("gated", [False, True])
def test_groupnorm_headline_every_head(gated):
    w = inputs.WORKLOADS["retnet1p3b_layer_bf16"]
    g = torch.Generator("cuda").manual_seed(3)
    y = (torch.randn((w.B, w.H, w.L, w.dv), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    gate = torch.randn((w.B, w.H, w.L, w.dv), generator=g, device="cuda").to(torch.bfloat16)
    z = ret.groupnorm(y, 1e-5, gate=gate if gated else None, act="swish")
    assert ret.device_status() == 0

    def row(b):
        ref = oracle.groupnorm(y[b:b + 1].cpu(), eps=1e-5)
        if gated:
            ref = oracle.gate(ref, gate[b:b + 1].cpu(), "swish")
        return ref

    for b, ref in enumerate(_map(row, range(w.B))):
        assert rel(z[b:b + 1], ref) <= TOL, b


@pytest.mark.parametrize("with_state", [False, True])
def test_chunkwise_backward_long_context_every_head(with_state):
    # one 16384-token call of the long-context layout, as bench.py times it.
    # dq_n needs only tokens <= n, so the oracle's backward of the first P tokens
    # gives the exact dq rows there; dk_m and dv_m need only tokens >= m, so the
    # backward of the last P tokens gives their exact rows there; dS0 comes from
    # the state terms over the whole call (linear in L).
    w = inputs.WORKLOADS["long_context_bf16"]
    L = w.L // inputs.LONG_CONTEXT_CALLS
    q, k, v = inputs.qkv_cuda(w.B, w.H, L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    gen = torch.Generator("cuda").manual_seed(4)
    dy = (torch.randn((w.B, w.H, L, w.dv), generator=gen, device="cuda") / 16.0).to(torch.bfloat16)
    s0 = torch.randn((w.B, w.H, w.dk, w.dv), generator=gen, device="cuda") * 0.5 if with_state else None
    dso = torch.randn((w.B, w.H, w.dk, w.dv), generator=gen, device="cuda") * 0.5 if with_state else None
    if with_state:
        dq, dkk, dvv, ds0 = ret.chunkwise_backward_state(q, k, v, gam, dy, 128, s0, dso)
    else:
        dq, dkk, dvv = ret.chunkwise_backward(q, k, v, gam, dy, 128)
    assert ret.device_status() == 0
    P = 1024
    qh, kh, vh, dyh = q.cpu(), k.cpu(), v.cpu(), dy.cpu()
    s0h = None if s0 is None else s0.cpu()
    dsoh = None if dso is None else dso.cpu()

    def head(h):
        one = lambda t, a, b: t[:, h:h + 1, a:b]  # noqa: E731
        st = lambda t: None if t is None else t[:, h:h + 1]  # noqa: E731
        g = gam[h:h + 1]
        pre = oracle.backward(one(qh, 0, P), one(kh, 0, P), one(vh, 0, P), g, one(dyh, 0, P), st(s0h), None)
        suf = oracle.backward(one(qh, L - P, L), one(kh, L - P, L), one(vh, L - P, L), g, one(dyh, L - P, L),
                              None, st(dsoh))
        ds = None
        if with_state:
            ds = oracle.state_backward(one(qh, 0, L), one(kh, 0, L), one(vh, 0, L), g, one(dyh, 0, L), st(s0h),
                                       st(dsoh))[3]
        return pre[0], suf[1], suf[2], ds

    refs = _map(head, range(w.H))
    assert rel(dq[:, :, :P], np.concatenate([r[0] for r in refs], axis=1)) <= TOL
    assert rel(dkk[:, :, L - P:], np.concatenate([r[1] for r in refs], axis=1)) <= TOL
    assert rel(dvv[:, :, L - P:], np.concatenate([r[2] for r in refs], axis=1)) <= TOL
    if with_state:
        assert rel(ds0, np.concatenate([r[3] for r in refs], axis=1)) <= TOL


def test_parallel_backward_msr_core_every_head():
    w = inputs.WORKLOADS["msr_core_bf16"]  # B2 H8 L2048 dk64 dv128
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    gen = torch.Generator("cuda").manual_seed(6)
    dy = (torch.randn((w.B, w.H, w.L, w.dv), generator=gen, device="cuda") / 16.0).to(torch.bfloat16)
    dq, dkk, dvv = ret.parallel_backward(q, k, v, gam, dy)
    assert ret.device_status() == 0
    qh, kh, vh, dyh = q.cpu(), k.cpu(), v.cpu(), dy.cpu()
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]

    def head(bh):
        b, h = bh
        sl = lambda t: t[b:b + 1, h:h + 1]  # noqa: E731
        return oracle.parallel_backward(sl(qh), sl(kh), sl(vh), gam[h:h + 1], sl(dyh))

    refs = _map(head, pairs)
    for i, got in enumerate((dq, dkk, dvv)):
        ref = np.stack([r[i][0, 0] for r in refs]).reshape(w.B, w.H, w.L, -1)
        assert rel(got, ref) <= TOL, i


def test_parallel_and_chunkwise_msr_core_every_head():
    # the two forms bench.py times on the MSR core, against the oracle
    w = inputs.WORKLOADS["msr_core_bf16"]
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    yp = ret.parallel(q, k, v, gam)
    yc, sc = ret.chunkwise(q, k, v, gam, w.chunk)
    assert ret.device_status() == 0
    y_ref, s_ref = oracle.recurrent(q.cpu(), k.cpu(), v.cpu(), gam)
    assert rel(yp, y_ref) <= TOL and rel(yc, y_ref) <= TOL and rel(sc, s_ref) <= TOL
