"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times, on heads sampled from the full tensors (the oracle checks each sampled
head over its whole sequence), plus properties that hold at any size.

Bound: max |gpu - oracle| / max |oracle| <= 2e-2 (bf16 inputs, fp32
accumulation and state), over the sampled heads."""
import numpy as np
import pytest
import torch

import oracle
import retnet_retention_chunkwise_b200 as ret
from retnet_retention_chunkwise_b200 import inputs

pytestmark = pytest.mark.gpu
TOL = 2e-2


def rel(gpu, ref):
    g = gpu.detach().double().cpu().numpy()
    assert np.all(np.isfinite(g))
    return float(np.max(np.abs(g - ref)) / max(np.max(np.abs(ref)), 1e-30))


def _heads(t, pairs):
    """[n, 1, L, d] host copy of the (b, h) pairs of a [B, H, L, d] tensor."""
    return torch.stack([t[b, h] for b, h in pairs]).unsqueeze(1).cpu()


def test_retnet1p3b_layer_sampled_heads():
    w = inputs.WORKLOADS["retnet1p3b_layer_bf16"]  # B4 H8 L8192 dk256 dv512, C128
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    y, s = ret.chunkwise(q, k, v, gam, w.chunk)
    assert ret.device_status() == 0
    pairs = [(0, 0), (3, 7), (1, 4)]
    g = torch.stack([gam[h] for _, h in pairs]).reshape(-1, 1)
    # the oracle runs each sampled head as its own (batch row, head 0) problem
    y_ref = np.zeros((len(pairs), w.L, w.dv))
    s_ref = np.zeros((len(pairs), w.dk, w.dv))
    for i, (b, h) in enumerate(pairs):
        yi, si = oracle.recurrent(_heads(q, [(b, h)]), _heads(k, [(b, h)]), _heads(v, [(b, h)]), g[i])
        y_ref[i], s_ref[i] = yi[0, 0], si[0, 0]
    assert rel(torch.stack([y[b, h] for b, h in pairs]), y_ref) <= TOL
    assert rel(torch.stack([s[b, h] for b, h in pairs]), s_ref) <= TOL


def test_decode_6p7b_sampled_heads():
    w = inputs.WORKLOADS["decode_6p7b_bf16"]  # B64 H16 dk256 dv512; 512-token prefill, C128
    steps = inputs.DECODE_STEPS
    gam = w.gammas()
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, 0)
    state = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    y_pre, _ = ret.chunkwise(q, k, v, gam, w.chunk, state_out=state)
    tq, tk, tv = inputs.qkv_cuda(steps, w.B * w.H, 1, w.dk, w.dv, w.dtype, 1)
    tq, tk, tv = (t.view(steps, w.B, w.H, 1, -1) for t in (tq, tk, tv))
    pairs = [(0, 0), (63, 15), (31, 8)]
    ys = []
    for n in range(steps):
        yn = ret.recurrent_step(tq[n], tk[n], tv[n], gam, state)
        ys.append(torch.stack([yn[b, h, 0] for b, h in pairs]))
    assert ret.device_status() == 0
    y_dec = torch.stack(ys, dim=1)  # [pairs, steps, dv]
    for i, (b, h) in enumerate(pairs):
        qq = torch.cat([q[b, h], tq[:, b, h, 0]]).reshape(1, 1, -1, w.dk).cpu()
        kk = torch.cat([k[b, h], tk[:, b, h, 0]]).reshape(1, 1, -1, w.dk).cpu()
        vv = torch.cat([v[b, h], tv[:, b, h, 0]]).reshape(1, 1, -1, w.dv).cpu()
        y_ref, s_ref = oracle.recurrent(qq, kk, vv, gam[h:h + 1])
        assert rel(y_pre[b, h], y_ref[0, 0, :w.L]) <= TOL
        assert rel(y_dec[i], y_ref[0, 0, w.L:]) <= TOL
        assert rel(state[b, h], s_ref[0, 0]) <= TOL


@pytest.mark.parametrize("C", [64, 128, 256])
def test_long_context_four_calls_match_one_call_and_oracle(C):
    w = inputs.WORKLOADS["long_context_bf16"]  # B1 H16 L65536 dk128 dv256
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    y_full, s_full = ret.chunkwise(q, k, v, gam, C)
    seg = w.L // inputs.LONG_CONTEXT_CALLS
    state = torch.zeros((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    parts = []
    for i in range(0, w.L, seg):
        y, _ = ret.chunkwise(q[:, :, i:i + seg].contiguous(), k[:, :, i:i + seg].contiguous(),
                             v[:, :, i:i + seg].contiguous(), gam, C, state_in=state, state_out=state)
        parts.append(y)
    y_split = torch.cat(parts, dim=2)
    assert ret.device_status() == 0
    # carried state reproduces the single call (both are checked against the oracle below)
    d = (y_split.double() - y_full.double()).abs().max().item() / y_full.double().abs().max().item()
    assert d <= TOL
    assert (state - s_full).abs().max().item() / s_full.abs().max().item() <= TOL
    for h in (0, 15):
        y_ref, s_ref = oracle.recurrent(_heads(q, [(0, h)]), _heads(k, [(0, h)]), _heads(v, [(0, h)]),
                                        gam[h:h + 1])
        assert rel(y_full[0, h], y_ref[0, 0]) <= TOL and rel(y_split[0, h], y_ref[0, 0]) <= TOL
        assert rel(s_full[0, h], s_ref[0, 0]) <= TOL and rel(state[0, h], s_ref[0, 0]) <= TOL


def test_state_only_headline_sampled_heads():
    # the state-only call at the shape bench.py times it
    w = inputs.WORKLOADS["retnet1p3b_layer_bf16"]
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    s = ret.chunkwise_state(k, v, gam, w.chunk)
    assert ret.device_status() == 0
    for b, h in [(0, 0), (3, 7)]:
        _, s_ref = oracle.recurrent(_heads(q, [(b, h)]), _heads(k, [(b, h)]), _heads(v, [(b, h)]), gam[h:h + 1])
        assert rel(s[b, h], s_ref[0, 0]) <= TOL


@pytest.mark.parametrize("gated", [False, True])
def test_groupnorm_headline_sampled_heads(gated):
    w = inputs.WORKLOADS["retnet1p3b_layer_bf16"]
    g = torch.Generator("cuda").manual_seed(3)
    y = (torch.randn((w.B, w.H, w.L, w.dv), generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    gate = torch.randn((w.B, w.H, w.L, w.dv), generator=g, device="cuda").to(torch.bfloat16)
    z = ret.groupnorm(y, 1e-5, gate=gate if gated else None, act="swish")
    assert ret.device_status() == 0
    for b, h in [(0, 0), (2, 5), (3, 7)]:
        ref = oracle.groupnorm(y[b, h].reshape(1, 1, w.L, w.dv).cpu(), eps=1e-5)
        if gated:
            ref = oracle.gate(ref, gate[b, h].reshape(1, 1, w.L, w.dv).cpu(), "swish")
        assert rel(z[b, h], ref[0, 0]) <= TOL


@pytest.mark.parametrize("with_state", [False, True])
def test_chunkwise_backward_long_context_call(with_state):
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
    for h in (0, 15):
        one = lambda t, a, b: t[0, h, a:b].reshape(1, 1, b - a, -1).cpu()  # noqa: E731
        st = lambda t: None if t is None else t[0, h].reshape(1, 1, w.dk, w.dv).cpu()  # noqa: E731
        g = gam[h:h + 1]
        pre = oracle.backward(one(q, 0, P), one(k, 0, P), one(v, 0, P), g, one(dy, 0, P), st(s0), None)
        assert rel(dq[0, h, :P], pre[0][0, 0]) <= TOL
        suf = oracle.backward(one(q, L - P, L), one(k, L - P, L), one(v, L - P, L), g, one(dy, L - P, L), None,
                              st(dso))
        assert rel(dkk[0, h, L - P:], suf[1][0, 0]) <= TOL
        assert rel(dvv[0, h, L - P:], suf[2][0, 0]) <= TOL
        if with_state:
            ds_ref = oracle.state_backward(one(q, 0, L), one(k, 0, L), one(v, 0, L), g, one(dy, 0, L), st(s0),
                                           st(dso))[3]
            assert rel(ds0[0, h], ds_ref[0, 0]) <= TOL


def test_parallel_backward_msr_core_sampled_heads():
    w = inputs.WORKLOADS["msr_core_bf16"]  # B2 H8 L2048 dk64 dv128
    q, k, v = inputs.qkv_cuda(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    gen = torch.Generator("cuda").manual_seed(6)
    dy = (torch.randn((w.B, w.H, w.L, w.dv), generator=gen, device="cuda") / 16.0).to(torch.bfloat16)
    dq, dkk, dvv = ret.parallel_backward(q, k, v, gam, dy)
    assert ret.device_status() == 0
    for b, h in [(0, 0), (1, 7)]:
        ref = oracle.parallel_backward(_heads(q, [(b, h)]), _heads(k, [(b, h)]), _heads(v, [(b, h)]),
                                       gam[h:h + 1], _heads(dy, [(b, h)]))
        for got, r in zip((dq, dkk, dvv), ref):
            assert rel(got[b, h], r[0, 0]) <= TOL
