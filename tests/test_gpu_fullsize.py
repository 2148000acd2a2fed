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
