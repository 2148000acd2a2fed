"""GPU parity: every kernel, through the C ABI, against the fp64 oracle.

Metric: max |gpu - oracle| / max |oracle|, over each tensor and over each of
its (b, h) slices on its own (tests/parity.py).  Bounds: 1e-4 for fp32 inputs,
2e-2 for bf16 inputs (fp32 accumulation and state).  Both sides read the
same seeded bytes; the oracle widens them to fp64 exactly.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import retnet_retention_chunkwise_b200 as ret
from retnet_retention_chunkwise_b200 import inputs
from tests.parity import rel

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}




def dev(*ts):
    return [None if t is None else t.cuda() for t in ts]


@pytest.fixture(autouse=True)
def _status_clean():
    yield
    assert ret.device_status() == 0


# ------------------------------------------------------------ fp32 (1e-4)
def test_single_head_f32_all_forms():
    w = inputs.WORKLOADS["single_head_f32"]
    q, k, v = inputs.qkv(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    gam = w.gammas()
    y_ref, s_ref = oracle.recurrent(q, k, v, gam)
    qd, kd, vd = dev(q, k, v)
    y = ret.parallel(qd, kd, vd, gam)
    assert rel(y, y_ref) <= 1e-4
    y, s = ret.chunkwise(qd, kd, vd, gam, w.chunk)
    assert rel(y, y_ref) <= 1e-4 and rel(s, s_ref) <= 1e-4
    state = torch.zeros(w.B, w.H, w.dk, w.dv, device="cuda")
    ys = [ret.recurrent_step(qd[:, :, n:n + 1].contiguous(), kd[:, :, n:n + 1].contiguous(),
                             vd[:, :, n:n + 1].contiguous(), gam, state) for n in range(w.L)]
    assert rel(torch.cat(ys, dim=2), y_ref) <= 1e-4 and rel(state, s_ref) <= 1e-4


@pytest.mark.parametrize("B,H,L,dk,dv,C", [(2, 3, 37, 16, 24, 16), (1, 2, 130, 64, 40, 32),
                                           (1, 1, 5, 8, 8, 64), (1, 2, 64, 256, 33, 7)])
def test_f32_ragged_with_state(B, H, L, dk, dv, C):
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.float32, seed=3)
    s_in = inputs.state(B, H, dk, dv, seed=4, scale=0.3)
    gam = torch.tensor([0.5, 0.999, 0.0][:H] if H <= 3 else [0.9] * H)
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    qd, kd, vd, sd = dev(q, k, v, s_in)
    y, s = ret.chunkwise(qd, kd, vd, gam, C, state_in=sd)
    assert rel(y, y_ref) <= 1e-4 and rel(s, s_ref) <= 1e-4
    y0_ref, _ = oracle.recurrent(q, k, v, gam)
    assert rel(ret.parallel(qd, kd, vd, gam), y0_ref) <= 1e-4


# ------------------------------------------------------ bf16 chunkwise (2e-2)
def _chunk_case(B, H, L, dk, dv, C, gam=None, with_state=False, seed=0, ws="auto"):
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed)
    gam = inputs.multiscale_gammas(H) if gam is None else torch.tensor(gam, dtype=torch.float32)
    s_in = inputs.state(B, H, dk, dv, seed=seed + 7, scale=0.5) if with_state else None
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    qd, kd, vd, sd = dev(q, k, v, s_in)
    kw = {} if ws == "auto" else {"workspace": ws}
    y, s = ret.chunkwise(qd, kd, vd, gam, C, state_in=sd, **kw)
    return rel(y, y_ref), rel(s, s_ref)


def test_msr_core_chunkwise():
    w = inputs.WORKLOADS["msr_core_bf16"]
    ey, es = _chunk_case(w.B, w.H, w.L, w.dk, w.dv, w.chunk)
    assert ey <= 2e-2 and es <= 2e-2, (ey, es)


@pytest.mark.parametrize("B,H,L,dk,dv,C", [
    (1, 2, 200, 64, 128, 64),      # ragged tail
    (1, 1, 50, 64, 128, 64),       # L < C
    (1, 1, 1, 64, 128, 16),        # single token
    (2, 2, 300, 128, 256, 128),    # dk 128, two dv slices
    (1, 2, 260, 256, 128, 128),    # dk 256 (single P buffer)
    (1, 1, 333, 64, 128, 48),      # C % 32 == 16
    (1, 1, 160, 128, 128, 16),     # smallest block
    (1, 2, 520, 256, 256, 32),
    (2, 3, 700, 256, 384, 64),     # dk 256, ragged, three dv slices
    (1, 2, 700, 128, 256, 256),    # blocks of 256 rows (two row halves), ragged tail
    (1, 1, 200, 64, 128, 256),     # L < C = 256: half b partly past the end
    (1, 1, 1, 64, 128, 256),       # single token in a 256 block
    (1, 2, 520, 128, 128, 144),    # C = 144: half b of 16 rows, C % 32 == 16
    (2, 1, 1000, 64, 256, 240),    # C = 240
])
def test_chunkwise_shapes(B, H, L, dk, dv, C):
    ey, es = _chunk_case(B, H, L, dk, dv, C, with_state=True, seed=L)
    assert ey <= 2e-2 and es <= 2e-2, (ey, es)


def test_chunkwise_special_gammas():
    # gamma = 0 keeps only the diagonal; gamma = 1 is un-normalised linear attention
    ey, es = _chunk_case(1, 3, 257, 64, 128, 64, gam=[0.0, 1.0, 0.5], with_state=True, seed=11)
    assert ey <= 2e-2 and es <= 2e-2, (ey, es)


@pytest.mark.parametrize("dk,C", [(128, 128), (128, 64), (256, 128), (256, 64), (128, 256), (64, 176)])
def test_chunkwise_small_gammas_direct_form(dk, C):
    # gamma^(C-1) < 2^-64 takes the direct form (decay applied to P and O);
    # the other heads take the rescaled form.
    ey, es = _chunk_case(1, 4, 300, dk, 128, C, gam=[0.5, 0.25, 0.6, 0.97], with_state=True, seed=13)
    assert ey <= 2e-2 and es <= 2e-2, (ey, es)


@pytest.mark.parametrize("dk,C", [(256, 128), (256, 64), (128, 128), (128, 256)])
def test_chunkwise_rescaled_state_renormalisation(dk, C):
    # gamma^(C-1) >= 2^-64 keeps these heads in the rescaled form, and the
    # decay of the stored state runs below 2^-64 after one to a few blocks
    # (every other block for 0.75 at C = 128), so the scaled state is
    # multiplied through several times in one call.
    B, H, L, dv = 1, 4, 1100, 256
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=17)
    gam = torch.tensor([0.75, 0.9, 0.97, 1.0])
    s_in = inputs.state(B, H, dk, dv, seed=3, scale=0.5)
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    qd, kd, vd, sd = dev(q, k, v, s_in)
    y, s = ret.chunkwise(qd, kd, vd, gam, C, state_in=sd)
    for h in range(H):  # per head: the gamma = 1 head would dominate a joint bound
        assert rel(y[:, h], y_ref[:, h]) <= 2e-2 and rel(s[:, h], s_ref[:, h]) <= 2e-2, h


@pytest.mark.parametrize("dk,C", [(64, 64), (128, 256)])
def test_chunkwise_sequence_split_matches_single_pass(dk, C):
    B, H, L, dv = 1, 2, 4096, 128
    assert ret.workspace_bytes(C, B, H, L, dk, dv) > 0
    ey, es = _chunk_case(B, H, L, dk, dv, C, with_state=True, seed=5)
    assert ey <= 2e-2 and es <= 2e-2, (ey, es)
    ey0, es0 = _chunk_case(B, H, L, dk, dv, C, with_state=True, seed=5, ws=None)
    assert ey0 <= 2e-2 and es0 <= 2e-2, (ey0, es0)


def test_chunkwise_state_in_place_and_split_calls():
    B, H, L, dk, dv, C = 1, 4, 1024, 128, 256, 128
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, 21)
    gam = inputs.multiscale_gammas(H)
    y_ref, s_ref = oracle.recurrent(q, k, v, gam)
    qd, kd, vd = dev(q, k, v)
    state = torch.zeros(B, H, dk, dv, device="cuda")
    ys = []
    for c0 in (0, 256, 640):  # uneven calls, state carried in place
        c1 = {0: 256, 256: 640, 640: L}[c0]
        y, _ = ret.chunkwise(qd[:, :, c0:c1].contiguous(), kd[:, :, c0:c1].contiguous(),
                             vd[:, :, c0:c1].contiguous(), gam, C, state_in=state, state_out=state)
        ys.append(y)
    assert rel(torch.cat(ys, dim=2), y_ref) <= 2e-2 and rel(state, s_ref) <= 2e-2


def test_chunkwise_empty_sequence_passes_state():
    s_in = inputs.state(1, 2, 64, 128, seed=1).cuda()
    e = torch.empty(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    ev = torch.empty(1, 2, 0, 128, dtype=torch.bfloat16, device="cuda")
    _, s = ret.chunkwise(e, e, ev, [0.5, 0.9], 64, state_in=s_in)
    assert torch.equal(s, s_in)


# ------------------------------------------------------- bf16 parallel (2e-2)
@pytest.mark.parametrize("B,H,L,dk,dv", [(2, 8, 2048, 64, 128), (1, 2, 1000, 128, 256),
                                         (1, 1, 300, 256, 128), (1, 3, 77, 64, 128),
                                         (1, 2, 129, 256, 256), (3, 1, 512, 128, 384)])
def test_parallel(B, H, L, dk, dv):
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=L)
    gam = inputs.multiscale_gammas(H) if H != 3 else torch.tensor([0.0, 1.0, 0.7])
    y_ref, _ = oracle.recurrent(q, k, v, gam)
    qd, kd, vd = dev(q, k, v)
    assert rel(ret.parallel(qd, kd, vd, gam), y_ref) <= 2e-2


def test_parallel_and_chunkwise_agree_msr_core():
    w = inputs.WORKLOADS["msr_core_bf16"]
    q, k, v = dev(*inputs.qkv(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed))
    gam = w.gammas()
    yp = ret.parallel(q, k, v, gam).double()
    yc, _ = ret.chunkwise(q, k, v, gam, w.chunk)
    assert (yp - yc.double()).abs().max().item() / yp.abs().max().item() <= 2e-2


# --------------------------------------------------------- decode (2e-2)
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_recurrent_steps(dt):
    B, H, dk, dv, steps = 2, 4, 256, 512, 12
    qs, ks, vs = inputs.decode_tokens(steps, B, H, dk, dv, dt, seed=1)
    s0 = inputs.state(B, H, dk, dv, seed=9, scale=0.2)
    gam = inputs.multiscale_gammas(H)
    q = torch.cat(list(qs), dim=2)
    k = torch.cat(list(ks), dim=2)
    v = torch.cat(list(vs), dim=2)
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s0)
    state = s0.cuda()
    ys = [ret.recurrent_step(qs[n].cuda(), ks[n].cuda(), vs[n].cuda(), gam, state) for n in range(steps)]
    tol = TOL[dt]
    assert rel(torch.cat(ys, dim=2), y_ref) <= tol and rel(state, s_ref) <= tol


def test_recurrent_step_odd_dv():
    B, H, dk, dv = 1, 2, 20, 30
    q, k, v = inputs.qkv(B, H, 1, dk, dv, torch.float32, seed=2)
    s0 = inputs.state(B, H, dk, dv, seed=3)
    gam = torch.tensor([0.25, 1.0])
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s0)
    state = s0.cuda()
    y = ret.recurrent_step(*dev(q, k, v), gam, state)
    assert rel(y, y_ref) <= 1e-4 and rel(state, s_ref) <= 1e-4


@pytest.mark.parametrize("dt,B,H,dk,dv", [
    (torch.bfloat16, 1, 40, 128, 512),
    (torch.bfloat16, 1, 24, 128, 512),
    (torch.float32, 1, 1, 256, 512),     # one head
    (torch.float32, 1, 2, 64, 30),       # scalar columns
])
def test_recurrent_steps_small_batch(dt, B, H, dk, dv):
    steps = 4
    qs, ks, vs = inputs.decode_tokens(steps, B, H, dk, dv, dt, seed=5)
    s0 = inputs.state(B, H, dk, dv, seed=6, scale=0.3)
    gam = inputs.multiscale_gammas(H)
    y_ref, s_ref = oracle.recurrent(torch.cat(list(qs), dim=2), torch.cat(list(ks), dim=2),
                                    torch.cat(list(vs), dim=2), gam, s0)
    state = s0.cuda()
    ys = [ret.recurrent_step(qs[n].cuda(), ks[n].cuda(), vs[n].cuda(), gam, state) for n in range(steps)]
    assert ret.device_status() == 0
    assert rel(torch.cat(ys, dim=2), y_ref) <= TOL[dt] and rel(state, s_ref) <= TOL[dt]


# ------------------------------------------------- host-buffer entry point
def test_chunkwise_host_matches_device_call_and_oracle():
    B, H, L, dk, dv, C = 2, 3, 700, 128, 256, 128
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=41)
    gam = inputs.multiscale_gammas(H)
    s_in = inputs.state(B, H, dk, dv, seed=4, scale=0.5)
    qd, kd, vd, sd = dev(q, k, v, s_in)
    y_d, s_d = ret.chunkwise(qd, kd, vd, gam, C, state_in=sd, workspace=None)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    # uneven groups (heads [0, 2) and [2, 3) of each batch row), no sequence split:
    # the same per-CTA work as the device call, so the same bits
    s_h = torch.empty_like(sd)
    y_h, _ = ret.chunkwise_host(qh, kh, vh, gam, C, state_in=sd, state_out=s_h, workspace=None, n_groups=4)
    torch.cuda.synchronize()
    assert ret.device_status() == 0
    assert torch.equal(y_h, y_d.cpu()) and torch.equal(s_h, s_d)
    # default workspace (sequence split per group), checked against the oracle
    s_h2 = torch.empty_like(sd)
    y_h2, _ = ret.chunkwise_host(qh, kh, vh, gam, C, state_in=sd, state_out=s_h2, n_groups=5)
    torch.cuda.synchronize()
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    assert rel(y_h2, y_ref) <= 2e-2 and rel(s_h2, s_ref) <= 2e-2


# ------------------------------------------- per-head group normalisation
@pytest.mark.parametrize("dt,dv,affine", [(torch.float32, 128, True), (torch.float32, 40, False),
                                          (torch.bfloat16, 512, True), (torch.bfloat16, 96, False)])
def test_groupnorm_standalone(dt, dv, affine):
    B, H, L = 2, 3, 37
    g = torch.Generator("cpu").manual_seed(dv)
    y = (torch.randn((B, H, L, dv), generator=g) * 2.0 + 0.5).to(dt)
    w = (torch.rand(H * dv, generator=g) + 0.5) if affine else None
    b = torch.randn(H * dv, generator=g) if affine else None
    ref = oracle.groupnorm(y, eps=1e-5, weight=w, bias=b)
    out = ret.groupnorm(y.cuda(), 1e-5, weight=None if w is None else w.cuda(), bias=None if b is None else b.cuda())
    tol = 1e-4 if dt == torch.float32 else 2e-2
    assert rel(out, ref) <= tol
    # in place
    yd = y.cuda()
    ret.groupnorm(yd, 1e-5, weight=None if w is None else w.cuda(), bias=None if b is None else b.cuda(), out=yd)
    assert torch.equal(yd, out)


@pytest.mark.parametrize("act", ["swish", "sigmoid"])
def test_chunkwise_groupnorm_gated(act):
    B, H, L, dk, dv, C = 1, 2, 300, 128, 256, 128
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=L + 11)
    gam = inputs.multiscale_gammas(H)
    s_in = inputs.state(B, H, dk, dv, seed=12, scale=0.5)
    g = torch.Generator("cpu").manual_seed(13)
    gate = (torch.randn((B, H, L, dv), generator=g) * 2.0).to(torch.bfloat16)
    w = torch.rand(H * dv, generator=g) + 0.5
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    z_ref = oracle.gate(oracle.groupnorm(y_ref, eps=1e-5, weight=w), gate, act)
    qd, kd, vd, sd = dev(q, k, v, s_in)
    z, s = ret.chunkwise_groupnorm(qd, kd, vd, gam, C, 1e-5, weight=w.cuda(), state_in=sd, gate=gate.cuda(), act=act)
    assert ret.device_status() == 0
    assert rel(z, z_ref) <= 2e-2 and rel(s, s_ref) <= 2e-2


@pytest.mark.parametrize("dt,dv", [(torch.bfloat16, 512), (torch.bfloat16, 128), (torch.bfloat16, 96),
                                   (torch.float32, 128), (torch.float32, 48)])
@pytest.mark.parametrize("act", ["swish", "sigmoid", "none"])
def test_groupnorm_gated(dt, dv, act):
    B, H, L = 2, 3, 29
    g = torch.Generator("cpu").manual_seed(dv + 7)
    y = (torch.randn((B, H, L, dv), generator=g) * 2.0 + 0.5).to(dt)
    gate = (torch.randn((B, H, L, dv), generator=g) * 3.0).to(dt)
    w = torch.rand(H * dv, generator=g) + 0.5
    b = torch.randn(H * dv, generator=g) * 0.1
    ref = oracle.gate(oracle.groupnorm(y, eps=1e-5, weight=w, bias=b), gate, act)
    yd, gd = y.cuda(), gate.cuda()
    out = ret.groupnorm(yd, 1e-5, weight=w.cuda(), bias=b.cuda(), gate=gd, act=act)
    tol = 1e-4 if dt == torch.float32 else 2e-2
    assert rel(out, ref) <= tol
    ret.groupnorm(yd, 1e-5, weight=w.cuda(), bias=b.cuda(), gate=gd, act=act, out=yd)  # in place
    assert torch.equal(yd, out)
    assert ret.device_status() == 0


@pytest.mark.parametrize("B,H,L,dk,dv,C", [
    (1, 2, 700, 256, 512, 128),    # sequence split, ragged tail, four dv slices
    (2, 2, 300, 256, 128, 64),
    (1, 2, 300, 128, 256, 128),
    (1, 2, 600, 64, 128, 256),     # 256-row blocks
])
def test_chunkwise_groupnorm(B, H, L, dk, dv, C):
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=L + dv)
    gam = inputs.multiscale_gammas(H)
    s_in = inputs.state(B, H, dk, dv, seed=8, scale=0.5)
    g = torch.Generator("cpu").manual_seed(3)
    w = torch.rand(H * dv, generator=g) + 0.5
    b = torch.randn(H * dv, generator=g) * 0.1
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    z_ref = oracle.groupnorm(y_ref, eps=1e-5, weight=w, bias=b)
    qd, kd, vd, sd = dev(q, k, v, s_in)
    z, s = ret.chunkwise_groupnorm(qd, kd, vd, gam, C, 1e-5, weight=w.cuda(), bias=b.cuda(), state_in=sd)
    assert ret.device_status() == 0
    assert rel(z, z_ref) <= 2e-2 and rel(s, s_ref) <= 2e-2, (rel(z, z_ref), rel(s, s_ref))
    # the same as the two calls in sequence
    y2, _ = ret.chunkwise(qd, kd, vd, gam, C, state_in=sd)
    assert torch.equal(ret.groupnorm(y2, 1e-5, weight=w.cuda(), bias=b.cuda()), z)


@pytest.mark.parametrize("B,H,L,dk,dv", [(1, 2, 300, 128, 64), (2, 1, 1000, 64, 192)])
def test_parallel_64_column_slices(B, H, L, dk, dv):
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=dv + L)
    gam = inputs.multiscale_gammas(H)
    y_ref, _ = oracle.recurrent(q, k, v, gam)
    qd, kd, vd = dev(q, k, v)
    assert rel(ret.parallel(qd, kd, vd, gam), y_ref) <= 2e-2


# ------------------------------------------------ backward of the parallel form
@pytest.mark.parametrize("dt,B,H,L,dk,dv", [
    (torch.bfloat16, 2, 4, 300, 64, 128),
    (torch.bfloat16, 1, 2, 1000, 128, 64),
    (torch.bfloat16, 1, 3, 257, 64, 64),
    (torch.bfloat16, 1, 2, 520, 128, 256),
    (torch.float32, 1, 2, 70, 32, 48),
])
def test_parallel_backward(dt, B, H, L, dk, dv):
    q, k, v = inputs.qkv(B, H, L, dk, dv, dt, seed=L + dk)
    g = torch.Generator("cpu").manual_seed(L)
    dy = (torch.randn((B, H, L, dv), generator=g) / math.sqrt(dv)).to(dt)
    gam = inputs.multiscale_gammas(H) if H != 3 else torch.tensor([0.0, 1.0, 0.9])
    dq_r, dk_r, dv_r = oracle.parallel_backward(q, k, v, gam, dy)
    qd, kd, vd, dyd = dev(q, k, v, dy)
    dq, dkk, dvv = ret.parallel_backward(qd, kd, vd, gam, dyd)
    assert ret.device_status() == 0
    tol = 1e-4 if dt == torch.float32 else 2e-2
    errs = (rel(dq, dq_r), rel(dkk, dk_r), rel(dvv, dv_r))
    assert max(errs) <= tol, errs


# ------------------------------------------------------------- guard bands
def _guarded(shape, dtype, fill):
    """A tensor of `shape` at the start of a larger buffer whose tail (64 KB)
    holds `fill`; returns (tensor, tail)."""
    n = int(np.prod(shape))
    pad = 65536 // torch.tensor([], dtype=dtype).element_size()
    buf = torch.full((n + pad,), fill, dtype=dtype, device="cuda")
    return buf[:n].view(shape), buf[n:]


@pytest.mark.parametrize("B,H,L,dk,dv,C", [(1, 2, 333, 64, 128, 64), (1, 1, 200, 128, 256, 256),
                                          (1, 2, 150, 256, 128, 128), (2, 1, 77, 128, 128, 16)])
def test_outputs_stay_inside_their_buffers(B, H, L, dk, dv, C):
    q, k, v = dev(*inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=3))
    gam = inputs.multiscale_gammas(H)
    y, y_tail = _guarded((B, H, L, dv), torch.bfloat16, 7.0)
    s, s_tail = _guarded((B, H, dk, dv), torch.float32, 7.0)
    ret.chunkwise(q, k, v, gam, C, state_out=s, out=y)
    yp, yp_tail = _guarded((B, H, L, dv), torch.bfloat16, 7.0)
    ret.parallel(q, k, v, gam, out=yp)
    yd, yd_tail = _guarded((B, H, 1, dv), torch.bfloat16, 7.0)
    st = torch.zeros((B, H, dk, dv), dtype=torch.float32, device="cuda")
    ret.recurrent_step(q[:, :, :1].contiguous(), k[:, :, :1].contiguous(), v[:, :, :1].contiguous(), gam, st, out=yd)
    z, z_tail = _guarded((B, H, L, dv), torch.bfloat16, 7.0)
    ret.groupnorm(yp, 1e-5, out=z)
    torch.cuda.synchronize()
    assert ret.device_status() == 0
    for name, tail in (("chunkwise y", y_tail), ("state", s_tail), ("parallel y", yp_tail),
                       ("decode y", yd_tail), ("groupnorm", z_tail)):
        assert bool((tail == 7.0).all()), f"{name}: write past the end of the output"


@pytest.mark.parametrize("dt,B,H,L,dk,dv,C", [
    (torch.bfloat16, 1, 2, 700, 128, 256, 128),
    (torch.bfloat16, 1, 2, 1000, 256, 128, 64),
    (torch.bfloat16, 1, 1, 600, 128, 128, 256),    # 256-row blocks
    (torch.bfloat16, 1, 2, 4096, 128, 128, 128),   # sequence split in all three calls
    (torch.float32, 1, 2, 70, 32, 48, 16),
])
def test_chunkwise_backward(dt, B, H, L, dk, dv, C):
    q, k, v = inputs.qkv(B, H, L, dk, dv, dt, seed=L + C)
    g = torch.Generator("cpu").manual_seed(L + 1)
    dy = (torch.randn((B, H, L, dv), generator=g) / math.sqrt(dv)).to(dt)
    gam = inputs.multiscale_gammas(H)
    dq_r, dk_r, dv_r = oracle.parallel_backward(q, k, v, gam, dy)
    qd, kd, vd, dyd = dev(q, k, v, dy)
    dq, dkk, dvv = ret.chunkwise_backward(qd, kd, vd, gam, dyd, C)
    assert ret.device_status() == 0
    tol = 1e-4 if dt == torch.float32 else 2e-2
    errs = (rel(dq, dq_r), rel(dkk, dk_r), rel(dvv, dv_r))
    assert max(errs) <= tol, errs


def _state_grad_inputs(dt, B, H, L, dk, dv, seed):
    q, k, v = inputs.qkv(B, H, L, dk, dv, dt, seed=seed)
    g = torch.Generator("cpu").manual_seed(seed + 1)
    dy = (torch.randn((B, H, L, dv), generator=g) / math.sqrt(dv)).to(dt)
    s0 = torch.randn((B, H, dk, dv), generator=g) / math.sqrt(dk)
    dso = torch.randn((B, H, dk, dv), generator=g) / math.sqrt(dv)
    return q, k, v, dy, s0, dso


@pytest.mark.parametrize("dt,B,H,L,dk,dv,C", [
    (torch.bfloat16, 1, 2, 700, 128, 256, 128),
    (torch.bfloat16, 2, 2, 1000, 256, 128, 64),
    (torch.bfloat16, 1, 1, 600, 128, 128, 256),    # 256-row blocks
    (torch.bfloat16, 1, 2, 4096, 128, 128, 128),   # sequence split in all three calls
    (torch.float32, 1, 2, 70, 32, 48, 16),
])
def test_chunkwise_backward_state(dt, B, H, L, dk, dv, C):
    q, k, v, dy, s0, dso = _state_grad_inputs(dt, B, H, L, dk, dv, L + C + 3)
    gam = inputs.multiscale_gammas(H)
    ref = oracle.backward(q, k, v, gam, dy, s0, dso)
    qd, kd, vd, dyd, s0d, dsod = dev(q, k, v, dy, s0, dso)
    got = ret.chunkwise_backward_state(qd, kd, vd, gam, dyd, C, s0d, dsod)
    assert ret.device_status() == 0
    tol = 1e-4 if dt == torch.float32 else 2e-2
    errs = [rel(a, b) for a, b in zip(got, ref)]
    assert max(errs) <= tol, errs


@pytest.mark.parametrize("dt", [torch.float32, torch.bfloat16])
def test_chunkwise_backward_state_small_gamma_heads(dt):
    # gamma 0 and 2^-70 take the zero-state route with the last-row term;
    # 0.5 and 1 the scaled initial state; checked head by head
    B, H, L, dk, dv, C = 1, 4, 37, 128, 128, 16
    q, k, v, dy, s0, dso = _state_grad_inputs(dt, B, H, L, dk, dv, 91)
    gam = np.array([0.0, 2.0 ** -70, 0.5, 1.0])
    ref = oracle.backward(q, k, v, gam, dy, s0, dso)
    got = ret.chunkwise_backward_state(*dev(q, k, v), gam, dy.cuda(), C, s0.cuda(), dso.cuda())
    assert ret.device_status() == 0
    tol = 1e-4 if dt == torch.float32 else 2e-2
    for h in range(H):
        errs = [rel(a[:, h], b[:, h]) for a, b in zip(got, ref) if np.max(np.abs(b[:, h])) > 0]
        assert max(errs) <= tol, (h, errs)
    assert torch.count_nonzero(got[3][:, 0]) == 0  # gamma = 0: dS0 = 0


def test_chunkwise_backward_state_aliasing_and_optional_states():
    dt, B, H, L, dk, dv, C = torch.bfloat16, 1, 2, 300, 128, 128, 64
    q, k, v, dy, s0, dso = _state_grad_inputs(dt, B, H, L, dk, dv, 17)
    gam = inputs.multiscale_gammas(H)
    qd, kd, vd, dyd, s0d, dsod = dev(q, k, v, dy, s0, dso)
    base = ret.chunkwise_backward_state(qd, kd, vd, gam, dyd, C, s0d, dsod)
    # dstate_in written over dstate_out: the same bits
    buf = dsod.clone()
    al = ret.chunkwise_backward_state(qd, kd, vd, gam, dyd, C, s0d, buf, dstate_in=buf)
    assert all(torch.equal(a, b) for a, b in zip(al, base))
    # and over state_in
    buf = s0d.clone()
    al = ret.chunkwise_backward_state(qd, kd, vd, gam, dyd, C, buf, dsod, dstate_in=buf)
    assert all(torch.equal(a, b) for a, b in zip(al, base))
    # no state at all: the same as chunkwise_backward, dS0 still returned
    dq, dkk, dvv, ds0 = ret.chunkwise_backward_state(qd, kd, vd, gam, dyd, C)
    plain = ret.chunkwise_backward(qd, kd, vd, gam, dyd, C)
    assert torch.equal(dq, plain[0]) and torch.equal(dkk, plain[1]) and torch.equal(dvv, plain[2])
    assert rel(ds0, oracle.backward(q, k, v, gam, dy)[3]) <= 2e-2
    # L = 0: dS0 = dS_out, zero without it
    e = torch.empty((B, H, 0, dk), dtype=dt, device="cuda")
    ev = torch.empty((B, H, 0, dv), dtype=dt, device="cuda")
    assert torch.equal(ret.chunkwise_backward_state(e, e, ev, gam, ev, C, s0d, dsod)[3], dsod)
    assert torch.count_nonzero(ret.chunkwise_backward_state(e, e, ev, gam, ev, C, s0d)[3]) == 0
    assert ret.device_status() == 0


def test_chunkwise_backward_state_chained_calls():
    # a sequence run as two calls with the state carried, differentiated call by
    # call from the end, gives the gradients of the whole sequence
    dt, B, H, L, dk, dv, C, cut = torch.bfloat16, 1, 2, 900, 128, 256, 128, 512
    q, k, v, dy, s0, dso = _state_grad_inputs(dt, B, H, L, dk, dv, 5)
    gam = inputs.multiscale_gammas(H)
    ref = oracle.backward(q, k, v, gam, dy, s0, dso)
    qd, kd, vd, dyd, s0d, dsod = dev(q, k, v, dy, s0, dso)
    parts = [slice(0, cut), slice(cut, L)]
    cont = lambda t, p: t[:, :, p].contiguous()  # noqa: E731
    _, s1 = ret.chunkwise(cont(qd, parts[0]), cont(kd, parts[0]), cont(vd, parts[0]), gam, C, state_in=s0d)
    g2 = ret.chunkwise_backward_state(cont(qd, parts[1]), cont(kd, parts[1]), cont(vd, parts[1]), gam,
                                      cont(dyd, parts[1]), C, s1, dsod)
    g1 = ret.chunkwise_backward_state(cont(qd, parts[0]), cont(kd, parts[0]), cont(vd, parts[0]), gam,
                                      cont(dyd, parts[0]), C, s0d, g2[3])
    assert ret.device_status() == 0
    for i in range(3):
        assert rel(torch.cat([g1[i], g2[i]], dim=2), ref[i]) <= 2e-2, i
    assert rel(g1[3], ref[3]) <= 2e-2


def test_chunkwise_backward_state_reused_segment_states():
    # 16 heads of dk 128, dv 256 over 2048 tokens in 64-row blocks: the dk sum
    # runs 8 segments and the dv sum 4, each of the dv sum's segments starting
    # from the transpose of the dk sum's scanned state at the same token.  dk_m
    # and dv_m need only the tokens n >= m, so the oracle's backward of the
    # window [512, 2048) (same dS_out) gives their exact rows there: rows of
    # three segments whose initial states came from the dk sum.
    B, H, L, dk, dv, C = 1, 16, 2048, 128, 256, 64
    q, k, v, dy, s0, dso = _state_grad_inputs(torch.bfloat16, B, H, L, dk, dv, 77)
    gam = inputs.multiscale_gammas(H)
    qd, kd, vd, dyd, s0d, dsod = dev(q, k, v, dy, s0, dso)
    _, dkk, dvv, _ = ret.chunkwise_backward_state(qd, kd, vd, gam, dyd, C, s0d, dsod)
    assert ret.device_status() == 0
    w0 = 512
    for h in (0, 9):
        sl = lambda t: t[:, h:h + 1, w0:]  # noqa: E731
        _, dk_r, dv_r, _ = oracle.backward(sl(q), sl(k), sl(v), gam[h:h + 1], sl(dy), None, dso[:, h:h + 1])
        assert rel(dkk[:, h:h + 1, w0:], dk_r) <= 2e-2, h
        assert rel(dvv[:, h:h + 1, w0:], dv_r) <= 2e-2, h


@pytest.mark.parametrize("B,H,L,dk,C,affine,gammas", [
    (2, 8, 2048, 64, 64, False, None),            # the MSR core, sequence split
    (1, 3, 1000, 128, 128, True, None),           # ragged tail, weight and bias
    (1, 2, 77, 64, 16, True, [0.5, 0.01]),        # gamma 0.01: the direct form; short blocks
])
def test_chunkwise_groupnorm_fused_epilogue(B, H, L, dk, C, affine, gammas):
    # dv = 128: one dv slice per head, so the chunkwise kernel normalises each
    # y row in its epilogue before the store (no second kernel); normalised
    # rows share one scale, so one relative bound covers every head
    dv = 128
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=L + 21)
    gam = inputs.multiscale_gammas(H) if gammas is None else torch.tensor(gammas)
    s_in = inputs.state(B, H, dk, dv, seed=22, scale=0.5)
    g = torch.Generator("cpu").manual_seed(23)
    w = torch.rand(H * dv, generator=g) + 0.5 if affine else None
    b = torch.randn(H * dv, generator=g) * 0.1 if affine else None
    y_ref, s_ref = oracle.recurrent(q, k, v, gam, s_in)
    z_ref = oracle.groupnorm(y_ref, eps=1e-5, weight=w, bias=b)
    qd, kd, vd, sd = dev(q, k, v, s_in)
    z, s = ret.chunkwise_groupnorm(qd, kd, vd, gam, C, 1e-5, weight=None if w is None else w.cuda(),
                                   bias=None if b is None else b.cuda(), state_in=sd)
    assert ret.device_status() == 0
    assert rel(z, z_ref) <= 2e-2 and rel(s, s_ref) <= 2e-2


@pytest.mark.parametrize("B,H,L,dk,dv,C", [
    (2, 8, 2048, 64, 128, 64),     # MSR core: sequence split, zeta on K's rows
    (8, 16, 1024, 64, 128, 64),    # 128 CTAs, no split
    (1, 4, 4096, 128, 256, 128),   # dk = 128, two dv slices, split
    (2, 4, 1024, 256, 512, 128),   # dk = 256 kernel
])
def test_chunkwise_cold_cache_repeatable(B, H, L, dk, dv, C):
    # Every call starts with q, k, v evicted from L2 (a 256 MB write), so the
    # first blocks' tiles arrive from DRAM as late as they can: an operand read
    # before its load has landed shows up as calls that differ from one another
    # or from the oracle.
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=31)
    gam = inputs.multiscale_gammas(H)
    y_ref, s_ref = oracle.recurrent(q, k, v, gam)
    qd, kd, vd = dev(q, k, v)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device="cuda")
    outs = []
    for _ in range(4):
        flush.fill_(1.0)
        outs.append(ret.chunkwise(qd, kd, vd, gam, C))
    torch.cuda.synchronize()
    assert ret.device_status() == 0
    for y, s in outs[1:]:
        assert torch.equal(y, outs[0][0]) and torch.equal(s, outs[0][1])
    assert rel(outs[0][0], y_ref) <= 2e-2 and rel(outs[0][1], s_ref) <= 2e-2


def test_chunkwise_groupnorm_unaligned_affine_takes_the_two_kernel_path():
    # weight and bias that are not 16-byte aligned cannot be read as float4 in
    # the fused epilogue: the call normalises in a second kernel instead, with
    # the same result
    B, H, L, dk, dv, C = 1, 2, 300, 64, 128, 64
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=41)
    gam = inputs.multiscale_gammas(H)
    g = torch.Generator("cpu").manual_seed(42)
    w = torch.rand(H * dv, generator=g) + 0.5
    b = torch.randn(H * dv, generator=g) * 0.1
    y_ref, s_ref = oracle.recurrent(q, k, v, gam)
    z_ref = oracle.groupnorm(y_ref, eps=1e-5, weight=w, bias=b)
    wd = torch.empty(H * dv + 1, device="cuda")[1:]
    bd = torch.empty(H * dv + 1, device="cuda")[1:]
    wd.copy_(w)
    bd.copy_(b)
    assert wd.data_ptr() % 16 != 0 and bd.data_ptr() % 16 != 0
    qd, kd, vd = dev(q, k, v)
    z, s = ret.chunkwise_groupnorm(qd, kd, vd, gam, C, 1e-5, weight=wd, bias=bd)
    assert rel(z, z_ref) <= 2e-2 and rel(s, s_ref) <= 2e-2
