"""The kernels built with index checks (-DRET_BOUNDS_CHECK, libretention_bc.so)
on small ragged cases.  A check that fails skips its access and sets the device
status to RET_EBOUNDS, with the site of the first failure kept for the report.
compute-sanitizer is not available on the test machines; this build is the
stand-in: every shared-memory tile row, TMEM column range, global output row
and state index the kernels compute at run time is checked, on shapes that
reach the ragged tails, blocks shorter than 32 rows, blocks of 129..256 rows,
the sequence split, the direct decay form and the anti-causal sums of the
backward pass.  The cases run in a child process that loads the checked
library (RETENTION_LIBRARY), and the results are also held to the oracle."""
import os
import subprocess
import sys

import pytest

from retnet_retention_chunkwise_b200 import build as _build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import ctypes, sys, math
sys.path.insert(0, sys.argv[1])
import torch
import oracle
import retnet_retention_chunkwise_b200 as ret
from retnet_retention_chunkwise_b200 import inputs
from tests.parity import rel
lib = ret.library()
site = lib.retention_debug_bounds_site
site.restype = ctypes.c_uint
fails = []

def check(name, got, ref, tol=2e-2):
    st = ret.device_status()
    s = site()
    e = max(rel(g, r) for g, r in zip(got, ref))
    if st != 0 or s != 0 or not e <= tol:
        fails.append((name, st, s, e))

for (B, H, L, dk, dv, C) in [(1, 2, 333, 64, 128, 48), (1, 2, 200, 128, 256, 64), (1, 1, 77, 256, 128, 16),
                             (1, 2, 700, 256, 256, 128), (1, 1, 520, 128, 128, 144), (1, 2, 600, 64, 128, 256),
                             (1, 2, 4096, 128, 128, 128), (1, 1, 1, 64, 128, 16)]:
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=L)
    for gam in ([0.97, 0.999][:H], [0.5, 0.0][:H]):
        g = torch.tensor(gam)
        s_in = inputs.state(B, H, dk, dv, seed=3, scale=0.5)
        y_ref, s_ref = oracle.recurrent(q, k, v, g, s_in)
        y, s = ret.chunkwise(q.cuda(), k.cuda(), v.cuda(), g, C, state_in=s_in.cuda())
        check(f"chunkwise {B},{H},{L},{dk},{dv},{C} {gam}", (y, s), (y_ref, s_ref))
        if C <= 128 and L > 1:
            check(f"parallel {L},{dk},{dv} {gam}", (ret.parallel(q.cuda(), k.cuda(), v.cuda(), g),),
                  (oracle.recurrent(q, k, v, g)[0],))
            sd = ret.chunkwise_state(k.cuda(), v.cuda(), g, C, state_in=s_in.cuda())
            check(f"state-only {L},{dk},{dv},{C} {gam}", (sd,), (s_ref,))

# the backward pass: its dk and dv are the anti-causal sums
for (B, H, L, dk, dv, C) in [(1, 2, 700, 128, 256, 128), (1, 2, 300, 256, 128, 64), (1, 1, 600, 128, 128, 256),
                             (1, 2, 2304, 128, 128, 128)]:
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=L + 1)
    gg = torch.Generator("cpu").manual_seed(L)
    dy = (torch.randn((B, H, L, dv), generator=gg) / math.sqrt(dv)).to(torch.bfloat16)
    s0 = torch.randn((B, H, dk, dv), generator=gg) / math.sqrt(dk)
    dso = torch.randn((B, H, dk, dv), generator=gg) / math.sqrt(dv)
    g = inputs.multiscale_gammas(H)
    ref = oracle.backward(q, k, v, g, dy, s0, dso)
    got = ret.chunkwise_backward_state(q.cuda(), k.cuda(), v.cuda(), g, dy.cuda(), C, s0.cuda(), dso.cuda())
    check(f"chunkwise backward {L},{dk},{dv},{C}", got, ref)
    if C <= 128:
        got = ret.parallel_backward(q.cuda(), k.cuda(), v.cuda(), g, dy.cuda())
        check(f"parallel backward {L},{dk},{dv}", got, oracle.parallel_backward(q, k, v, g, dy))

# decode and GroupNorm with the gate, ragged widths
q, k, v = inputs.qkv(2, 3, 1, 128, 96, torch.bfloat16, seed=5)
st0 = inputs.state(2, 3, 128, 96, seed=6)
g = inputs.multiscale_gammas(3)
y_ref, s_ref = oracle.recurrent(q, k, v, g, st0)
state = st0.cuda()
y = ret.recurrent_step(q.cuda(), k.cuda(), v.cuda(), g, state)
check("decode", (y, state), (y_ref, s_ref))
yy = torch.randn((2, 3, 37, 96)).to(torch.bfloat16)
gate = torch.randn((2, 3, 37, 96)).to(torch.bfloat16)
z = ret.groupnorm(yy.cuda(), 1e-5, gate=gate.cuda(), act="swish")
check("groupnorm gated", (z,), (oracle.gate(oracle.groupnorm(yy, eps=1e-5), gate, "swish"),))
print("FAILS", fails)
sys.exit(1 if fails else 0)
'''


def test_bounds_checked_build_on_ragged_cases():
    lib = _build.LIB_BOUNDS_CHECK
    if not os.path.exists(lib):
        pytest.fail("libretention_bc.so is missing: build it with `python -m retnet_retention_chunkwise_b200.build "
                    "--bounds-check` (the __graft_entry__ build does)")
    env = dict(os.environ, RETENTION_LIBRARY=lib)
    out = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-4000:] + out.stderr[-4000:]
