"""Failure detection without a GPU fault: a chunkwise call whose K load for one
block is never issued (host-set fault injection) must end its bounded wait,
tear down cleanly and report RET_ETIMEOUT; the context stays usable and the
next call is correct."""
import pytest
import torch

import oracle
import retnet_retention_chunkwise_b200 as ret
from retnet_retention_chunkwise_b200 import _abi, inputs
from tests.parity import rel

pytestmark = pytest.mark.gpu




@pytest.mark.parametrize("dk,dv,C", [(128, 128, 128), (256, 256, 128), (128, 128, 256)])
def test_dropped_load_times_out_then_recovers(monkeypatch, dk, dv, C):
    B, H, L = 1, 2, 640
    q, k, v = inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed=31)
    gam = inputs.multiscale_gammas(H)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    assert ret.device_status() == _abi.RET_OK
    monkeypatch.setenv("RETENTION_WAIT_LIMIT_MS", "100")
    monkeypatch.setenv("RETENTION_DEBUG_DROP_BLOCK", "2")
    ret.chunkwise(qd, kd, vd, gam, C, workspace=None)  # launches; the wait for block 2 expires
    assert ret.device_status() == _abi.RET_ETIMEOUT
    assert ret.device_status() == _abi.RET_OK  # the status word was cleared
    monkeypatch.delenv("RETENTION_DEBUG_DROP_BLOCK")
    y, s = ret.chunkwise(qd, kd, vd, gam, C, workspace=None)
    assert ret.device_status() == _abi.RET_OK
    y_ref, s_ref = oracle.recurrent(q, k, v, gam)
    assert rel(y, y_ref) <= 2e-2 and rel(s, s_ref) <= 2e-2
