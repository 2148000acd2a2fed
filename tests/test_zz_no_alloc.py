"""The allocation-free chunkwise entry point (retention_chunkwise_static_ws).

Some callers cannot allocate device memory (a graph being captured, runtimes
with a fixed memory plan, hosts that own all device memory), so the library
offers a chunkwise call whose sequence-split scratch is a fixed array inside
the library.  This file checks, through the C ABI, that its results match the
regular entry point (which gets a caller-provided workspace) on two calls in a
row (bit for bit: both run the same kernels with the same sequence split),
that both match the fp64 oracle, and that a shape needing more scratch than
the array holds is refused before anything is launched.

The file name makes pytest collect it last.
"""
import ctypes

import pytest
import torch

import oracle
from retnet_retention_chunkwise_b200 import _abi, inputs
from tests.parity import rel

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the bf16 bound of the other parity tests


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.fixture(scope="module")
def lib():
    return _abi.load()


def _case(seed, B=1, H=2, L=4096, dk=64, dv=128):
    q, k, v = (t.cuda() for t in inputs.qkv(B, H, L, dk, dv, torch.bfloat16, seed))
    s_in = inputs.state(B, H, dk, dv, seed=seed + 1, scale=0.5).cuda()
    return q, k, v, s_in


def test_static_scratch_matches_regular_entry_point_twice(lib):
    B, H, L, dk, dv, C = 1, 2, 4096, 64, 128, 64
    shape = _abi.RetShape(B, H, L, dk, dv)
    need = lib.retention_chunkwise_workspace_bytes(C, shape, _abi.RET_BF16)
    assert 0 < need <= _abi.STATIC_WS_BYTES  # this shape uses the split and fits the array
    gam = (ctypes.c_float * H)(*inputs.multiscale_gammas(H).tolist())
    ws = torch.empty(need // 4, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (3, 4):  # two calls in a row, different data
        q, k, v, s_in = _case(seed, B, H, L, dk, dv)
        y_or, s_or = oracle.recurrent(q.cpu(), k.cpu(), v.cpu(), inputs.multiscale_gammas(H), s_in.cpu())
        y_ref, s_ref = torch.empty_like(v), torch.empty_like(s_in)
        y, s = torch.empty_like(v), torch.empty_like(s_in)
        rc = lib.retention_chunkwise(_ptr(q), _ptr(k), _ptr(v), gam, _ptr(y_ref), _ptr(s_in), _ptr(s_ref), C,
                                     shape, _abi.RET_BF16, _ptr(ws), need, stream)
        assert rc == _abi.RET_OK
        rc = lib.retention_chunkwise_static_ws(_ptr(q), _ptr(k), _ptr(v), gam, _ptr(y), _ptr(s_in), _ptr(s), C,
                                               shape, _abi.RET_BF16, stream)
        assert rc == _abi.RET_OK
        torch.cuda.synchronize()
        assert lib.retention_get_device_status(stream) == _abi.RET_OK
        assert torch.equal(y, y_ref) and torch.equal(s, s_ref)
        assert rel(y, y_or) <= TOL and rel(s, s_or) <= TOL


def test_static_scratch_shape_without_split(lib):
    B, H, L, dk, dv, C = 4, 8, 512, 256, 512, 128  # 128 (b, h, dv-slice) CTAs: no split is planned
    shape = _abi.RetShape(B, H, L, dk, dv)
    assert lib.retention_chunkwise_workspace_bytes(C, shape, _abi.RET_BF16) == 0
    gam = (ctypes.c_float * H)(*inputs.multiscale_gammas(H).tolist())
    q, k, v, s_in = _case(7, B, H, L, dk, dv)
    y_ref, s_ref, y, s = torch.empty_like(v), torch.empty_like(s_in), torch.empty_like(v), torch.empty_like(s_in)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.retention_chunkwise(_ptr(q), _ptr(k), _ptr(v), gam, _ptr(y_ref), _ptr(s_in), _ptr(s_ref), C, shape,
                                   _abi.RET_BF16, None, 0, stream) == _abi.RET_OK
    assert lib.retention_chunkwise_static_ws(_ptr(q), _ptr(k), _ptr(v), gam, _ptr(y), _ptr(s_in), _ptr(s), C, shape,
                                             _abi.RET_BF16, stream) == _abi.RET_OK
    torch.cuda.synchronize()
    assert lib.retention_get_device_status(stream) == _abi.RET_OK
    assert torch.equal(y, y_ref) and torch.equal(s, s_ref)
    y_or, s_or = oracle.recurrent(q.cpu(), k.cpu(), v.cpu(), inputs.multiscale_gammas(H), s_in.cpu())
    assert rel(y, y_or) <= TOL and rel(s, s_or) <= TOL


def test_static_scratch_refuses_oversize_split(lib):
    # one head of dk=256, dv=256 over 64K tokens splits into ~74 segments of
    # 256 KiB each: more than the fixed array holds
    shape = _abi.RetShape(1, 1, 65536, 256, 256)
    assert lib.retention_chunkwise_workspace_bytes(128, shape, _abi.RET_BF16) > _abi.STATIC_WS_BYTES
    gam = (ctypes.c_float * 1)(0.99)
    # NULL tensors: the size check refuses the call first; were it ever to let
    # the call through, the NULL check would still stop it before any launch
    rc = lib.retention_chunkwise_static_ws(None, None, None, gam, None, None, None, 128, shape, _abi.RET_BF16, None)
    assert rc == _abi.RET_EUNSUPPORTED
