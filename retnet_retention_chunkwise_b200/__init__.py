"""retnet_retention_chunkwise_b200 -- the retention contraction of Multi-Scale
Retention (RetNet) on NVIDIA B200 (sm_100a).

    y_n = sum_{m<=n} gamma_h^(n-m) (q_n . k_m) v_m  (+ gamma_h^(n+1) q_n S_in)

in its parallel, chunkwise and recurrent forms (page "Retentive Networks --
Microsoft Propone l'Alternativa Architetturale ai Transformer", section "Il
meccanismo: Multi-Scale Retention").  The work is done by the hand-written
CUDA kernels of ``libretention.so`` behind the C ABI of ``include/retention.h``;
this module only checks tensors and marshals pointers (PyTorch supplies device
memory and the current stream).  There is no CPU path: without the compiled
library every call raises.

Tensors: q, k [B, H, L, dk]; v [B, H, L, dv]; state fp32 [B, H, dk, dv]; all
contiguous CUDA tensors; bf16 (tensor-core path) or fp32 (CUDA-core path).
``gamma`` is a host sequence / CPU tensor of H values in [0, 1].
"""
from __future__ import annotations

import ctypes
import threading

import torch

from . import _abi

__all__ = ["parallel", "chunkwise", "chunkwise_host", "recurrent_step", "groupnorm", "chunkwise_groupnorm",
           "parallel_backward", "chunkwise_backward", "chunkwise_backward_state", "chunkwise_state",
           "state_fold", "device_status",
           "workspace_bytes", "RetentionError", "library"]

_LIB = None
_LOCK = threading.Lock()


class RetentionError(RuntimeError):
    """A libretention call returned a status other than RET_OK."""

    def __init__(self, status: int, where: str):
        name = library().retention_status_str(status).decode()
        super().__init__(f"{where}: {name}")
        self.status = status


def library() -> ctypes.CDLL:
    """The loaded libretention.so (raises ImportError if it was not built)."""
    global _LIB
    if _LIB is None:
        with _LOCK:
            if _LIB is None:
                _LIB = _abi.load()
    return _LIB


def _check(rc: int, where: str):
    if rc != _abi.RET_OK:
        raise RetentionError(rc, where)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _abi.RET_BF16
    if t.dtype == torch.float32:
        return _abi.RET_F32
    raise TypeError(f"retention: unsupported dtype {t.dtype} (bf16 or fp32)")


def _cuda(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"retention: {name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"retention: {name} must be contiguous")


def _gamma(gamma, H: int):
    if isinstance(gamma, torch.Tensor):
        if gamma.is_cuda:
            raise ValueError("retention: gamma must be on the host (it is read at launch)")
        g = gamma.detach().to(torch.float32).reshape(-1).tolist()
    else:
        g = [float(x) for x in gamma]
    if len(g) != H:
        raise ValueError(f"retention: gamma has {len(g)} values for {H} heads")
    return (ctypes.c_float * H)(*g)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shape(q, v):
    B, H, L, dk = q.shape
    return _abi.RetShape(B, H, L, dk, v.shape[-1])


def _qkv(q, k, v):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda(t, n)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("retention: expected q, k [B,H,L,dk] and v [B,H,L,dv]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("retention: q, k, v must share a dtype")
    return _dtype(q)


def parallel(q, k, v, gamma, *, out=None):
    """Parallel form: y = (Q K^T (.) D) V per head.  Returns y [B,H,L,dv]."""
    dt = _qkv(q, k, v)
    s = _shape(q, v)
    y = out if out is not None else torch.empty(v.shape, dtype=v.dtype, device=v.device)
    _cuda(y, "out")
    _check(library().retention_parallel(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(y), s, dt,
                                        _stream()), "retention_parallel")
    return y


_WS = {}


def workspace_bytes(chunk: int, B: int, H: int, L: int, dk: int, dv: int,
                    dtype: torch.dtype = torch.bfloat16) -> int:
    """Scratch bytes that let the chunkwise call split long sequences across CTAs."""
    code = _abi.RET_BF16 if dtype == torch.bfloat16 else _abi.RET_F32
    return int(library().retention_chunkwise_workspace_bytes(chunk, _abi.RetShape(B, H, L, dk, dv), code))


def _workspace(nbytes: int, device):
    if nbytes == 0:
        return None
    key = (device.index if device.index is not None else torch.cuda.current_device())
    ws = _WS.get(key)
    if ws is None or ws.numel() * 4 < nbytes:
        ws = torch.empty((nbytes + 3) // 4, dtype=torch.float32, device=device)
        _WS[key] = ws
    return ws


def chunkwise(q, k, v, gamma, chunk: int, *, state_in=None, state_out=None, return_state=True,
              out=None, workspace="auto"):
    """Chunkwise form with block length ``chunk``.

    Returns (y, state_out).  ``state_in`` (fp32 [B,H,dk,dv], optional) is the
    state before the first token; ``state_out`` may be given (it may be the same
    tensor as ``state_in``) or is allocated when ``return_state``.
    ``workspace`` (CUDA tensor) enables the sequence split; the default "auto"
    uses a cached buffer of ``workspace_bytes(...)``; None runs without one.
    """
    dt = _qkv(q, k, v)
    s = _shape(q, v)
    y = out if out is not None else torch.empty(v.shape, dtype=v.dtype, device=v.device)
    _cuda(y, "out")
    sshape = (s.B, s.H, s.dk, s.dv)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        if t is not None:
            _cuda(t, n)
            if t.dtype != torch.float32 or tuple(t.shape) != sshape:
                raise ValueError(f"retention: {n} must be fp32 {sshape}")
    if state_out is None and return_state:
        state_out = torch.empty(sshape, dtype=torch.float32, device=q.device)
    if isinstance(workspace, str):
        workspace = _workspace(int(library().retention_chunkwise_workspace_bytes(chunk, s, dt)), q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(library().retention_chunkwise(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(y),
                                         _ptr(state_in), _ptr(state_out), int(chunk), s, dt,
                                         _ptr(workspace), wbytes, _stream()), "retention_chunkwise")
    return y, state_out


def chunkwise_host(q, k, v, gamma, chunk: int, *, dev=None, out=None, state_in=None, state_out=None,
                   workspace="auto", n_groups: int = 0):
    """Chunkwise form on host tensors: q, k, v are copied to the device, the form
    runs there and y comes back to ``out`` (a host tensor, page-locked if it is
    allocated here), with the copies of the two directions and the kernels of
    successive (b, h) groups overlapped by the library (retention_chunkwise_host).

    ``dev`` = (q_dev, k_dev, v_dev, y_dev) CUDA tensors of the same shapes, or
    None to allocate them.  ``state_in`` / ``state_out`` are CUDA fp32 tensors as
    for :func:`chunkwise`.  Returns (y_host, state_out).  The call is
    asynchronous on the current stream: synchronise before reading y_host.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"retention: {n} must be a contiguous host tensor")
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("retention: expected q, k [B,H,L,dk] and v [B,H,L,dv]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("retention: q, k, v must share a dtype")
    dt = _dtype(q)
    s = _shape(q, v)
    device = torch.device("cuda", torch.cuda.current_device())
    if out is None:
        out = torch.empty(v.shape, dtype=v.dtype).pin_memory()
    if out.is_cuda or tuple(out.shape) != tuple(v.shape) or out.dtype != v.dtype or not out.is_contiguous():
        raise ValueError("retention: out must be a contiguous host tensor shaped like v")
    if dev is None:
        dev = tuple(torch.empty(t.shape, dtype=t.dtype, device=device) for t in (q, k, v, v))
    for t, h, n in zip(dev, (q, k, v, v), ("q_dev", "k_dev", "v_dev", "y_dev")):
        _cuda(t, n)
        if tuple(t.shape) != tuple(h.shape) or t.dtype != h.dtype:
            raise ValueError(f"retention: {n} must match its host tensor")
    sshape = (s.B, s.H, s.dk, s.dv)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        if t is not None:
            _cuda(t, n)
            if t.dtype != torch.float32 or tuple(t.shape) != sshape:
                raise ValueError(f"retention: {n} must be fp32 {sshape}")
    if isinstance(workspace, str):
        workspace = _workspace(int(library().retention_chunkwise_host_workspace_bytes(chunk, s, dt, n_groups)),
                               device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(library().retention_chunkwise_host(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(out),
                                              *(_ptr(t) for t in dev), _ptr(state_in), _ptr(state_out),
                                              int(chunk), s, dt, _ptr(workspace), wbytes, int(n_groups),
                                              _stream()), "retention_chunkwise_host")
    return out, state_out


def _gn_params(weight, bias, H: int, dv: int, device):
    for t, n in ((weight, "weight"), (bias, "bias")):
        if t is not None:
            _cuda(t, n)
            if t.dtype != torch.float32 or t.numel() != H * dv or t.device != device:
                raise ValueError(f"retention: {n} must be fp32 with H*dv values on the device of y")


def groupnorm(y, eps: float = 1e-5, *, weight=None, bias=None, out=None, gate=None, act: str = "swish"):
    """Per-head group normalisation of y [B,H,L,dv]: each (b, h, n) row of dv
    values by its own mean and biased variance, then ``* weight + bias`` per
    channel (fp32 [H*dv] CUDA tensors, optional).  ``out`` may be ``y``.

    With ``gate`` (y's shape and dtype) the result is multiplied by
    ``act(gate)``, act one of "none", "swish", "sigmoid" (retention_groupnorm_gated)."""
    _cuda(y, "y")
    dt = _dtype(y)
    if y.dim() != 4:
        raise ValueError("retention: y must be [B,H,L,dv]")
    B, H, L, dv = y.shape
    out = out if out is not None else torch.empty_like(y)
    _cuda(out, "out")
    if out.shape != y.shape or out.dtype != y.dtype:
        raise ValueError("retention: out must match y")
    _gn_params(weight, bias, H, dv, y.device)
    s = _abi.RetShape(B, H, L, 1, dv)
    if gate is None:
        _check(library().retention_groupnorm(_ptr(y), _ptr(out), float(eps), _ptr(weight), _ptr(bias), s, dt,
                                             _stream()), "retention_groupnorm")
        return out
    _cuda(gate, "gate")
    if gate.shape != y.shape or gate.dtype != y.dtype:
        raise ValueError("retention: gate must match y")
    if act not in _abi.GATE_ACTS:
        raise ValueError(f"retention: act must be one of {sorted(_abi.GATE_ACTS)}")
    _check(library().retention_groupnorm_gated(_ptr(y), _ptr(gate), _ptr(out), float(eps), _ptr(weight),
                                               _ptr(bias), _abi.GATE_ACTS[act], s, dt, _stream()),
           "retention_groupnorm_gated")
    return out


def chunkwise_groupnorm(q, k, v, gamma, chunk: int, eps: float = 1e-5, *, weight=None, bias=None,
                        state_in=None, state_out=None, return_state=True, out=None, workspace="auto",
                        gate=None, act: str = "swish"):
    """Chunkwise form followed by the per-head group normalisation of its output
    (see :func:`groupnorm`), and with ``gate`` (v's shape and dtype) the output
    gate act(gate).  Returns (normalised y, state_out).  bf16 with dv = 128,
    dk <= 128, chunk <= 128 and no gate normalise in the chunkwise kernel's
    epilogue; otherwise the normalisation is a second kernel on the stream."""
    dt = _qkv(q, k, v)
    s = _shape(q, v)
    y = out if out is not None else torch.empty(v.shape, dtype=v.dtype, device=v.device)
    _cuda(y, "out")
    sshape = (s.B, s.H, s.dk, s.dv)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        if t is not None:
            _cuda(t, n)
            if t.dtype != torch.float32 or tuple(t.shape) != sshape:
                raise ValueError(f"retention: {n} must be fp32 {sshape}")
    if state_out is None and return_state:
        state_out = torch.empty(sshape, dtype=torch.float32, device=q.device)
    _gn_params(weight, bias, s.H, s.dv, q.device)
    if isinstance(workspace, str):
        workspace = _workspace(int(library().retention_chunkwise_gn_workspace_bytes(chunk, s, dt)), q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if gate is None:
        _check(library().retention_chunkwise_gn(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(y),
                                                _ptr(state_in), _ptr(state_out), int(chunk), s, dt, float(eps),
                                                _ptr(weight), _ptr(bias), _ptr(workspace), wbytes, _stream()),
               "retention_chunkwise_gn")
        return y, state_out
    _cuda(gate, "gate")
    if gate.shape != v.shape or gate.dtype != v.dtype:
        raise ValueError("retention: gate must match v")
    if act not in _abi.GATE_ACTS:
        raise ValueError(f"retention: act must be one of {sorted(_abi.GATE_ACTS)}")
    _check(library().retention_chunkwise_gn_gated(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(y),
                                                  _ptr(state_in), _ptr(state_out), int(chunk), s, dt, float(eps),
                                                  _ptr(weight), _ptr(bias), _ptr(gate), _abi.GATE_ACTS[act],
                                                  _ptr(workspace), wbytes, _stream()),
           "retention_chunkwise_gn_gated")
    return y, state_out


def parallel_backward(q, k, v, gamma, dy, *, workspace=None):
    """Gradients (dq, dk, dv) of :func:`parallel` for the upstream gradient dy
    (retention_parallel_backward).  ``workspace``: a CUDA tensor of at least
    ``retention_parallel_backward_workspace_bytes`` bytes, or None to allocate."""
    dt = _qkv(q, k, v)
    _cuda(dy, "dy")
    if dy.shape != v.shape or dy.dtype != v.dtype:
        raise ValueError("retention: dy must match v")
    s = _shape(q, v)
    need = int(library().retention_parallel_backward_workspace_bytes(s, dt))
    if workspace is None:
        workspace = torch.empty((need + 3) // 4, dtype=torch.float32, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    _check(library().retention_parallel_backward(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(dy),
                                                 _ptr(dq), _ptr(dk), _ptr(dv), s, dt, _ptr(workspace), wbytes,
                                                 _stream()), "retention_parallel_backward")
    return dq, dk, dv


def chunkwise_backward(q, k, v, gamma, dy, chunk: int, *, workspace=None):
    """Gradients (dq, dk, dv) of :func:`chunkwise` from a zero state, for the
    upstream gradient dy of y, through the chunkwise form (cost linear in L;
    retention_chunkwise_backward)."""
    dt = _qkv(q, k, v)
    _cuda(dy, "dy")
    if dy.shape != v.shape or dy.dtype != v.dtype:
        raise ValueError("retention: dy must match v")
    s = _shape(q, v)
    need = int(library().retention_chunkwise_backward_workspace_bytes(int(chunk), s, dt))
    if workspace is None:
        workspace = torch.empty((need + 3) // 4, dtype=torch.float32, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    _check(library().retention_chunkwise_backward(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(dy),
                                                  _ptr(dq), _ptr(dk), _ptr(dv), int(chunk), s, dt, _ptr(workspace),
                                                  wbytes, _stream()), "retention_chunkwise_backward")
    return dq, dk, dv


def chunkwise_backward_state(q, k, v, gamma, dy, chunk: int, state_in=None, dstate_out=None, *,
                             dstate_in=None, workspace=None):
    """Gradients (dq, dk, dv, dstate_in) of :func:`chunkwise` started from
    ``state_in`` (None: zero), for upstream gradients dy of y and
    ``dstate_out`` of its state_out (None: unused); retention_chunkwise_backward_state.

    ``dstate_in`` may be given as the output buffer (fp32 [B,H,dk,dv]); it may be
    the same tensor as ``dstate_out``."""
    dt = _qkv(q, k, v)
    _cuda(dy, "dy")
    if dy.shape != v.shape or dy.dtype != v.dtype:
        raise ValueError("retention: dy must match v")
    s = _shape(q, v)
    for name, t in (("state_in", state_in), ("dstate_out", dstate_out), ("dstate_in", dstate_in)):
        if t is not None:
            _cuda(t, name)
            if t.dtype != torch.float32 or tuple(t.shape) != (s.B, s.H, s.dk, s.dv) or not t.is_contiguous():
                raise ValueError(f"retention: {name} must be contiguous fp32 [B,H,dk,dv]")
    if dstate_in is None:
        dstate_in = torch.empty((s.B, s.H, s.dk, s.dv), dtype=torch.float32, device=q.device)
    need = int(library().retention_chunkwise_backward_state_workspace_bytes(int(chunk), s, dt))
    if workspace is None:
        workspace = torch.empty((need + 3) // 4, dtype=torch.float32, device=q.device)
    wbytes = workspace.numel() * workspace.element_size()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    _check(library().retention_chunkwise_backward_state(
        _ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(dy), _ptr(state_in), _ptr(dstate_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dstate_in),
        int(chunk), s, dt, _ptr(workspace), wbytes, _stream()), "retention_chunkwise_backward_state")
    return dq, dk, dv, dstate_in


def chunkwise_state(k, v, gamma, chunk: int, *, state_in=None, out=None, workspace=None):
    """The state_out of :func:`chunkwise` on (k, v) without computing y:
    gamma^L state_in + sum_t gamma^(L-1-t) k_t^T v_t, fp32 [B,H,dk,dv]
    (retention_chunkwise_state)."""
    _cuda(k, "k")
    _cuda(v, "v")
    dt = _dtype(k)
    if v.dtype != k.dtype or k.dim() != 4 or v.dim() != 4 or k.shape[:3] != v.shape[:3]:
        raise ValueError("retention: k [B,H,L,dk] and v [B,H,L,dv] must match in dtype and B, H, L")
    s = _shape(k, v)
    shape = (s.B, s.H, s.dk, s.dv)
    for name, t in (("state_in", state_in), ("out", out)):
        if t is not None:
            _cuda(t, name)
            if t.dtype != torch.float32 or tuple(t.shape) != shape:
                raise ValueError(f"retention: {name} must be fp32 [B,H,dk,dv]")
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=k.device)
    need = int(library().retention_chunkwise_state_workspace_bytes(int(chunk), s, dt))
    if workspace is None and need > 0:
        workspace = torch.empty((need + 3) // 4, dtype=torch.float32, device=k.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(library().retention_chunkwise_state(_ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(state_in), _ptr(out),
                                               int(chunk), s, dt, _ptr(workspace), wbytes, _stream()),
           "retention_chunkwise_state")
    return out


def state_fold(parts, lens, gamma, *, state_in=None, out=None):
    """The state after consecutive runs from the runs' own sums: S = state_in,
    then S = gamma^len_i S + parts[i] for each run i (retention_state_fold).

    parts: fp32 CUDA tensor [n,B,H,dk,dv]; lens: n run lengths (ints)."""
    _cuda(parts, "parts")
    if parts.dtype != torch.float32 or parts.dim() != 5:
        raise ValueError("retention: parts must be fp32 [n,B,H,dk,dv]")
    n, B, H, dk, dv = parts.shape
    lens = [int(x) for x in lens]
    if len(lens) != n:
        raise ValueError("retention: one length per part")
    shape = (B, H, dk, dv)
    for name, t in (("state_in", state_in), ("out", out)):
        if t is not None:
            _cuda(t, name)
            if t.dtype != torch.float32 or tuple(t.shape) != shape:
                raise ValueError(f"retention: {name} must be fp32 [B,H,dk,dv]")
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=parts.device)
    c_lens = (ctypes.c_int * max(n, 1))(*lens)
    _check(library().retention_state_fold(_ptr(parts) if n > 0 else None, c_lens, n, _gamma(gamma, H),
                                          _ptr(state_in), _ptr(out), _abi.RetShape(B, H, 0, dk, dv), _stream()),
           "retention_state_fold")
    return out


def recurrent_step(q, k, v, gamma, state, *, out=None):
    """One decode step in place on ``state``: S <- gamma S + k^T v, y = q S.

    q, k [B,H,1,dk], v [B,H,1,dv]; state fp32 [B,H,dk,dv].  Returns y [B,H,1,dv].
    """
    dt = _qkv(q, k, v)
    if q.shape[2] != 1:
        raise ValueError("retention: recurrent_step takes one token (L == 1)")
    s = _shape(q, v)
    _cuda(state, "state")
    if state.dtype != torch.float32 or tuple(state.shape) != (s.B, s.H, s.dk, s.dv):
        raise ValueError("retention: state must be fp32 [B,H,dk,dv]")
    y = out if out is not None else torch.empty(v.shape, dtype=v.dtype, device=v.device)
    _cuda(y, "out")
    _check(library().retention_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _gamma(gamma, s.H), _ptr(y),
                                              _ptr(state), s, dt, _stream()), "retention_recurrent_step")
    return y


def device_status() -> int:
    """Synchronise the current stream; return (and clear) the device status code."""
    return int(library().retention_get_device_status(_stream()))
