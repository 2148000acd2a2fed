"""fp64 CPU oracle for the retention contraction -- test infrastructure only.

This package is the checker: ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are its only
callers.  The product path (``retnet_retention_chunkwise_b200``) never imports
it, and it imports nothing from there.

The arithmetic lives in ``retention_oracle.c`` (plain C, fp64, one thread per
(batch, head) pair); this module only compiles it with gcc and marshals numpy
arrays.  Each C function cites the passage it follows:

* ``recurrent``  -- S_n = gamma S_{n-1} + k_n^T v_n, y_n = q_n S_n (the
  definition; page "Retentive Networks -- Microsoft Propone l'Alternativa
  Architetturale ai Transformer", section "Il meccanismo: Multi-Scale
  Retention").
* ``parallel``   -- the double sum y_n = sum_{m<=n} gamma^(n-m) (q_n.k_m) v_m
  (same section), plus gamma^(n+1) q_n S_in for a carried-in state.
* ``chunkwise``  -- the block form of the same section, derived by splitting
  the sum at each block start.
* ``parallel_backward`` -- dq, dk, dv of the parallel form for an upstream dy:
  the chain rule on each term of the definition's double sum (the pages give
  no backward pass).
* ``groupnorm``  -- one normalisation group per head over its dv values (author
  responses on paperhub.cn, reply on GroupNorm vs LayerNorm), mean and biased
  variance per (b, h, n), optional per-channel affine.

Inputs are float64 numpy arrays (bf16 or fp32 values widen to fp64 exactly).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "retention_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")

_lib = None


def build(src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile the C oracle with gcc (-O2, no fast-math: IEEE fp64)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
           "-fno-fast-math", "-ffp-contract=off", *extra_flags, src, "-o", out, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build() -> bool:
    return (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)


def load(path: str | None = None):
    """Load (building first if stale) the oracle library and declare signatures."""
    global _lib
    if path is None:
        if _lib is not None:
            return _lib
        if _needs_build():
            build()
        path = _LIB
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.oracle_recurrent.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp, i]
    lib.oracle_parallel.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp, i]
    lib.oracle_chunkwise.argtypes = [i, i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp, i]
    lib.oracle_groupnorm.argtypes = [i, i, i, i, dp, ctypes.c_double, dp, dp, dp]
    lib.oracle_parallel_backward.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp, dp]
    lib.oracle_state_backward.argtypes = [i, i, i, i, i] + [dp] * 11
    lib.oracle_gate.argtypes = [ctypes.c_long, dp, dp, i, dp]
    for f in (lib.oracle_recurrent, lib.oracle_parallel, lib.oracle_chunkwise, lib.oracle_groupnorm,
              lib.oracle_parallel_backward, lib.oracle_state_backward, lib.oracle_gate):
        f.restype = ctypes.c_int
    if path == _LIB:
        _lib = lib
    return lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor -> exact fp64 copy
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _run(form: str, q, k, v, gamma, state_in=None, chunk: int = 0,
         nthreads: int = 0, lib=None):
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    gamma = _f64(gamma).reshape(-1)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or gamma.shape[0] != H:
        raise ValueError("oracle: shape mismatch")
    s_in = _f64(state_in)
    if s_in is not None and s_in.shape != (B, H, dk, dv):
        raise ValueError("oracle: state_in must be [B,H,dk,dv]")
    y = np.zeros((B, H, L, dv), dtype=np.float64)
    s_out = np.zeros((B, H, dk, dv), dtype=np.float64)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(s_in), _ptr(y), _ptr(s_out), int(nthreads))
    if form == "recurrent":
        rc = lib.oracle_recurrent(B, H, L, dk, dv, *args)
    elif form == "parallel":
        rc = lib.oracle_parallel(B, H, L, dk, dv, *args)
    elif form == "chunkwise":
        rc = lib.oracle_chunkwise(B, H, L, dk, dv, int(chunk), *args)
    else:
        raise ValueError(form)
    if rc != 0:
        raise ValueError(f"oracle_{form}: invalid arguments")
    return y, s_out


def recurrent(q, k, v, gamma, state_in=None, nthreads: int = 0, lib=None):
    """Recurrent definition in fp64.  Returns (y [B,H,L,dv], state_out [B,H,dk,dv])."""
    return _run("recurrent", q, k, v, gamma, state_in, 0, nthreads, lib)


def parallel(q, k, v, gamma, state_in=None, nthreads: int = 0, lib=None):
    """Double-sum (parallel) form in fp64.  Same outputs as :func:`recurrent`."""
    return _run("parallel", q, k, v, gamma, state_in, 0, nthreads, lib)


def chunkwise(q, k, v, gamma, chunk: int, state_in=None, nthreads: int = 0, lib=None):
    """Block (chunkwise) form in fp64 with block length ``chunk``."""
    return _run("chunkwise", q, k, v, gamma, state_in, chunk, nthreads, lib)


def recurrent_step(q, k, v, gamma, state, nthreads: int = 0, lib=None):
    """One decode step (q, k, v of shape [B,H,1,d]) from ``state``; returns (y, new_state)."""
    return _run("recurrent", q, k, v, gamma, state, 0, nthreads, lib)


def groupnorm(y, eps: float = 1e-5, weight=None, bias=None, lib=None):
    """Per-head group normalisation of y [B,H,L,dv] in fp64 (weight, bias: [H*dv] or None)."""
    lib = lib or load()
    y = _f64(y)
    B, H, L, dv = y.shape
    w = None if weight is None else _f64(weight).reshape(-1)
    b = None if bias is None else _f64(bias).reshape(-1)
    for t in (w, b):
        if t is not None and t.shape[0] != H * dv:
            raise ValueError("oracle: weight and bias must have H*dv values")
    out = np.zeros_like(y)
    if lib.oracle_groupnorm(B, H, L, dv, _ptr(y), float(eps), _ptr(w), _ptr(b), _ptr(out)) != 0:
        raise ValueError("oracle_groupnorm: invalid arguments")
    return out


GATE_ACTS = {"none": 0, "swish": 1, "sigmoid": 2}


def gate(z, g, act: str = "swish", lib=None):
    """out = act(g) * z elementwise in fp64 (act: "none", "swish", "sigmoid")."""
    lib = lib or load()
    z, g = _f64(z), _f64(g)
    if z.shape != g.shape:
        raise ValueError("oracle: gate shape mismatch")
    out = np.zeros_like(z)
    if lib.oracle_gate(z.size, _ptr(z), _ptr(g), GATE_ACTS[act], _ptr(out)) != 0:
        raise ValueError("oracle_gate: invalid arguments")
    return out


def parallel_backward(q, k, v, gamma, dy, lib=None):
    """Gradients (dq, dk, dv) of the parallel form (no carried state) for upstream dy, in fp64."""
    lib = lib or load()
    q, k, v, dy = _f64(q), _f64(k), _f64(v), _f64(dy)
    gamma = _f64(gamma).reshape(-1)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or dy.shape != v.shape or gamma.shape[0] != H:
        raise ValueError("oracle: shape mismatch")
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    if lib.oracle_parallel_backward(B, H, L, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(dy), _ptr(dq),
                                    _ptr(dkk), _ptr(dvv)) != 0:
        raise ValueError("oracle_parallel_backward: invalid arguments")
    return dq, dkk, dvv


def state_backward(q, k, v, gamma, dy, state_in=None, dstate_out=None, lib=None):
    """Only the terms a carried state adds to (dq, dk, dv), and dstate_in, in
    fp64 (oracle_state_backward; linear in L, for long sequences)."""
    lib = lib or load()
    q, k, v, dy = _f64(q), _f64(k), _f64(v), _f64(dy)
    gamma = _f64(gamma).reshape(-1)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    s0 = None if state_in is None else _f64(state_in)
    dso = None if dstate_out is None else _f64(dstate_out)
    for t in (s0, dso):
        if t is not None and t.shape != (B, H, dk, dv):
            raise ValueError("oracle: state shape mismatch")
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    ds0 = np.zeros((B, H, dk, dv))
    if lib.oracle_state_backward(B, H, L, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(dy), _ptr(s0),
                                 _ptr(dso), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(ds0)) != 0:
        raise ValueError("oracle_state_backward: invalid arguments")
    return dq, dkk, dvv, ds0


def backward(q, k, v, gamma, dy, state_in=None, dstate_out=None, lib=None):
    """Gradients (dq, dk, dv, dstate_in) of y and state_out with respect to q,
    k, v and state_in, for upstream dy and dstate_out (None: zero), in fp64.

    The terms without state come from oracle_parallel_backward, the terms of
    the carried state from oracle_state_backward."""
    lib = lib or load()
    dq, dkk, dvv = parallel_backward(q, k, v, gamma, dy, lib=lib)
    q, k, v, dy = _f64(q), _f64(k), _f64(v), _f64(dy)
    gamma = _f64(gamma).reshape(-1)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    s0 = None if state_in is None else _f64(state_in)
    dso = None if dstate_out is None else _f64(dstate_out)
    for t in (s0, dso):
        if t is not None and t.shape != (B, H, dk, dv):
            raise ValueError("oracle: state shape mismatch")
    ds0 = np.zeros((B, H, dk, dv))
    if lib.oracle_state_backward(B, H, L, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(dy),
                                 _ptr(s0), _ptr(dso),
                                 _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(ds0)) != 0:
        raise ValueError("oracle_state_backward: invalid arguments")
    return dq, dkk, dvv, ds0
