"""CUDA graphs around the decode step.

One decode step moves 2 * dk * dv * 4 bytes of state per head; at small batch
that is a few microseconds of HBM time, less than the host time of a call
(argument checks, the ctypes crossing, the launch).  Capturing a run of steps
once as a CUDA graph and replaying it removes the host time from every step
after the first.  The library's calls allocate nothing and make no
synchronising call, so they can be captured as they are; the graph keeps the
pointers and the decay values of the capture, so inputs go through static
buffers that the caller fills before each replay.
"""
from __future__ import annotations

import torch


class DecodeGraph:
    """`n_steps` recurrent steps on `state` (fp32 [B,H,dk,dv], updated in place),
    captured once.  Fill ``q``, ``k`` [n_steps,B,H,1,dk] and ``v``
    [n_steps,B,H,1,dv], call :meth:`replay`, read ``y`` [n_steps,B,H,1,dv]."""

    def __init__(self, state: torch.Tensor, gamma, n_steps: int, dtype=torch.bfloat16):
        from retnet_retention_chunkwise_b200 import library, recurrent_step
        if not state.is_cuda or state.dtype != torch.float32 or state.dim() != 4:
            raise ValueError("retention: state must be a CUDA fp32 [B,H,dk,dv] tensor")
        if n_steps < 1:
            raise ValueError("retention: n_steps >= 1")
        library()  # load before capture
        B, H, dk, dv = state.shape
        dev = state.device
        self.state = state
        self.q = torch.zeros((n_steps, B, H, 1, dk), dtype=dtype, device=dev)
        self.k = torch.zeros((n_steps, B, H, 1, dk), dtype=dtype, device=dev)
        self.v = torch.zeros((n_steps, B, H, 1, dv), dtype=dtype, device=dev)
        self.y = torch.zeros((n_steps, B, H, 1, dv), dtype=dtype, device=dev)
        self._gamma = gamma
        self._step = recurrent_step
        # one eager step on a scratch state first (outside the capture), so that
        # nothing is set up for the first time while the stream is capturing
        scratch = torch.zeros_like(state)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            self._step(self.q[0], self.k[0], self.v[0], gamma, scratch, out=self.y[0])
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        # thread-local capture: CUDA calls made meanwhile by other threads of the
        # process (a collective library's watchdog, a sampler) do not end it
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            for n in range(n_steps):
                self._step(self.q[n], self.k[n], self.v[n], gamma, self.state, out=self.y[n])

    def replay(self):
        """Run the captured steps on the current stream."""
        self.graph.replay()
        return self.y
