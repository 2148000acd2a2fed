"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds no retention arithmetic: it only draws q, k, v and fixes the
per-head decay values and shapes of the named workloads.  Both the CUDA path
and the fp64 oracle consume the exact same bytes produced here.

Recipe: ``torch.Generator('cpu').manual_seed(seed)``, then q, k, v drawn in that
order as ``randn(shape) / sqrt(dk)`` in fp32, then cast (round to nearest even)
to the workload dtype.  Signed values on purpose: retention scores may be
negative (author responses on paperhub.cn, "Retentive Network: A Successor to
Transformer ...", reply on capability vs full attention).  The per-head decay is
gamma_h = 1 - 2^(-5-h), exactly representable in fp32; the pages give no values
for gamma, only that heads use different ones, some near 1 and some smaller
(page "Retentive Networks -- Microsoft ...", section "Il meccanismo").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    dk: int
    dv: int
    chunk: int
    dtype: torch.dtype
    gamma: tuple = field(default=())
    seed: int = 0

    def gammas(self) -> torch.Tensor:
        if self.gamma:
            return torch.tensor(self.gamma, dtype=torch.float32)
        return multiscale_gammas(self.H)


def multiscale_gammas(H: int) -> torch.Tensor:
    """gamma_h = 1 - 2^(-5-h), h = 0..H-1 (fp32, exact)."""
    return torch.tensor([1.0 - 2.0 ** (-5 - h) for h in range(H)], dtype=torch.float32)


def qkv(B: int, H: int, L: int, dk: int, dv: int, dtype=torch.bfloat16, seed: int = 0,
        scale: float | None = None):
    """Seeded q, k [B,H,L,dk] and v [B,H,L,dv] on the CPU, N(0,1)/sqrt(dk)."""
    g = torch.Generator("cpu").manual_seed(seed)
    s = (1.0 / math.sqrt(dk)) if scale is None else scale
    q = torch.randn((B, H, L, dk), generator=g, dtype=torch.float32) * s
    k = torch.randn((B, H, L, dk), generator=g, dtype=torch.float32) * s
    v = torch.randn((B, H, L, dv), generator=g, dtype=torch.float32) * s
    return q.to(dtype), k.to(dtype), v.to(dtype)


def qkv_cuda(B: int, H: int, L: int, dk: int, dv: int, dtype=torch.bfloat16, seed: int = 0,
             device="cuda"):
    """Seeded q, k, v drawn on the device (torch CUDA generator), same recipe as
    :func:`qkv`.  For workloads too large to draw on the host; the oracle reads
    these exact bytes after a copy to the host."""
    g = torch.Generator(device=device).manual_seed(seed)
    s = 1.0 / math.sqrt(dk)
    out = []
    for d in (dk, dk, dv):
        out.append((torch.randn((B, H, L, d), generator=g, device=device, dtype=torch.float32) * s).to(dtype))
    return tuple(out)


def decode_tokens(steps: int, B: int, H: int, dk: int, dv: int, dtype=torch.bfloat16,
                  seed: int = 1):
    """Seeded single-token q, k [steps,B,H,1,dk] and v [steps,B,H,1,dv] for decode."""
    g = torch.Generator("cpu").manual_seed(seed)
    s = 1.0 / math.sqrt(dk)
    q = torch.randn((steps, B, H, 1, dk), generator=g, dtype=torch.float32) * s
    k = torch.randn((steps, B, H, 1, dk), generator=g, dtype=torch.float32) * s
    v = torch.randn((steps, B, H, 1, dv), generator=g, dtype=torch.float32) * s
    return q.to(dtype), k.to(dtype), v.to(dtype)


def state(B: int, H: int, dk: int, dv: int, seed: int = 2, scale: float = 1.0):
    """A seeded fp32 state [B,H,dk,dv] for tests that carry a non-zero state in."""
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn((B, H, dk, dv), generator=g, dtype=torch.float32) * scale


# The named workloads (shapes of the 1.3B / 6.7B head layouts and the small
# parity cases).  C is the chunk length; decode uses a chunkwise prefill.
WORKLOADS = {
    "single_head_f32": Workload("single_head_f32", 1, 1, 64, 16, 16, 16, torch.float32, (0.9,)),
    "msr_core_bf16": Workload("msr_core_bf16", 2, 8, 2048, 64, 128, 64, torch.bfloat16),
    "retnet1p3b_layer_bf16": Workload("retnet1p3b_layer_bf16", 4, 8, 8192, 256, 512, 128,
                                      torch.bfloat16),
    "decode_6p7b_bf16": Workload("decode_6p7b_bf16", 64, 16, 512, 256, 512, 128, torch.bfloat16),
    "long_context_bf16": Workload("long_context_bf16", 1, 16, 65536, 128, 256, 128,
                                  torch.bfloat16),
}
DECODE_STEPS = 1024
LONG_CONTEXT_CALLS = 4
