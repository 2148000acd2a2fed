"""Benchmark of the retention hot path on B200 (one JSON line on rank 0).

Headline step: one chunkwise forward (blocks of C = 128, fp32 state carried
between blocks, state_out returned) over the RetNet-1.3B-shaped layer
B=4, H=8, L=8192, dk=256, dv=512, bf16 q/k/v already resident in HBM.
value = tokens/s = B * L * steps / time, whole job (all ranks).

Also measured in the same run (same timing rules, reported under "forms"):
  decode     -- 1024 recurrent steps, B=64, H=16, dk=256, dv=512, fp32 state
                after a 512-token chunkwise prefill (6.7B-shaped heads);
  parallel   -- parallel form, B=2, H=8, L=2048, dk=64, dv=128 (MSR core);
  parallel_backward -- its gradients dq, dk, dv on the same shape;
  decode_batch1_graph -- decode at batch 1, eager calls against the same
                steps replayed from a CUDA graph;
  chunkwise_backward_long_context -- the gradients through the chunkwise form,
                one 16384-token call of the long-context layout;
  chunkwise_backward_state_long_context -- the same with a carried state
                (state_in, the gradient of state_out, the gradient of state_in);
  chunkwise_msr_core -- chunkwise C=64 on the same MSR-core shape;
  chunkwise_gn_msr_core -- the same with the per-head GroupNorm fused into its
                epilogue, beside the chunkwise call followed by the GroupNorm
                kernel (two_kernel_ms);
  long_context_C{64,128,256} -- B=1, H=16, L=65536, dk=128, dv=256 as four
                16384-token calls with the state carried in place;
  chunkwise_state_headline -- the state-only call (no y) on the headline shape;
  groupnorm  -- per-head group normalisation of a headline-sized output;
  groupnorm_gated -- the same followed by the swish output gate.

Timing: CUDA events on the launching stream, >= 3 warm-up steps, barrier +
synchronize on both sides, max over ranks.  The headline inputs (537 MB) exceed
the 126 MB L2; the small shapes flush L2 (a 256 MB write) before every timed
call and time each call with its own events.  SM clocks and clock-event reasons
are sampled through NVML during the timed region.

--impl reference runs the fp64 CPU oracle (the checker, not a GPU baseline) on
a bounded sample of the headline workload, K timed steps after W warm-ups.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from retnet_retention_chunkwise_b200 import inputs, replicas  # noqa: E402

METRIC = "retention tokens/sec (chunkwise fwd, decode) and % of tensor/HBM roofline"
HEADLINE = inputs.WORKLOADS["retnet1p3b_layer_bf16"]
L2_BYTES = 126 * 1024 * 1024
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
# ncu DRAM traffic of one headline launch, with the digest of the kernel source
# it was captured on (written next to the ncu summary of that capture)
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "chunkwise_tc256_retnet1p3b_layer.traffic.json")


# --------------------------------------------------------------- accounting
def chunk_flops_per_head_token(C, dk, dv):
    """Algorithmic flops of the chunkwise form per (head, token): causal intra-block
    pairs (C+1)/2 per row for Q K^T and P V, plus the cross-block term and the state
    update (2 dk dv each)."""
    return (C + 1) * (dk + dv) + 4 * dk * dv


def chunk_bytes(B, H, L, dk, dv, state_in=False, state_out=True):
    """Algorithmic bytes: q, k, v read once, y written once (bf16), fp32 state in/out."""
    b = B * H * L * (2 * dk + 2 * dv) * 2
    sb = B * H * dk * dv * 4
    return b + (sb if state_in else 0) + (sb if state_out else 0)


def parallel_flops(B, H, L, dk, dv):
    """Causal pairs L(L+1)/2, each 2(dk + dv) flops."""
    return B * H * L * (L + 1) // 2 * 2 * (dk + dv)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured (MEASURED_PEAKS.json)"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback (earlier measurement on this pool)"}


# The headline kernel's source: in chunkwise_tc.cuh the shared helpers (from
# the namespace opening to the dk <= 128 kernel) and chunkwise_tc256_kernel's
# own section (up to the sequence-split helpers that follow it), plus
# tc_common.cuh.  Comments outside those regions and the other kernels of the
# file do not enter it.
HEADLINE_SOURCE_REGIONS = (
    (b"namespace ret {",
     b"template <int DK, bool REV, bool GN = false>\n__global__ void __launch_bounds__(kCW_MainThreads, 1)\n"
     b"chunkwise_tc_kernel("),
    (b"// dk = 256: one stage", b"// Segment sums for the sequence split"),
)


def kernel_source_digest():
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "retnet_retention_chunkwise_b200", "csrc")
    with open(os.path.join(d, "chunkwise_tc.cuh"), "rb") as fh:
        src = fh.read()
    for start, end in HEADLINE_SOURCE_REGIONS:
        i, j = src.find(start), src.find(end)
        h.update(src if i < 0 or j < i else src[i:j])  # a missing marker hashes the whole file
    with open(os.path.join(d, "tc_common.cuh"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic():
    """dram bytes per launch of the headline kernel from the ncu capture's JSON
    record, or None if absent or captured on a different kernel source."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        if rec.get("kernel_source_sha256_16") != kernel_source_digest():
            return None
        return float(rec["dram_bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
               0x1: "gpu_idle"}

    def __init__(self, index, period=0.01):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        self.period, self._stop = period, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        get_r = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples), "source": "nvml" if self.ok else "unavailable"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "source": "nvml"}


# --------------------------------------------------------------- distributed
class Dist:
    def __init__(self, gpus):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            torch.cuda.set_device(self.local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", self.local))
            self.pg = dist
        else:
            torch.cuda.set_device(0)

    def barrier(self):
        if self.pg:
            t = torch.zeros(1, device="cuda")
            self.pg.all_reduce(t)
            torch.cuda.synchronize()

    def max(self, x: float) -> float:
        return replicas.max_over_ranks(x, device="cuda")

    def sum(self, x: float) -> float:
        return replicas.sum_over_ranks(x, device="cuda")

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ------------------------------------------------------------------ helpers
def gpu_qkv(B, H, L, dk, dv, seed):
    """Seeded N(0,1)/sqrt(dk) bf16 q, k, v drawn on the device."""
    return list(inputs.qkv_cuda(B, H, L, dk, dv, torch.bfloat16, seed))


_FLUSH = None


def flush_l2():
    global _FLUSH
    if _FLUSH is None:
        _FLUSH = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    _FLUSH.fill_(1.0)


def time_calls(fn, steps, warmup, dist, flush=False):
    """Per-call device times (ms) of `fn` on the current stream, plus the total of the
    bracketed region.  With flush, an L2 flush (outside the events) precedes each call."""
    for _ in range(warmup):
        if flush:
            flush_l2()
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(st)
    for a, b in ev:
        if flush:
            flush_l2()
        a.record(st)
        fn()
        b.record(st)
    t_end.record(st)
    torch.cuda.synchronize()
    dist.barrier()
    per = [a.elapsed_time(b) for a, b in ev]
    return per, t_start.elapsed_time(t_end)


# --------------------------------------------------------------- workloads
def bench_headline(ret, args, dist, peaks):
    w = HEADLINE
    q, k, v = gpu_qkv(w.B, w.H, w.L, w.dk, w.dv, seed=w.seed)
    gam = w.gammas()
    y = torch.empty_like(v)
    s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    ws_bytes = ret.workspace_bytes(w.chunk, w.B, w.H, w.L, w.dk, w.dv)
    launches_per_call = 3 if ws_bytes > 0 else 1

    def step():
        ret.chunkwise(q, k, v, gam, w.chunk, state_out=s_out, out=y)

    with ClockSampler(dist.local) as clk:
        per, total = time_calls(step, args.steps, args.warmup, dist)
    assert ret.device_status() == 0, "device status set during the headline run"
    t_ms = dist.max(total / args.steps)
    kern_ms = dist.max(statistics.mean(per))
    tokens = w.B * w.L
    head_tokens = w.B * w.H * w.L
    flops = head_tokens * chunk_flops_per_head_token(w.chunk, w.dk, w.dv)
    nbytes = chunk_bytes(w.B, w.H, w.L, w.dk, w.dv, state_in=False, state_out=True)
    ach_gbs = nbytes / (kern_ms * 1e-3) / 1e9
    ach_tf = flops / (kern_ms * 1e-3) / 1e12
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    bound = "hbm" if t_hbm >= t_tensor else "tensor"
    roof = {"bound": bound,
            "achieved": round(ach_gbs if bound == "hbm" else ach_tf, 1),
            "peak": peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops"],
            "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
            "frac": round((ach_gbs / peaks["hbm_gbs"]) if bound == "hbm" else (ach_tf / peaks["bf16_tflops"]), 4),
            "traffic": measured_traffic(),
            "kernel": "chunkwise_tc256_kernel",
            "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
            "kernel_ms": round(kern_ms, 4),
            "tensor": {"achieved_tflops": round(ach_tf, 1), "peak": peaks["bf16_tflops"],
                       "frac": round(ach_tf / peaks["bf16_tflops"], 4),
                       "frac_of_sustained": round(ach_tf / peaks["bf16_tflops_sustained"], 4)},
            "hbm": {"achieved_gbs": round(ach_gbs, 1), "peak": peaks["hbm_gbs"],
                    "frac": round(ach_gbs / peaks["hbm_gbs"], 4)},
            "peak_source": peaks["source"]}
    value = dist.sum(tokens * args.steps) / (t_ms * 1e-3 * args.steps)
    res = {"value": value, "ms_per_step": t_ms, "roofline": roof, "clocks": clk.summary(),
           "gpu_launches": launches_per_call * args.steps}
    del q, k, v, y
    return res


def bench_e2e(ret, args, dist):
    """Same metric through the public API with host buffers: every step copies q, k, v
    from pinned host memory, runs the call, and reads y back to the host (one
    retention_chunkwise_host call per step)."""
    w = HEADLINE
    qh, kh, vh = (t.pin_memory() for t in (torch.empty((w.B, w.H, w.L, d), dtype=torch.bfloat16)
                                          for d in (w.dk, w.dk, w.dv)))
    for t in (qh, kh, vh):
        t.normal_(0.0, 1.0 / math.sqrt(w.dk))
    yh = torch.empty((w.B, w.H, w.L, w.dv), dtype=torch.bfloat16).pin_memory()
    gam = w.gammas()
    dev = tuple(torch.empty_like(t, device="cuda") for t in (qh, kh, vh, yh))
    sd = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    sh = torch.empty(sd.shape, dtype=torch.float32).pin_memory()

    def step():
        # retention_chunkwise_host: q, k, v host -> device, the kernels, y device -> host,
        # overlapped across groups of heads inside the library; then state_out to the host
        ret.chunkwise_host(qh, kh, vh, gam, w.chunk, dev=dev, out=yh, state_out=sd)
        sh.copy_(sd, non_blocking=True)

    steps = 10
    _, total = time_calls(step, steps, max(args.warmup, 3), dist)
    t_ms = dist.max(total / steps)
    value = dist.sum(w.B * w.L * steps) / (t_ms * 1e-3 * steps)
    return {"value": value, "unit": "tokens/s", "ms_per_step": round(t_ms, 3), "steps": steps,
            "h2d_bytes_per_step": sum(t.numel() * 2 for t in (qh, kh, vh)),
            "d2h_bytes_per_step": yh.numel() * 2 + sh.numel() * 4}


def bench_decode(ret, args, dist, peaks):
    w = inputs.WORKLOADS["decode_6p7b_bf16"]
    steps = inputs.DECODE_STEPS
    gam = w.gammas()
    q, k, v = gpu_qkv(w.B, w.H, w.L, w.dk, w.dv, seed=0)
    state = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    ret.chunkwise(q, k, v, gam, w.chunk, state_out=state)  # 512-token prefill
    del q, k, v
    tq, tk, tv = gpu_qkv(steps, w.B * w.H, 1, w.dk, w.dv, seed=1)  # [steps, B*H, 1, d]
    tq = tq.view(steps, w.B, w.H, 1, w.dk)
    tk = tk.view(steps, w.B, w.H, 1, w.dk)
    tv = tv.view(steps, w.B, w.H, 1, w.dv)
    y = torch.empty((w.B, w.H, 1, w.dv), dtype=torch.bfloat16, device="cuda")
    for n in range(3):
        ret.recurrent_step(tq[n], tk[n], tv[n], gam, state, out=y)
    torch.cuda.synchronize()
    dist.barrier()
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    a0, b0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(st)
    for n in range(steps):
        ev[n][0].record(st)
        ret.recurrent_step(tq[n], tk[n], tv[n], gam, state, out=y)
        ev[n][1].record(st)
    b0.record(st)
    torch.cuda.synchronize()
    dist.barrier()
    assert ret.device_status() == 0
    total = dist.max(a0.elapsed_time(b0))
    kern = dist.max(statistics.mean(a.elapsed_time(b) for a, b in ev))
    nbytes = w.B * w.H * (2 * w.dk * w.dv * 4 + (2 * w.dk + 2 * w.dv) * 2)
    gbs = nbytes / (kern * 1e-3) / 1e9
    return {"workload": "B64 H16 dk256 dv512, 1024 steps after a 512-token prefill",
            "tokens_per_s": dist.sum(w.B * steps) / (total * 1e-3),
            "ms_per_token_step": round(total / steps, 4), "kernel_ms": round(kern, 4),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes,
                         "kernel": "recurrent_step_kernel<bf16>"},
            "gpu_launches": steps}


def bench_decode_graph(ret, args, dist, peaks):
    """Decode at batch 1 (one sequence, 6.7B-shaped heads): a step moves 16.8 MB
    of state, a few microseconds of HBM time, so eager calls are bound by the
    host.  The same steps captured once as a CUDA graph (graphs.DecodeGraph)
    and replayed."""
    from retnet_retention_chunkwise_b200.graphs import DecodeGraph
    B, H, dk, dv, n = 1, 16, 256, 512, 64
    gam = inputs.multiscale_gammas(H)
    state = torch.zeros((B, H, dk, dv), dtype=torch.float32, device="cuda")
    tq, tk, tv = gpu_qkv(n, B * H, 1, dk, dv, seed=1)
    tq, tk, tv = (t.view(n, B, H, 1, -1) for t in (tq, tk, tv))
    y = torch.empty((B, H, 1, dv), dtype=torch.bfloat16, device="cuda")

    def eager():
        for i in range(n):
            ret.recurrent_step(tq[i], tk[i], tv[i], gam, state, out=y)

    _, t_eager = time_calls(eager, 10, max(args.warmup, 3), dist)
    g = DecodeGraph(state, gam, n)
    g.q.copy_(tq)
    g.k.copy_(tk)
    g.v.copy_(tv)
    _, t_graph = time_calls(g.replay, 10, max(args.warmup, 3), dist)
    assert ret.device_status() == 0
    e = dist.max(t_eager) / (10 * n)
    gr = dist.max(t_graph) / (10 * n)
    nbytes = B * H * (2 * dk * dv * 4 + (2 * dk + 2 * dv) * 2)
    return {"workload": "B1 H16 dk256 dv512, 64 steps per graph",
            "eager_ms_per_step": round(e, 4), "graph_ms_per_step": round(gr, 4),
            "tokens_per_s_graph": dist.sum(B) / (gr * 1e-3),
            "hbm_frac_graph": round(nbytes / (gr * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}


def _shape_of(w):
    from retnet_retention_chunkwise_b200 import _abi
    return _abi.RetShape(w.B, w.H, w.L, w.dk, w.dv)


def bench_small(ret, args, dist, peaks):
    out = {}
    w = inputs.WORKLOADS["msr_core_bf16"]
    q, k, v = gpu_qkv(w.B, w.H, w.L, w.dk, w.dv, seed=0)
    gam = w.gammas()
    y = torch.empty_like(v)
    n = 50
    per, _ = time_calls(lambda: ret.parallel(q, k, v, gam, out=y), n, max(args.warmup, 3), dist, flush=True)
    t = dist.max(statistics.median(per))
    fl = parallel_flops(w.B, w.H, w.L, w.dk, w.dv)
    out["parallel"] = {"workload": "B2 H8 L2048 dk64 dv128, L2 flushed",
                       "tokens_per_s": dist.sum(w.B * w.L) / (t * 1e-3), "kernel_ms": round(t, 4),
                       "roofline": {"bound": "tensor", "achieved": round(fl / (t * 1e-3) / 1e12, 1),
                                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                    "frac": round(fl / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                                    "algorithmic_flops": fl, "kernel": "parallel_tc_kernel<64>"}}
    dy = torch.randn_like(v) / math.sqrt(w.dv)
    ws = torch.empty(int(ret.library().retention_parallel_backward_workspace_bytes(
        _shape_of(w), 1)) // 4 + 64, dtype=torch.float32, device="cuda")
    per, _ = time_calls(lambda: ret.parallel_backward(q, k, v, gam, dy, workspace=ws), n, max(args.warmup, 3),
                        dist, flush=True)
    t = dist.max(statistics.median(per))
    out["parallel_backward"] = {"workload": "B2 H8 L2048 dk64 dv128, L2 flushed",
                                "tokens_per_s": dist.sum(w.B * w.L) / (t * 1e-3), "call_ms": round(t, 4),
                                "tensor": {"achieved_tflops": round(3 * fl / (t * 1e-3) / 1e12, 1),
                                           "frac": round(3 * fl / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                                           "algorithmic_flops": 3 * fl}}
    del dy, ws
    per, _ = time_calls(lambda: ret.chunkwise(q, k, v, gam, w.chunk, out=y, return_state=False), n,
                        max(args.warmup, 3), dist, flush=True)
    t = dist.max(statistics.median(per))
    nb = chunk_bytes(w.B, w.H, w.L, w.dk, w.dv, state_out=False)
    out["chunkwise_msr_core"] = {"workload": "B2 H8 L2048 dk64 dv128 C64, L2 flushed",
                                 "tokens_per_s": dist.sum(w.B * w.L) / (t * 1e-3), "call_ms": round(t, 4),
                                 "hbm_frac": round(nb / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    per, _ = time_calls(lambda: ret.chunkwise_groupnorm(q, k, v, gam, w.chunk, 1e-5, out=y, return_state=False),
                        n, max(args.warmup, 3), dist, flush=True)
    t_f = dist.max(statistics.median(per))

    def two_calls():
        ret.chunkwise(q, k, v, gam, w.chunk, out=y, return_state=False)
        ret.groupnorm(y, 1e-5, out=y)
    per, _ = time_calls(two_calls, n, max(args.warmup, 3), dist, flush=True)
    t_2 = dist.max(statistics.median(per))
    out["chunkwise_gn_msr_core"] = {"workload": "B2 H8 L2048 dk64 dv128 C64 + GroupNorm, L2 flushed",
                                    "tokens_per_s": dist.sum(w.B * w.L) / (t_f * 1e-3),
                                    "call_ms": round(t_f, 4), "two_kernel_ms": round(t_2, 4),
                                    "hbm_frac": round(nb / (t_f * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    del q, k, v, y
    w = inputs.WORKLOADS["long_context_bf16"]
    q, k, v = gpu_qkv(w.B, w.H, w.L, w.dk, w.dv, seed=0)
    gam = w.gammas()
    seg = w.L // inputs.LONG_CONTEXT_CALLS
    parts = [(q[:, :, i:i + seg].contiguous(), k[:, :, i:i + seg].contiguous(), v[:, :, i:i + seg].contiguous())
             for i in range(0, w.L, seg)]
    del q, k, v
    y = torch.empty_like(parts[0][2])
    state = torch.zeros((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    for C in (64, 128, 256):
        def four_calls():
            state.zero_()
            for qq, kk, vv in parts:
                ret.chunkwise(qq, kk, vv, gam, C, state_in=state, state_out=state, out=y)
        per, _ = time_calls(four_calls, 10, max(args.warmup, 3), dist)
        t = dist.max(statistics.median(per))
        fl = w.B * w.H * w.L * chunk_flops_per_head_token(C, w.dk, w.dv)
        nb = chunk_bytes(w.B, w.H, w.L, w.dk, w.dv) + 2 * inputs.LONG_CONTEXT_CALLS * w.B * w.H * w.dk * w.dv * 4
        out[f"long_context_C{C}"] = {
            "workload": "B1 H16 L65536 dk128 dv256, 4 calls, state carried",
            "tokens_per_s": dist.sum(w.B * w.L) / (t * 1e-3), "ms_per_65536_tokens": round(t, 4),
            "hbm_frac": round(nb / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "tensor_frac": round(fl / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}
    # backward through the chunkwise form, one 16384-token call of the same layout
    qq, kk, vv = parts[0]
    dy = torch.randn_like(vv) / math.sqrt(w.dv)
    per, _ = time_calls(lambda: ret.chunkwise_backward(qq, kk, vv, gam, dy, 128), 10, max(args.warmup, 3), dist)
    t = dist.max(statistics.median(per))
    fl = 3 * w.B * w.H * seg * chunk_flops_per_head_token(128, w.dk, w.dv)
    out["chunkwise_backward_long_context"] = {
        "workload": "B1 H16 L16384 dk128 dv256 C128",
        "tokens_per_s": dist.sum(w.B * seg) / (t * 1e-3), "call_ms": round(t, 4),
        "tensor_frac": round(fl / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}
    # the same call carrying a state: state_in, dstate_out in, dstate_in out
    s0 = torch.randn((w.B, w.H, w.dk, w.dv), device="cuda") / math.sqrt(w.dk)
    dso = torch.randn_like(s0) / math.sqrt(w.dv)
    ds0 = torch.empty_like(s0)
    per, _ = time_calls(lambda: ret.chunkwise_backward_state(qq, kk, vv, gam, dy, 128, s0, dso, dstate_in=ds0), 10,
                        max(args.warmup, 3), dist)
    t = dist.max(statistics.median(per))
    out["chunkwise_backward_state_long_context"] = {
        "workload": "B1 H16 L16384 dk128 dv256 C128, with states",
        "tokens_per_s": dist.sum(w.B * seg) / (t * 1e-3), "call_ms": round(t, 4),
        "tensor_frac": round(fl / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}
    del parts, y, dy, s0, dso, ds0
    # state only (no y) on the headline shape: k and v read once (403 MB, larger than L2)
    w = HEADLINE
    k = (torch.randn((w.B, w.H, w.L, w.dk), device="cuda") / math.sqrt(w.dk)).to(torch.bfloat16)
    v = (torch.randn((w.B, w.H, w.L, w.dv), device="cuda") / math.sqrt(w.dk)).to(torch.bfloat16)
    s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    need = ret.library().retention_chunkwise_state_workspace_bytes(w.chunk, ret._shape(k, v), ret._abi.RET_BF16)
    wsb = torch.empty((need + 3) // 4, dtype=torch.float32, device="cuda")
    per, _ = time_calls(lambda: ret.chunkwise_state(k, v, w.gammas(), w.chunk, out=s_out, workspace=wsb), 20,
                        max(args.warmup, 3), dist)
    t = dist.max(statistics.median(per))
    nb = (k.numel() + v.numel()) * 2 + s_out.numel() * 4
    fl = 2 * w.B * w.H * w.L * w.dk * w.dv
    out["chunkwise_state_headline"] = {
        "workload": "B4 H8 L8192 dk256 dv512, k v in, fp32 state out",
        "call_ms": round(t, 4), "tokens_per_s": dist.sum(w.B * w.L) / (t * 1e-3),
        "roofline": {"bound": "hbm", "achieved": round(nb / (t * 1e-3) / 1e9, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(nb / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                     "algorithmic_bytes": nb, "kernel": "chunk_state_kernel<256> + state_fold_kernel"},
        "tensor_frac": round(fl / (t * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}
    del k, v, s_out, wsb
    # per-head group normalisation of a headline-sized output (268 MB, larger than L2), in place
    y = (torch.randn((w.B, w.H, w.L, w.dv), device="cuda") * 0.5).to(torch.bfloat16)
    per, _ = time_calls(lambda: ret.groupnorm(y, 1e-5, out=y), 20, max(args.warmup, 3), dist)
    t = dist.max(statistics.median(per))
    nb = 2 * y.numel() * y.element_size()
    out["groupnorm"] = {"workload": "B4 H8 L8192 dv512, in place",
                        "kernel_ms": round(t, 4), "tokens_per_s": dist.sum(w.B * w.L) / (t * 1e-3),
                        "roofline": {"bound": "hbm", "achieved": round(nb / (t * 1e-3) / 1e9, 1),
                                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                     "frac": round(nb / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                     "algorithmic_bytes": nb, "kernel": "groupnorm_rows_kernel<bf16>"}}
    # the same with the swish output gate: y and the gate read once, the result written once
    gate = torch.randn_like(y)
    per, _ = time_calls(lambda: ret.groupnorm(y, 1e-5, out=y, gate=gate, act="swish"), 20, max(args.warmup, 3), dist)
    t = dist.max(statistics.median(per))
    nb = 3 * y.numel() * y.element_size()
    out["groupnorm_gated"] = {"workload": "B4 H8 L8192 dv512, swish gate, in place",
                              "kernel_ms": round(t, 4), "tokens_per_s": dist.sum(w.B * w.L) / (t * 1e-3),
                              "roofline": {"bound": "hbm", "achieved": round(nb / (t * 1e-3) / 1e9, 1),
                                           "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                           "frac": round(nb / (t * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                                           "algorithmic_bytes": nb, "kernel": "groupnorm_rows_kernel<bf16>"}}
    del y, gate
    return out


def bench_headline_sustained(ret, args, dist, peaks, seconds=1.5):
    """The headline call repeated for about `seconds` (the power cap and the
    clock it settles at show up here, unlike in a short burst), with the SM
    clock sampled during the run."""
    w = HEADLINE
    q, k, v = gpu_qkv(w.B, w.H, w.L, w.dk, w.dv, seed=w.seed)
    gam = w.gammas()
    y = torch.empty_like(v)
    s_out = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    step = lambda: ret.chunkwise(q, k, v, gam, w.chunk, state_out=s_out, out=y)  # noqa: E731
    n = max(20, int(seconds / 0.25e-3))
    with ClockSampler(dist.local) as clk:
        per, _ = time_calls(step, n, 5, dist)
    assert ret.device_status() == 0
    kern = dist.max(statistics.mean(per))
    flops = w.B * w.H * w.L * chunk_flops_per_head_token(w.chunk, w.dk, w.dv)
    nbytes = chunk_bytes(w.B, w.H, w.L, w.dk, w.dv, state_in=False, state_out=True)
    tf = flops / (kern * 1e-3) / 1e12
    return {"steps": n, "kernel_ms": round(kern, 4), "clocks": clk.summary(),
            "hbm_frac": round(nbytes / (kern * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "tensor_frac": round(tf / peaks["bf16_tflops"], 4),
            "tensor_frac_of_sustained": round(tf / peaks["bf16_tflops_sustained"], 4)}


# ------------------------------------------------------------ CPU / oracle
def oracle_sample(nthreads=None, L=None):
    """A bounded sample of the headline workload for the fp64 oracle: `nthreads`
    (b, h) heads of batch row 0, the first L positions.  Returns (fn, tokens) where
    tokens counts B*L-style tokens (one token = all H heads of one position)."""
    import oracle
    w = HEADLINE
    nthreads = nthreads or max(1, min(os.cpu_count() or 1, w.B * w.H))
    L = L or w.L
    q, k, v = inputs.qkv(1, nthreads, L, w.dk, w.dv, torch.bfloat16, seed=w.seed)
    q, k, v = (t.double().numpy() for t in (q, k, v))
    g = w.gammas()
    gam = torch.stack([g[i % w.H] for i in range(nthreads)]).double().numpy()
    lib = oracle.load()

    def fn():
        oracle.recurrent(q, k, v, gam, nthreads=nthreads, lib=lib)
    return fn, nthreads * L / w.H, nthreads, L


def cpu_baseline():
    fn, tokens, nthreads, L = oracle_sample()
    t0 = time.perf_counter()
    fn()
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": f"fp64 recurrent oracle on {nthreads} of {HEADLINE.B * HEADLINE.H} heads x {L} positions "
                      f"of the headline workload ({dt:.1f} s), tokens scaled by heads/H"}


def oracle_timings():
    """The fp64 oracle (oracle_recurrent) timed on this host for every
    configuration: T = all cores over (b, h), plus one thread for the two small
    ones.  Bounded samples of the large ones (T heads; tokens scaled by T/H).
    A CPU baseline, not the target."""
    import oracle
    lib = oracle.load()
    T = os.cpu_count() or 1

    def timed(q, k, v, gam, threads, reps=1):
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle.recurrent(q, k, v, gam, nthreads=threads, lib=lib)
        return (time.perf_counter() - t0) / reps

    def heads(w, n, L, seed):
        q, k, v = inputs.qkv(1, n, L, w.dk, w.dv, w.dtype, seed)
        g = w.gammas()
        return q, k, v, torch.stack([g[i % w.H] for i in range(n)])

    out = {"threads": T}
    w = inputs.WORKLOADS["single_head_f32"]
    q, k, v = inputs.qkv(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    t1 = timed(q, k, v, w.gammas(), 1, reps=200)
    out["single_head_f32"] = {"tokens_per_s_1thread": round(w.B * w.L / t1), "sample": "whole workload"}
    w = inputs.WORKLOADS["msr_core_bf16"]
    q, k, v = inputs.qkv(w.B, w.H, w.L, w.dk, w.dv, w.dtype, w.seed)
    t1, tT = timed(q, k, v, w.gammas(), 1), timed(q, k, v, w.gammas(), T)
    out["msr_core_bf16"] = {"tokens_per_s_1thread": round(w.B * w.L / t1), "tokens_per_s": round(w.B * w.L / tT),
                            "sample": "whole workload"}
    w = inputs.WORKLOADS["retnet1p3b_layer_bf16"]
    n, L = min(T, w.B * w.H), 2048
    tT = timed(*heads(w, n, L, 0), T)
    out["retnet1p3b_layer_bf16"] = {"tokens_per_s": round(n / w.H * L / tT), "sample": f"{n} heads x {L} tokens"}
    w = inputs.WORKLOADS["decode_6p7b_bf16"]
    n, steps = min(T, w.B * w.H), inputs.DECODE_STEPS
    tT = timed(*heads(w, n, steps, 1), T)
    out["decode_6p7b_bf16"] = {"tokens_per_s": round(n / w.H * steps / tT),
                               "sample": f"{n} heads x {steps} steps from a zero state"}
    w = inputs.WORKLOADS["long_context_bf16"]
    n, L = min(T, w.B * w.H), 4096
    tT = timed(*heads(w, n, L, 0), T)
    out["long_context_bf16"] = {"tokens_per_s": round(n / w.H * L / tT), "sample": f"{n} heads x {L} tokens"}
    return out


def headline_config(world: int) -> dict:
    """The workload both arms report (the reference arm times a sample of it)."""
    w = HEADLINE
    return {"workload": "retnet1p3b_layer_bf16: chunkwise forward, C=128, fp32 state out",
            "global_batch": w.B * world, "B_per_gpu": w.B, "H": w.H, "seq_len": w.L,
            "dk": w.dk, "dv": w.dv, "chunk": w.chunk,
            "parallelism": f"dp{world}: independent (b, h) replicas, no collective",
            "l2": "inputs 537 MB > 126 MB L2, no flush"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    fn, tokens, nthreads, L = oracle_sample(L=256)
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    dt = (time.perf_counter() - t0) / args.steps
    value = tokens / dt
    w = HEADLINE
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": headline_config(int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                             "sample": f"each step: fp64 recurrent oracle on {nthreads} heads x {L} positions "
                                       f"of the headline workload, tokens scaled by heads/H"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Repeated calls of one form on one shape (for ncu); prints per-call ms."""
    import retnet_retention_chunkwise_b200 as ret
    torch.cuda.set_device(0)
    kind, dims = args.profile.split(":")
    d = [int(x) for x in dims.split(",")]
    if kind == "chunkwise":
        B, H, L, dk, dv, C = d
        q, k, v = gpu_qkv(B, H, L, dk, dv, seed=0)
        gam = inputs.multiscale_gammas(H)
        fn = lambda: ret.chunkwise(q, k, v, gam, C)  # noqa: E731
    elif kind == "parallel":
        B, H, L, dk, dv = d
        q, k, v = gpu_qkv(B, H, L, dk, dv, seed=0)
        gam = inputs.multiscale_gammas(H)
        fn = lambda: ret.parallel(q, k, v, gam)  # noqa: E731
    elif kind == "decode":
        B, H, dk, dv = d
        q, k, v = gpu_qkv(B, H, 1, dk, dv, seed=1)
        gam = inputs.multiscale_gammas(H)
        st = torch.zeros((B, H, dk, dv), dtype=torch.float32, device="cuda")
        fn = lambda: ret.recurrent_step(q, k, v, gam, st)  # noqa: E731
    elif kind in ("groupnorm", "groupnorm_gated"):
        B, H, L, dv = d
        g = torch.Generator("cuda").manual_seed(0)
        y = torch.randn((B, H, L, dv), generator=g, device="cuda").to(torch.bfloat16)
        gate = torch.randn((B, H, L, dv), generator=g, device="cuda").to(torch.bfloat16)
        if kind == "groupnorm":
            fn = lambda: ret.groupnorm(y, 1e-5, out=y)  # noqa: E731
        else:
            fn = lambda: ret.groupnorm(y, 1e-5, out=y, gate=gate, act="swish")  # noqa: E731
    elif kind == "state":
        B, H, L, dk, dv, C = d
        _, k, v = gpu_qkv(B, H, L, dk, dv, seed=0)
        gam = inputs.multiscale_gammas(H)
        fn = lambda: ret.chunkwise_state(k, v, gam, C)  # noqa: E731
    else:
        raise SystemExit(f"unknown profile kind {kind}")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        print(f"{kind} {dims}: {a.elapsed_time(b):.4f} ms", flush=True)
    assert ret.device_status() == 0


def run_sequence(args):
    """--mode sequence: one sequence of the long-context layout (B=1, H=16,
    dk=128, dv=256, C=128) cut across the ranks, each rank holding a run of
    65536 tokens (weak scaling: the sequence is 65536 * N tokens).  A step is
    chunkwise_sequence_sharded on every rank: the run's state-only sum, one
    NCCL all-gather of the sums, the fold, the chunkwise call from the folded
    state.  value = tokens of the whole sequence / max-over-ranks time."""
    import datetime
    import socket

    import torch.distributed as tdist

    import retnet_retention_chunkwise_b200 as ret
    from retnet_retention_chunkwise_b200 import sequence
    ret.library()
    dist = Dist(args.gpus)
    own_group = False
    if not tdist.is_initialized():  # one rank: a one-rank NCCL group of its own
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        store = tdist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
        tdist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                                 device_id=torch.device("cuda", torch.cuda.current_device()))
        own_group = True
    w = inputs.WORKLOADS["long_context_bf16"]
    C, L_run = 128, w.L
    q, k, v = gpu_qkv(w.B, w.H, L_run, w.dk, w.dv, seed=dist.rank)
    gam = w.gammas()
    lens = [L_run] * dist.world

    def step():
        sequence.chunkwise_sequence_sharded(q, k, v, gam, C, lens=lens)

    steps = min(args.steps, 200)
    with ClockSampler(dist.local) as clk:
        _, total = time_calls(step, steps, args.warmup, dist)
    assert ret.device_status() == 0
    t_ms = dist.max(total / steps)
    value = dist.sum(w.B * L_run * steps) / (t_ms * 1e-3 * steps)
    line = {"metric": METRIC, "mode": "sequence", "value": value, "unit": "tokens/s", "n_gpus": dist.world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": t_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "long_context_bf16 sequence cut across ranks: B=1 H=16 dk=128 dv=256 C=128, "
                                   f"{L_run} tokens per rank", "seq_len": L_run * dist.world,
                       "parallelism": f"sequence-sharded over {dist.world} ranks, one all-gather of "
                                      "B*H*dk*dv fp32 run sums per step"},
            "clocks": clk.summary(), "gpu_launches": None}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    if own_group:
        tdist.destroy_process_group()
    dist.close()


# ----------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-forms", action="store_true", help="headline only")
    ap.add_argument("--mode", default="headline", choices=["headline", "sequence"],
                    help="sequence: time one long-context sequence cut across the ranks instead")
    ap.add_argument("--profile", default=None,
                    help="run only one kind of call for a profiler, no JSON: "
                         "chunkwise:B,H,L,dk,dv,C | parallel:B,H,L,dk,dv | decode:B,H,dk,dv | "
                         "groupnorm:B,H,L,dv | groupnorm_gated:B,H,L,dv | state:B,H,L,dk,dv,C")
    args = ap.parse_args()
    if args.warmup < 3 and args.profile is None:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    if args.profile:
        run_profile_case(args)
        return
    if args.mode == "sequence":
        run_sequence(args)
        return
    import retnet_retention_chunkwise_b200 as ret
    ret.library()
    dist = Dist(args.gpus)
    peaks = load_peaks()
    head = bench_headline(ret, args, dist, peaks)
    e2e = bench_e2e(ret, args, dist)
    forms = {}
    if not args.no_forms:
        # the line is long: decode goes last, so a reader of its tail sees it
        forms.update(bench_small(ret, args, dist, peaks))
        forms["headline_sustained"] = bench_headline_sustained(ret, args, dist, peaks)
        forms["decode_batch1_graph"] = bench_decode_graph(ret, args, dist, peaks)
        forms["decode"] = bench_decode(ret, args, dist, peaks)
    cpu = None
    if dist.rank == 0 and dist.world == 1:
        cpu = cpu_baseline()
        if not args.no_forms:
            cpu["per_config"] = oracle_timings()
    w = HEADLINE
    line = {"metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1)/sqrt(dk) bf16 q,k,v; gamma_h = 1 - 2^(-5-h)",
            "config": headline_config(dist.world),
            "roofline": head["roofline"], "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": head["gpu_launches"], "clocks": head["clocks"], "forms": forms}
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
