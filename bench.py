"""Benchmark of the batch-1 MoE decode hot path on B200.

One step = one Ling-shaped MoE layer (router GEMV + top-8-of-512 softmax
routing + MXFP4 gate/up/SiLU/down over the selected experts + shared expert +
combine) followed by the 157,184 x 2,560 online-FP8 LM head (GEMV + per-row
scale + top-29 + logits), for M = 1 token; the same step at M = 4 (the verify
step) is reported beside it.  Metric: microseconds per step (lower is
better), and the LM head's achieved HBM bandwidth against the measured peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs an independent replica on its own GPU
(the path has no cross-GPU exchange); the reported time is the max over
ranks and `value` is that time divided by all steps of all ranks.

Inputs are synthetic and seeded (normal weights, bf16 activations; see
moe_decode_gemv_b200/inputs.py), drawn on the GPU for speed.  Eight layer
copies rotate from step to step, so the 5.2 MB router and the shared expert
are not served from L2; with the 403 MB head in every step, the bytes touched
per step exceed the 126 MB L2 several times over.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "us per MoE layer + LM head per decode step (M=1/M=4); achieved HBM GB/s vs peak"
UNIT = "us/step"
N_LAYERS = 8
N_X = 64
HEAD_TOPK = 29


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-m4", action="store_true")
    p.add_argument("--only", choices=["all", "head", "moe"], default="all",
                   help="profiling aid: time only one half of the step (small device footprint)")
    p.add_argument("--layers", type=int, default=N_LAYERS, help="layer copies that rotate (profiling aid)")
    p.add_argument("--profile-m", type=int, choices=[1, 4], default=1, help="tokens per step with --only (profiling aid)")
    p.add_argument("--no-stream", action="store_true", help="skip the 16-layer decode-stream leg")
    p.add_argument("--stream-steps", type=int, default=200)
    return p.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (replicas)
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, local, backend="nccl"):
    import datetime

    import torch
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a float over ranks (the slowest replica sets the job's time)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """SM clock, power and clock-event reasons sampled during a window, by
    read-only NVML queries in a thread (nvidia-smi when NVML is missing).
    Nothing here changes a setting of the GPU."""

    def __init__(self, gpu_index: int, period_s: float = 0.02):
        self.samples = []  # (time, sm_mhz, sm_max_mhz, power_w, reasons bitmask)
        self.window = None
        self.source = None
        self._stop = threading.Event()
        self.proc = None
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def loop():
                while not self._stop.is_set():
                    try:
                        self.samples.append((time.time(), float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                             sm_max, pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0, int(reasons(h))))
                    except Exception:  # a query this driver lacks: stop sampling, report what there is
                        return
                    self._stop.wait(period_s)

            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            self.source = "nvml"
        except Exception:
            self._start_smi(gpu_index, int(period_s * 1000))

    def _start_smi(self, gpu_index, period_ms):
        cmd = ["nvidia-smi", "-i", str(gpu_index),
               "--query-gpu=timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", str(max(period_ms, 50))]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
            self.source = "nvidia-smi"
        except (OSError, ValueError):
            self.proc = None

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 5:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                self.samples.append((ts, float(parts[1]), float(parts[2]), float(parts[3]), int(parts[4], 16)))
            except (ValueError, IndexError):
                continue

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples (NVML and nvidia-smi)"],
                    "source": self.source}
        t0, t1 = self.window if self.window else (0, 1e18)
        inwin = [s for s in self.samples if t0 - 0.05 <= s[0] <= t1 + 0.05] or self.samples[-3:]
        reasons = set()
        for s in inwin:
            for bit, name in REASON_BITS.items():
                if s[4] & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in inwin), "sm_max_mhz": max(s[2] for s in inwin),
                "power_w_max": max(s[3] for s in inwin), "samples": len(inwin), "reasons": sorted(reasons),
                "source": self.source}


# ---------------------------------------------------------------------------
# workload on the GPU
# ---------------------------------------------------------------------------

class Workload:
    def __init__(self, B, I, seed: int, device, n_layers: int = N_LAYERS, head: bool = True):
        import torch
        self.B, self.torch = B, torch
        s, h = I.LING_MOE, I.LING_HEAD
        self.s, self.h = s, h
        self.layers, self.bias = [], []
        for l in range(n_layers):
            router = I.router_weight(seed, s.experts, s.hidden, layer=l, device=device)
            banks, shared = [], []
            for kind in ("gate", "up", "down"):
                rows, cols = (s.inter, s.hidden) if kind != "down" else (s.hidden, s.inter)
                st = I.normal(seed, f"L{l}/bank/{kind}", (s.experts, rows, cols), I.WEIGHT_STD, device=device)
                banks.append(B.moe_quantize_mxfp4(st))
                del st
                sh = I.expert_matrix(seed, s, "shared", kind, layer=l, device=device)
                shared.append(B.moe_quantize_mxfp4(sh))
            # load time: regroup the quantised bytes into the layout moe_decode streams
            self.layers.append((router, B.moe_pack_experts(tuple(banks)), B.moe_pack_experts(tuple(shared))))
            # the skewed regime: a per-expert logit bias N(0, 2^2), so tokens share experts
            self.bias.append(I.router_bias(seed, s.experts, layer=l, device=device))
            del banks, shared
        self.head_bf16 = self.head = None
        if head:
            self.head_bf16 = I.normal(seed, "lmhead", (h.vocab, h.hidden), I.WEIGHT_STD, device=device)
            self.head = B.lmhead_quantize_fp8(self.head_bf16)
        self.x = {M: I.hidden_states(seed, N_X * M, s.hidden, tag=f"bench{M}", device=device).view(N_X, M, s.hidden)
                  for M in (1, 4)}
        self.out = {M: torch.empty((M, s.hidden), dtype=torch.float32, device=device) for M in (1, 4)}
        self.ids = {M: torch.empty((M, s.top_k), dtype=torch.int32, device=device) for M in (1, 4)}
        self.w = {M: torch.empty((M, s.top_k), dtype=torch.float32, device=device) for M in (1, 4)}
        self.tk_ids = {M: torch.empty((M, HEAD_TOPK), dtype=torch.int32, device=device) for M in (1, 4)}
        self.tk_vals = {M: torch.empty((M, HEAD_TOPK), dtype=torch.float32, device=device) for M in (1, 4)}
        self.logits = {M: torch.empty((M, h.vocab), dtype=torch.float32, device=device) for M in (1, 4)}
        self.moe_ws = {M: B.new_workspace(B.moe_workspace_bytes(M, s.top_k, s.experts, s.hidden, s.inter), device)
                       for M in (1, 4)}
        self.head_ws = {M: B.new_workspace(B.lmhead_workspace_bytes(M, HEAD_TOPK, h.vocab, h.hidden), device)
                        for M in (1, 4)}
        torch.cuda.synchronize()

    def step(self, i: int, M: int, ev=None, x_moe=None, x_head=None, skewed: bool = False):
        """One decode step: MoE layer (layer i mod 8) then the LM head."""
        B = self.B
        xm = self.x[M][i % N_X] if x_moe is None else x_moe
        xh = self.x[M][(i + 1) % N_X] if x_head is None else x_head
        if ev is not None:
            ev[0].record()
        if self.layers:
            l = i % len(self.layers)
            router, banks, shared = self.layers[l]
            B.moe_decode(xm, router, self.bias[l] if skewed else None, banks, shared, self.s.top_k, self.out[M],
                         self.ids[M], self.w[M], workspace=self.moe_ws[M])
        if ev is not None:
            ev[1].record()
        if self.head is not None:
            B.lmhead_decode(xh, self.head, HEAD_TOPK, self.tk_ids[M], self.tk_vals[M], self.logits[M],
                            workspace=self.head_ws[M])
        if ev is not None:
            ev[2].record()

    def bf16_head(self, i: int, M: int):
        self.B.lmhead_decode_bf16(self.x[M][i % N_X], self.head_bf16, HEAD_TOPK, self.tk_ids[M], self.tk_vals[M],
                                  self.logits[M], workspace=self.head_ws[M])


def _q(v, f):
    v = sorted(v)
    return v[min(len(v) - 1, int(f * len(v)))]


def block_steps(steps):
    """Steps between two timing events in the distribution pass: 20 when
    there are at least 200 steps (so at least 10 blocks), else a tenth."""
    return 20 if steps >= 200 else max(1, steps // 10)


def time_steps(wl, M, steps, warmup, dist, device, skewed=False):
    """Device time of `steps` steps, in three passes over the same steps on
    the launching stream: (1) CUDA events every `block` steps only, for the
    distribution of the per-step time over blocks (inside a block every
    kernel keeps its programmatic launch, across steps too); (2) two events
    around all steps, for the mean of back-to-back steps; (3) an extra event
    between the MoE layer and the head of every step, for the split between
    them (us)."""
    torch = wl.torch
    for i in range(warmup):
        wl.step(i, M, skewed=skewed)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    # (1) per-step time over blocks of steps
    block = block_steps(steps)
    nblk = max(1, steps // block)
    bounds = [ev() for _ in range(nblk + 1)]
    t0 = time.time()
    bounds[0].record()
    for b in range(nblk):
        for i in range(block):
            wl.step(warmup + b * block + i, M, skewed=skewed)
        bounds[b + 1].record()
    torch.cuda.synchronize()
    t1 = time.time()
    step = [bounds[b].elapsed_time(bounds[b + 1]) * 1e3 / block for b in range(nblk)]
    # (2) back-to-back
    e0, e1 = ev(), ev()
    e0.record()
    for i in range(steps):
        wl.step(warmup + steps + i, M, skewed=skewed)
    e1.record()
    torch.cuda.synchronize()
    total_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    # (3) the split
    evs = [(ev(), ev(), ev()) for _ in range(steps)]
    for i in range(steps):
        wl.step(warmup + 2 * steps + i, M, ev=evs[i], skewed=skewed)
    torch.cuda.synchronize()
    moe = [e[0].elapsed_time(e[1]) * 1e3 for e in evs]
    head = [e[1].elapsed_time(e[2]) * 1e3 for e in evs]
    med = max_over_ranks(statistics.median(step), dist, device)
    return {"total_us": total_ms * 1e3, "per_step_us": total_ms * 1e3 / steps, "block_steps": block,
            "step_us_median": med, "step_us_p10": _q(step, 0.1), "step_us_p90": _q(step, 0.9),
            "moe_us_mean": statistics.fmean(moe), "moe_us_median": statistics.median(moe),
            "moe_us_p10": _q(moe, 0.1), "moe_us_p90": _q(moe, 0.9),
            "head_us_mean": statistics.fmean(head), "head_us_median": statistics.median(head),
            "head_us_p10": _q(head, 0.1), "head_us_p90": _q(head, 0.9),
            "wall": (t0, t1)}


def distinct_experts(wl, M, n, skewed=False):
    """|U|, the distinct routed experts one M-token step streams, over n steps."""
    torch = wl.torch
    us = []
    for i in range(n):
        wl.step(i, M, skewed=skewed)
        torch.cuda.synchronize()
        us.append(len(set(wl.ids[M].cpu().numpy().reshape(-1).tolist())))
    return {"mean": statistics.fmean(us), "min": min(us), "max": max(us), "steps": n}


def read_ceiling(B, buf, reps=20):
    """This GPU's practical HBM read rate: moe_stream_read over a buffer larger
    than L2, CUDA events, best and median of `reps` runs."""
    import torch
    sink = torch.zeros((1,), dtype=torch.int32, device=buf.device)
    nbytes = buf.numel() * buf.element_size() // 16 * 16
    for _ in range(3):
        B.moe_stream_read(buf, sink)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        B.moe_stream_read(buf, sink)
        e1.record()
        ts.append((e0, e1))
    torch.cuda.synchronize()
    us = [a.elapsed_time(b) * 1e3 for a, b in ts]
    return {"kernel": "moe_stream_read", "bytes": nbytes, "gbs_best": nbytes / (min(us) * 1e-6) / 1e9,
            "gbs_median": nbytes / (statistics.median(us) * 1e-6) / 1e9}


def time_e2e(wl, M, steps, warmup, dist, device):
    """The same steps through the public API with host buffers: each step copies
    its two hidden states from pinned host memory and reads back the MoE output
    and the top-k ids and values."""
    torch = wl.torch
    s = wl.s
    hx = [wl.x[M][i % N_X].cpu().pin_memory() for i in range(N_X)]
    dx_m = torch.empty((M, s.hidden), dtype=torch.bfloat16, device=device)
    dx_h = torch.empty((M, s.hidden), dtype=torch.bfloat16, device=device)
    h_out = torch.empty((M, s.hidden), dtype=torch.float32).pin_memory()
    h_ids = torch.empty((M, HEAD_TOPK), dtype=torch.int32).pin_memory()
    h_vals = torch.empty((M, HEAD_TOPK), dtype=torch.float32).pin_memory()

    def one(i):
        dx_m.copy_(hx[i % N_X], non_blocking=True)
        dx_h.copy_(hx[(i + 1) % N_X], non_blocking=True)
        wl.step(i, M, x_moe=dx_m, x_head=dx_h)
        h_out.copy_(wl.out[M], non_blocking=True)
        h_ids.copy_(wl.tk_ids[M], non_blocking=True)
        h_vals.copy_(wl.tk_vals[M], non_blocking=True)

    for i in range(warmup):
        one(i)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        one(warmup + i)
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    h2d = 2 * M * s.hidden * 2
    d2h = M * s.hidden * 4 + M * HEAD_TOPK * 8
    return ms * 1e3 / steps, h2d, d2h


def time_bf16_head(wl, M, steps):
    torch = wl.torch
    for i in range(5):
        wl.bf16_head(i, M)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(steps):
        wl.bf16_head(i, M)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / steps


# ---------------------------------------------------------------------------
# the decode-step stream: 16 layers + LM head, greedy feedback
# ---------------------------------------------------------------------------

STREAM_LAYERS = 16


class Stream:
    """A stack of 16 Ling-shaped layers (each re-routed from the previous
    layer's RMS-normalised output), the FP8 LM head and a bf16 embedding table;
    one step embeds the previous greedy tokens, runs the stack and the head."""

    def __init__(self, B, I, seed, device, M, head, x_table=None):
        import torch
        self.B, self.torch, self.M = B, torch, M
        s, h = I.LING_MOE, I.LING_HEAD
        self.s, self.h = s, h
        self.layers = []
        for l in range(STREAM_LAYERS):
            router = I.router_weight(seed, s.experts, s.hidden, layer=100 + l, device=device)
            banks, shared = [], []
            for kind in ("gate", "up", "down"):
                rows, cols = (s.inter, s.hidden) if kind != "down" else (s.hidden, s.inter)
                st = I.normal(seed, f"S{l}/bank/{kind}", (s.experts, rows, cols), I.WEIGHT_STD, device=device)
                banks.append(B.moe_quantize_mxfp4(st))
                del st
                shared.append(B.moe_quantize_mxfp4(I.expert_matrix(seed, s, "shared", kind, layer=100 + l,
                                                                    device=device)))
            self.layers.append((router, B.moe_pack_experts(tuple(banks)), B.moe_pack_experts(tuple(shared))))
            del banks, shared
        self.head = head
        self.table = I.normal(seed, "embed", (h.vocab, h.hidden), 1.0, device=device)
        self.ids = torch.arange(M, dtype=torch.int32, device=device).view(M, 1).repeat(1, 1) * 7 + 3
        self.x = torch.empty((M, s.hidden), dtype=torch.bfloat16, device=device)
        self.y = torch.empty((M, s.hidden), dtype=torch.float32, device=device)
        self.tv = torch.empty((M, 1), dtype=torch.float32, device=device)
        self.moe_ws = B.new_workspace(B.moe_workspace_bytes(M, s.top_k, s.experts, s.hidden, s.inter), device)
        self.head_ws = B.new_workspace(B.lmhead_workspace_bytes(M, 1, h.vocab, h.hidden), device)
        torch.cuda.synchronize()

    def step(self):
        B = self.B
        B.moe_embed_gather(self.table, self.ids, self.x, ids_stride=1)
        for router, banks, shared in self.layers:
            B.moe_decode(self.x, router, None, banks, shared, self.s.top_k, self.y, workspace=self.moe_ws)
            B.moe_rmsnorm_bf16(self.y, self.x, 1e-6)
        B.lmhead_decode(self.x, self.head, 1, self.ids, self.tv, None, workspace=self.head_ws)

    def run(self, steps, warmup=3):
        """Device time per step; the step is captured as one CUDA graph when
        capture works, else launched directly."""
        torch = self.torch
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        graph = None
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step()
            graph = g
        except Exception as exc:  # capture unsupported: direct launches
            graph = None
            capture_error = str(exc).splitlines()[0]
        run = graph.replay if graph is not None else self.step
        for _ in range(warmup):
            run()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(steps):
            run()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / steps
        out = {"steps": steps, "us_per_step": us, "cuda_graph": graph is not None}
        if graph is None:
            out["capture_error"] = capture_error
        return out


def stream_leg(wl, B, I, A, seed, device, steps):
    res = {}
    for M in (1, 4):
        st = Stream(B, I, seed, device, M, wl.head)
        r = st.run(steps if M == 1 else max(steps // 4, 1))
        if M == 1:
            nbytes = STREAM_LAYERS * A.moe_layer_bytes(I.LING_MOE, I.LING_MOE.top_k) + A.lmhead_fp8_bytes(I.LING_HEAD)
            r["algorithmic_bytes_per_step"] = nbytes
            r["achieved_gbs"] = nbytes / (r["us_per_step"] * 1e-6) / 1e9
        res[f"m{M}"] = r
        del st
        import torch
        torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def _run_threads(fn, items, n_threads):
    """fn over items on n_threads Python threads: the oracle's C calls release
    the interpreter lock, so the threads run on separate cores."""
    if n_threads <= 1 or len(items) <= 1:
        return [fn(it) for it in items]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=n_threads) as ex:
        return list(ex.map(fn, items))


class OracleBench:
    """The oracle (plain C, fp64) on the benchmark's own configurations, on the
    host's cores: the tiny layer + tiny head in full (C0), the Ling layer at
    M=1 and M=4 (C1: router, then every selected expert and the shared expert
    in full), and the full 157,184 x 2,560 FP8 head (C3).  Work is split into
    independent calls -- experts per (token, expert) pair, head rows in slabs
    -- that threads run side by side; quantisation is load time, untimed."""

    def __init__(self, seed: int, head_rows: int | None = None):
        import numpy as np
        import torch

        import oracle
        from moe_decode_gemv_b200 import inputs as I
        self.np, self.torch, self.O, self.I, self.seed = np, torch, oracle.load(), I, seed
        self.host_cores = os.cpu_count() or 1
        self.cache = {}
        self.router = {s: I.router_weight(seed, s.experts, s.hidden).numpy() for s in (I.TINY_MOE, I.LING_MOE)}
        self.heads = {}
        self.head_rows = head_rows  # None: the full head
        self._head(I.TINY_HEAD, None)
        self._head(I.LING_HEAD, head_rows)

    def _head(self, h, rows):
        """The FP8 head quantised by the oracle, slab by slab (all cores)."""
        I = self.I
        V = h.vocab if rows is None else min(rows, h.vocab)
        slab = 8192
        starts = list(range(0, V, slab))

        def quant(r0):
            r1 = min(V, r0 + slab)
            w = I.normal(self.seed, f"lmhead/{r0}", (r1 - r0, h.hidden), I.WEIGHT_STD)
            return self.O.fp8_rowquant(w)

        parts = _run_threads(quant, starts, self.host_cores)
        self.heads[h] = (self.np.concatenate([q for q, _ in parts]), self.np.concatenate([sc for _, sc in parts]))

    def _expert(self, s, e):
        key = (s, e)
        if key not in self.cache:
            self.cache[key] = {k: self.O.mxfp4_quantize(self.I.expert_matrix(self.seed, s, e, k))
                               for k in ("gate", "up", "down")}
        return self.cache[key]

    def moe_step(self, s, x, n_threads) -> float:
        """Seconds for one layer step of x [M, H] bf16: router, top-k, the
        selected experts and the shared expert, weighted combine."""
        np = self.np
        M = x.shape[0]
        _, ids, w = self.O.router(x, self.router[s], None, s.top_k)
        for e in set(ids.reshape(-1).tolist()) | {"shared"}:
            self._expert(s, e)  # quantisation is load time: outside the timed region
        t0 = time.perf_counter()
        _, ids, w = self.O.router(x, self.router[s], None, s.top_k)
        tasks = [(m, int(ids[m, r]), float(w[m, r])) for m in range(M) for r in range(s.top_k)]
        tasks += [(m, "shared", 1.0) for m in range(M)]

        def run(t):
            m, e, wt = t
            q = self._expert(s, e)
            out, _ = self.O.expert_mlp(x[m:m + 1], q["gate"], q["up"], q["down"])
            return m, wt * out

        y = np.zeros((M, s.hidden))
        for m, part in _run_threads(run, tasks, n_threads):
            y[m] += part
        return time.perf_counter() - t0

    def head_step(self, h, x, k, n_threads) -> float:
        """Seconds for the head on x [M, H] bf16: logits over the head's rows
        (slabs in parallel), then the top-k of each token."""
        np = self.np
        q, sc = self.heads[h]
        V = q.shape[0]
        slab = max(1024, -(-V // max(n_threads, 1)))
        t0 = time.perf_counter()
        parts = _run_threads(lambda r0: self.O.lmhead_fp8(x, q[r0:r0 + slab], sc[r0:r0 + slab]),
                             list(range(0, V, slab)), n_threads)
        logits = np.concatenate(parts, axis=1)
        for m in range(x.shape[0]):
            self.O.topk(logits[m], k)
        return time.perf_counter() - t0

    def step_us(self, M: int, n_threads: int, tag: str) -> dict:
        """One step of the Ling layer + head at M tokens: us for each part."""
        I = self.I
        x = I.hidden_states(self.seed, M, I.LING_MOE.hidden, tag=tag)
        moe = self.moe_step(I.LING_MOE, x, n_threads)
        head = self.head_step(I.LING_HEAD, x, HEAD_TOPK, n_threads)
        scale = I.LING_HEAD.vocab / self.heads[I.LING_HEAD][0].shape[0]  # 1 for the full head
        return {"moe_us": moe * 1e6, "head_us": head * scale * 1e6, "step_us": (moe + head * scale) * 1e6}

    def tiny_us(self, n_threads: int) -> float:
        I = self.I
        x = I.hidden_states(self.seed, 1, I.TINY_MOE.hidden, tag="cpu-tiny")
        return (self.moe_step(I.TINY_MOE, x, n_threads) + self.head_step(I.TINY_HEAD, x, HEAD_TOPK, n_threads)) * 1e6

    def describe(self, n_threads):
        rows = "all 157,184 rows" if self.head_rows is None else f"the first {self.head_rows} rows, scaled to 157,184"
        return (f"oracle (plain C, fp64) on {n_threads} thread(s) of {self.host_cores} host cores: Ling layer in full "
                f"(router, every selected expert and the shared expert, combine) + FP8 head over {rows} + top-{HEAD_TOPK}")


def cpu_baseline(seed, reps=2):
    """The oracle timed on the host's cores, 1 thread and all of them: C0 in
    full, C1 (Ling layer) and C3 (Ling head) at M=1 and M=4, `reps` steps
    each (median)."""
    ob = OracleBench(seed)
    T = ob.host_cores
    detail = {}
    for n in sorted({1, T}):
        d = {"C0_tiny_step_us": statistics.median(ob.tiny_us(n) for _ in range(reps))}
        for M in (1, 4):
            runs = [ob.step_us(M, n, tag=f"cpu{M}-{r}") for r in range(reps)]
            d[f"C1_moe_m{M}_us"] = statistics.median(r["moe_us"] for r in runs)
            d[f"C3_head_m{M}_us"] = statistics.median(r["head_us"] for r in runs)
            d[f"step_m{M}_us"] = statistics.median(r["step_us"] for r in runs)
        detail[f"{n}_threads"] = d
    best = detail[f"{T}_threads"]
    return {"value": best["step_m1_us"], "unit": UNIT, "cores": T, "host_cores": T, "kind": "oracle",
            "sample": ob.describe(T) + f"; median of {reps} steps per configuration; 1-thread timings in detail",
            "detail": detail}


def reference_arm(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    budget = 150.0
    probe = OracleBench(args.seed, head_rows=8192)
    T = probe.host_cores
    per = probe.step_us(1, T, tag="ref-probe")["step_us"] * 1e-6  # the full step, estimated from 8,192 head rows
    total = args.steps + args.warmup
    rows = None if per * total <= budget else max(8192, int(157184 * budget / (per * total)) // 8192 * 8192)
    ob = OracleBench(args.seed, head_rows=rows)
    for i in range(args.warmup):
        ob.step_us(1, T, tag=f"ref{i}")
    times = [ob.step_us(1, T, tag=f"ref{args.warmup + i}")["step_us"] for i in range(args.steps)]
    us = statistics.median(times)
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(),
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": T, "host_cores": T, "kind": "oracle",
                             "sample": ob.describe(T)},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# roofline bookkeeping
# ---------------------------------------------------------------------------

FALLBACK_HBM_GBS = 6650.0  # an earlier copy-bandwidth measurement on this kind of B200


def measured_peaks():
    """The HBM copy bandwidth the roofline divides by: the measured figure
    from MEASURED_PEAKS.json (`hbm_gbs`, a number or an object with a
    `value`), else the fallback, with the reason in the kind string."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(p):
        return FALLBACK_HBM_GBS, "fallback"
    try:
        with open(p) as f:
            v = json.load(f)["hbm_gbs"]
        if isinstance(v, dict):
            v = v["value"]
        v = float(v)
        if not (v > 0 and v < 1e5):
            raise ValueError(f"hbm_gbs = {v}")
        return v, "measured"
    except (OSError, ValueError, KeyError, TypeError) as exc:
        return FALLBACK_HBM_GBS, f"fallback (MEASURED_PEAKS.json unreadable: {type(exc).__name__})"


def source_code_only(text: str) -> str:
    """C/CUDA source without its comments, whitespace runs collapsed: what
    the compiler sees, so that editing a comment keeps a profile valid."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":                       # a string or character literal, copied whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):       # a line comment
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):       # a block comment
            j = text.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of the LM-head kernel's code (comments and layout excluded)."""
    h = hashlib.sha256()
    for name in ("lmhead_fp8.cu", "common.cuh"):
        with open(os.path.join(ROOT, "moe_decode_gemv_b200", "csrc", name), encoding="utf-8") as f:
            h.update(source_code_only(f.read()).encode())
            h.update(b"\0")
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per launch of the LM-head kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "lmhead_fp8_157184x2560_m1_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    try:
        return float(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def workload_config():
    return {"workload": "Ling-shaped MoE layer (H=2560, I=768, E=512, top-8, +1 shared, MXFP4) + online-FP8 LM head "
                        "(157184x2560, top-29 + logits), M=1 decode step",
            "hidden": 2560, "expert_inter": 768, "experts": 512, "top_k": 8, "shared_experts": 1,
            "vocab": 157184, "head_top_k": HEAD_TOPK, "M": 1, "layer_copies_rotated": N_LAYERS,
            "l2": "inputs larger than L2: 8 rotating layer copies and the 403 MB head in every step",
            "weights": "experts MXFP4 (E2M1 + E8M0/32), router fp32, LM head E4M3 + fp32 row scale",
            "activations": "bf16 in, fp32 accumulate and out"}


def main():
    args = parse()
    if args.impl == "reference":
        return reference_arm(args)
    world, rank, local = dist_env()
    import torch
    dist = dist_init(world, local)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    from moe_decode_gemv_b200 import accounting as A
    from moe_decode_gemv_b200 import binding as B
    from moe_decode_gemv_b200 import inputs as I

    sampler = ClockSampler(local)  # started early: it samples through every timed region below
    n_layers = 0 if args.only == "head" else args.layers
    wl = Workload(B, I, args.seed + rank, device, n_layers=n_layers, head=args.only != "moe")
    m1 = time_steps(wl, 1 if args.only == "all" else args.profile_m, args.steps, args.warmup, dist, device)
    sampler.mark(*m1["wall"])
    clocks = sampler.stop()
    if args.only != "all":
        # profiling aid: no end-to-end, M=4 or CPU legs
        print(json.dumps({"only": args.only, "M": args.profile_m, "steps": args.steps, "per_step_us": m1["per_step_us"],
                          "moe_us_mean": m1["moe_us_mean"], "head_us_mean": m1["head_us_mean"], "clocks": clocks}))
        return 0
    e2e_us, h2d, d2h = time_e2e(wl, 1, args.steps, args.warmup, dist, device)
    m4 = {}
    if not args.no_m4:
        for regime, skewed in (("uniform", False), ("skewed", True)):
            m4[regime] = time_steps(wl, 4, max(args.steps // 2, 1), args.warmup, dist, device, skewed=skewed)
            m4[regime]["distinct_experts"] = distinct_experts(wl, 4, 32, skewed=skewed)
    bf16_head_us = time_bf16_head(wl, 1, 200)
    status = [B.moe_workspace_status(ws) for ws in list(wl.moe_ws.values()) + list(wl.head_ws.values())]
    if any(s != B.Status.OK for s in status):
        raise SystemExit(f"device status not OK: {status}")

    s, h = I.LING_MOE, I.LING_HEAD
    head_bytes = A.lmhead_fp8_bytes(h)
    moe_bytes_m1 = A.moe_layer_bytes(s, s.top_k)
    peak, peak_kind = measured_peaks()
    gbs = lambda nbytes, us: nbytes / (us * 1e-6) / 1e9
    achieved = gbs(head_bytes, m1["head_us_mean"])
    # the headline: median device time per M=1 step over all ranks' steps
    value = m1["step_us_median"] / world
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": m1["step_us_median"] / 1e3, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": workload_config(),
        "value_stats": {"median_us": m1["step_us_median"], "p10_us": m1["step_us_p10"], "p90_us": m1["step_us_p90"],
                        "back_to_back_mean_us": m1["per_step_us"], "steps": args.steps,
                        "block_steps": m1["block_steps"],
                        "timing": "CUDA events on the launching stream every block_steps steps; value = the median "
                                  "over blocks of the block time / block_steps; inputs larger than L2 (8 rotating "
                                  "layer copies + the 403 MB head per step)"},
        "arithmetic": "fp32 accumulate; MoE gate/up on tcgen05 block-scaled FP4 with x as eight E2M1 base-4 "
                      "digits per 32-block, down on f16 MMA with h as two f16 parts per 16-value slice; head x as "
                      "two E4M3 parts; weights MXFP4 (experts) and E4M3 + fp32 row scale (head)",
        "roofline": {"bound": "hbm", "kernel": "lmhead_fp8_kernel (FP8 LM head, M=1)", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": profiled_traffic(), "algorithmic_bytes_per_launch": head_bytes},
        "breakdown_m1": {"moe_us_mean": m1["moe_us_mean"], "moe_us_median": m1["moe_us_median"],
                         "moe_us_p10": m1["moe_us_p10"], "moe_us_p90": m1["moe_us_p90"],
                         "head_us_mean": m1["head_us_mean"], "head_us_median": m1["head_us_median"],
                         "head_us_p10": m1["head_us_p10"], "head_us_p90": m1["head_us_p90"],
                         "moe_bytes": moe_bytes_m1, "moe_gbs": gbs(moe_bytes_m1, m1["moe_us_mean"]),
                         "moe_frac": gbs(moe_bytes_m1, m1["moe_us_mean"]) / peak,
                         "head_gbs": achieved, "head_frac": achieved / peak},
        "bf16_head_us": bf16_head_us,
        "bf16_head_gbs": gbs(A.lmhead_bf16_bytes(h), bf16_head_us),
        "clocks": clocks,
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * args.steps,  # one MoE and one LM-head kernel per timed step (pass 1)
        "path": B.moe_query_path(),
    }
    for regime, r in m4.items():
        u = r["distinct_experts"]["mean"]
        mb = A.moe_layer_bytes(s, u)
        line.setdefault("m4", {})[regime] = {
            "step_us_median": r["step_us_median"], "step_us_p10": r["step_us_p10"], "step_us_p90": r["step_us_p90"],
            "moe_us_mean": r["moe_us_mean"], "head_us_mean": r["head_us_mean"], "steps": max(args.steps // 2, 1),
            "distinct_experts": r["distinct_experts"], "moe_bytes_at_mean_U": mb,
            "moe_gbs": gbs(mb, r["moe_us_mean"]), "moe_frac": gbs(mb, r["moe_us_mean"]) / peak,
            "head_gbs": gbs(head_bytes, r["head_us_mean"]), "head_frac": gbs(head_bytes, r["head_us_mean"]) / peak}
    line["read_ceiling"] = read_ceiling(B, wl.head.q)
    if not args.no_stream:
        try:
            line["stream_16_layers"] = stream_leg(wl, B, I, A, args.seed + rank, device, args.stream_steps)
        except Exception as exc:  # the headline numbers above stand without this leg
            line["stream_16_layers"] = {"error": f"{type(exc).__name__}: {str(exc).splitlines()[0][:200]}"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = cpu_baseline(args.seed)
        except Exception as exc:  # the GPU numbers above stand without the host leg
            line["cpu_baseline"] = {"kind": "oracle", "error": f"{type(exc).__name__}: {str(exc).splitlines()[0][:200]}"}
    if dist is not None:
        dist.barrier()
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
