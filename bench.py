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
    """nvidia-smi sampling of SM clock and throttle reasons during a window."""

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.samples = []
        self.proc = None
        self.window = None
        cmd = ["nvidia-smi", "-i", str(gpu_index),
               "--query-gpu=timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", str(period_ms)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def _read(self):
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
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.proc is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t0, t1 = self.window if self.window else (0, 1e18)
        inwin = [s for s in self.samples if t0 - 0.05 <= s[0] <= t1 + 0.05] or self.samples[-3:]
        reasons = set()
        for s in inwin:
            for bit, name in REASON_BITS.items():
                if s[4] & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in inwin), "sm_max_mhz": max(s[2] for s in inwin),
                "power_w_max": max(s[3] for s in inwin), "samples": len(inwin), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# workload on the GPU
# ---------------------------------------------------------------------------

class Workload:
    def __init__(self, B, I, seed: int, device, n_layers: int = N_LAYERS, head: bool = True):
        import torch
        self.B, self.torch = B, torch
        s, h = I.LING_MOE, I.LING_HEAD
        self.s, self.h = s, h
        self.layers = []
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

    def step(self, i: int, M: int, ev=None, x_moe=None, x_head=None):
        """One decode step: MoE layer (layer i mod 8) then the LM head."""
        B = self.B
        xm = self.x[M][i % N_X] if x_moe is None else x_moe
        xh = self.x[M][(i + 1) % N_X] if x_head is None else x_head
        if ev is not None:
            ev[0].record()
        if self.layers:
            router, banks, shared = self.layers[i % len(self.layers)]
            B.moe_decode(xm, router, None, banks, shared, self.s.top_k, self.out[M], self.ids[M], self.w[M],
                         workspace=self.moe_ws[M])
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


def time_steps(wl, M, steps, warmup, dist, device):
    """Device time of `steps` steps: total, MoE part and head part (us)."""
    torch = wl.torch
    for i in range(warmup):
        wl.step(i, M)
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(steps):
        wl.step(warmup + i, M, ev=evs[i])
    torch.cuda.synchronize()
    t1 = time.time()
    total_ms = evs[0][0].elapsed_time(evs[-1][2])
    moe = [e[0].elapsed_time(e[1]) * 1e3 for e in evs]
    head = [e[1].elapsed_time(e[2]) * 1e3 for e in evs]
    total_ms = max_over_ranks(total_ms, dist, device)
    q = lambda v, f: sorted(v)[min(len(v) - 1, int(f * len(v)))]
    return {"total_us": total_ms * 1e3, "per_step_us": total_ms * 1e3 / steps,
            "moe_us_mean": statistics.fmean(moe), "moe_us_median": statistics.median(moe),
            "moe_us_p10": q(moe, 0.1), "moe_us_p90": q(moe, 0.9),
            "head_us_mean": statistics.fmean(head), "head_us_median": statistics.median(head),
            "head_us_p10": q(head, 0.1), "head_us_p90": q(head, 0.9),
            "wall": (t0, t1)}


def distinct_experts(wl, M, n):
    """|U|, the distinct routed experts one M-token step streams, over n steps."""
    torch = wl.torch
    us = []
    for i in range(n):
        wl.step(i, M)
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

class OracleStep:
    """The oracle on a bounded sample of one decode step: the full router for
    one token, a 32-row slice of each of the 8 selected experts and of the
    shared expert, and a slice of the LM head's rows.  The measured time is
    scaled by the inverse of each slice's fraction of its part of the step."""

    def __init__(self, seed: int, head_rows: int = 1024, expert_rows: int = 32):
        import numpy as np

        import oracle
        from moe_decode_gemv_b200 import inputs as I
        self.np, self.O, self.I = np, oracle.load(), I
        s, h = I.LING_MOE, I.LING_HEAD
        self.s, self.h = s, h
        self.expert_rows, self.head_rows = expert_rows, head_rows
        self.router = I.router_weight(seed, s.experts, s.hidden).numpy()
        self.x = [I.hidden_states(seed, 1, s.hidden, tag=f"cpu{i}") for i in range(8)]
        self.xb = [t.view(__import__("torch").int16).numpy().view(np.uint16) for t in self.x]
        # LM-head slices, quantised by the oracle (load time, untimed)
        self.head_slices = []
        for j in range(4):
            r0 = (j * 37 * 1024) % (h.vocab - head_rows)
            w = I.normal(seed, f"lmhead/{r0}", (head_rows, h.hidden), I.WEIGHT_STD)
            wb = w.view(__import__("torch").int16).numpy().view(np.uint16)
            self.head_slices.append(self.O.fp8_rowquant(wb))
        self.expert_cache = {}

    def _expert_slice(self, e):
        """Gate/up rows [0, r) and down columns [0, r) of expert e, quantised."""
        if e in self.expert_cache:
            return self.expert_cache[e]
        np, I, s, r = self.np, self.I, self.s, self.expert_rows
        import torch
        q = {}
        for kind in ("gate", "up", "down"):
            m = I.expert_matrix(0, s, e, kind)
            m = m[:r] if kind != "down" else m[:, :r].contiguous()
            q[kind] = self.O.mxfp4_quantize(m.view(torch.int16).numpy().view(np.uint16))
        self.expert_cache[e] = q
        return q

    def prepare(self, i):
        _, ids, _ = self.O.router(self.xb[i % 8], self.router, None, self.s.top_k)
        for e in list(ids[0]) + ["shared"]:
            self._expert_slice(e if e == "shared" else int(e))
        return ids

    def run(self, i) -> float:
        """Seconds of oracle work scaled to one full step."""
        O, s, h = self.O, self.s, self.h
        xb = self.xb[i % 8]
        t0 = time.perf_counter()
        _, ids, _ = O.router(xb, self.router, None, s.top_k)
        t1 = time.perf_counter()
        for e in list(ids[0]) + ["shared"]:
            q = self._expert_slice(e if e == "shared" else int(e))
            O.expert_mlp(xb, q["gate"], q["up"], q["down"])
        t2 = time.perf_counter()
        qh, sh = self.head_slices[i % len(self.head_slices)]
        logits = O.lmhead_fp8(xb, qh, sh)
        O.topk(logits[0], HEAD_TOPK)
        t3 = time.perf_counter()
        return (t1 - t0) + (t2 - t1) * (s.inter / self.expert_rows) + (t3 - t2) * (h.vocab / self.head_rows)

    def describe(self):
        return (f"oracle (plain C, fp64, 1 thread) per step: full router for 1 token; gate/up rows and down "
                f"columns [0,{self.expert_rows}) of the 8 routed + shared experts, scaled x{self.s.inter // self.expert_rows}; "
                f"LM-head rows slice of {self.head_rows} of {self.h.vocab}, scaled x{self.h.vocab / self.head_rows:.1f}")


def cpu_baseline(seed, budget_s=15.0):
    st = OracleStep(seed)
    for i in range(8):
        st.prepare(i)
    times = []
    t_start = time.perf_counter()
    i = 0
    while time.perf_counter() - t_start < budget_s or i < 3:
        times.append(st.run(i))
        i += 1
    us = statistics.fmean(times) * 1e6
    return {"value": us, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": st.describe() + f"; {i} steps"}


def reference_arm(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    budget = 120.0
    st = OracleStep(args.seed)
    for i in range(8):
        st.prepare(i)
    # size the sample so that warmup + steps fit the budget
    probe = [st.run(i) for i in range(2)]
    t_probe = time.perf_counter()
    st.run(2)
    per = time.perf_counter() - t_probe
    total = args.steps + args.warmup
    if per * total > budget:
        shrink = max(1, int(per * total / budget) + 1)
        st.head_rows = max(64, st.head_rows // shrink)
        st.head_slices = [(q[: st.head_rows], s[: st.head_rows]) for q, s in st.head_slices]
    for i in range(args.warmup):
        st.run(i)
    times = [st.run(args.warmup + i) for i in range(args.steps)]
    us = statistics.fmean(times) * 1e6
    line = {"impl": "reference", "metric": METRIC, "value": us, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(),
            "cpu_baseline": {"value": us, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": st.describe()},
            "e2e": {"value": us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    del probe
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# roofline bookkeeping
# ---------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in ("lmhead_kernels.cu", "common.cuh"):
        with open(os.path.join(ROOT, "moe_decode_gemv_b200", "csrc", name), "rb") as f:
            h.update(f.read())
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

    n_layers = 0 if args.only == "head" else args.layers
    wl = Workload(B, I, args.seed + rank, device, n_layers=n_layers, head=args.only != "moe")
    sampler = ClockSampler(local)
    m1 = time_steps(wl, 1, args.steps, args.warmup, dist, device)
    sampler.mark(*m1["wall"])
    clocks = sampler.stop()
    if args.only != "all":
        # profiling aid: no end-to-end, M=4 or CPU legs
        print(json.dumps({"only": args.only, "steps": args.steps, "per_step_us": m1["per_step_us"],
                          "moe_us_mean": m1["moe_us_mean"], "head_us_mean": m1["head_us_mean"], "clocks": clocks}))
        return 0
    e2e_us, h2d, d2h = time_e2e(wl, 1, args.steps, args.warmup, dist, device)
    m4 = None if args.no_m4 else time_steps(wl, 4, max(args.steps // 2, 1), args.warmup, dist, device)
    bf16_head_us = time_bf16_head(wl, 1, 200)
    status = [B.moe_workspace_status(ws) for ws in list(wl.moe_ws.values()) + list(wl.head_ws.values())]
    if any(s != B.Status.OK for s in status):
        raise SystemExit(f"device status not OK: {status}")

    head_bytes = A.lmhead_fp8_bytes(I.LING_HEAD)
    moe_bytes_m1 = A.moe_layer_bytes(I.LING_MOE, I.LING_MOE.top_k)
    peak, peak_kind = measured_peaks()
    achieved = head_bytes / (m1["head_us_mean"] * 1e-6) / 1e9
    value = m1["total_us"] / (args.steps * world)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": m1["per_step_us"] / 1e3, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic", "config": workload_config(),
        "roofline": {"bound": "hbm", "kernel": "lmhead_fp8_tiled_kernel (FP8 LM head, M=1)", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": profiled_traffic(), "algorithmic_bytes_per_launch": head_bytes},
        "breakdown_m1": {"moe_us_mean": m1["moe_us_mean"], "moe_us_median": m1["moe_us_median"],
                         "moe_us_p10": m1["moe_us_p10"], "moe_us_p90": m1["moe_us_p90"],
                         "head_us_mean": m1["head_us_mean"], "head_us_median": m1["head_us_median"],
                         "head_us_p10": m1["head_us_p10"], "head_us_p90": m1["head_us_p90"],
                         "moe_bytes": moe_bytes_m1,
                         "moe_gbs": moe_bytes_m1 / (m1["moe_us_mean"] * 1e-6) / 1e9,
                         "head_gbs": achieved},
        "bf16_head_us": bf16_head_us,
        "bf16_head_gbs": A.lmhead_bf16_bytes(I.LING_HEAD) / (bf16_head_us * 1e-6) / 1e9,
        "clocks": clocks,
        "e2e": {"value": e2e_us, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * args.steps,  # one MoE and one LM-head kernel per timed step
        "path": B.moe_query_path(),
    }
    if m4 is not None:
        line["m4"] = {"us_per_step": m4["per_step_us"], "moe_us_mean": m4["moe_us_mean"],
                      "head_us_mean": m4["head_us_mean"], "steps": max(args.steps // 2, 1),
                      "distinct_experts": distinct_experts(wl, 4, 16)}
    line["read_ceiling"] = read_ceiling(B, wl.head.q)
    if not args.no_stream:
        try:
            line["stream_16_layers"] = stream_leg(wl, B, I, A, args.seed + rank, device, args.stream_steps)
        except Exception as exc:  # the headline numbers above stand without this leg
            line["stream_16_layers"] = {"error": f"{type(exc).__name__}: {str(exc).splitlines()[0][:200]}"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.seed)
    if dist is not None:
        dist.barrier()
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
