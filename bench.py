#!/usr/bin/env python
"""Benchmark of Maglev's injected sliding-window attention on B200.

Headline: fwd+bwd TFLOP/s of one d20 decoder layer (B=4, T=2048, d=1280,
10 heads x 128, window 512, bf16): memory projection, injection, banded
attention, consistency loss (lambda = 0.1) and the full backward, per step.
Alongside: recurrent decode tokens/s (64 sequences, 20 layers, 512-entry
rings), the dominant kernel's roofline, clocks, an end-to-end number through
host buffers, and the CPU oracle timed on this host.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch with torch.distributed.run: every rank runs an independent
replica on its own GPU (weak scaling, no collective on the data path); the
time is the max over ranks.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "Injected-SWA attn fwd+bwd TFLOP/s & % bf16 peak; decode tokens/s"
LAYER = dict(B=4, T=2048, H=10, hd=128, d=1280, W=512, lam=0.1)
DECODE = dict(B=64, L=20, H=10, hd=128, d=1280, W=512, first_pos=512)
STACK = dict(B=8, T=2048, H=10, hd=128, L=20, W=512, lam=0.1)
# LM head over the memory states of the d20 layer's tokens; the pages give no
# vocabulary size, 65,536 stands in
LMHEAD = dict(N=8192, d=1280, V=65536, softcap=15.0)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Datasheet dense peaks of one B200 (context beside the measured peaks).
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}

# DRAM bytes (read + write) per launch, as stored from an ncu capture of the
# kernel at the benchmark's shape (dram__bytes_read.sum + dram__bytes_write.sum);
# each entry records the sha256 of the kernel source it was taken on and is
# ignored (traffic null) once that source changes. The bench line marks these
# figures "traffic_source": "stored ncu capture", since they are not measured
# during the run.
NCU_TRAFFIC: dict[str, dict] = {
    "attn_bwd_tc": {"bytes": 164081408, "src": "tc_attn_bwd.cu", "src_sha": "1673693a89fbd72f"},
    "attn_fwd_tc": {"bytes": 63595264, "src": "tc_attn_fwd.cu", "src_sha": "cdc1badd0e6a9b5c"},
    "decode_step": {"bytes": 171966464, "src": "decode.cu", "src_sha": "188f1e09ac4c8bae"},
}

def stored_traffic(name: str):
    """The stored ncu DRAM bytes of `name` if taken on its current source, else None."""
    tr = NCU_TRAFFIC.get(name)
    return tr["bytes"] if tr and tr.get("src_sha") == src_sha(tr.get("src", "")) else None


# --------------------------------------------------------------------------- work model
def window_pairs(T: int, W: int) -> int:
    """(query, key) pairs inside the window: sum_i min(i + 1, W)."""
    if T <= W:
        return T * (T + 1) // 2
    return W * (W + 1) // 2 + (T - W) * W


def layer_flops(B, T, H, hd, d, W):
    pairs = window_pairs(T, W) * B * H
    attn_fwd = 4.0 * hd * pairs                  # QK^T and PV
    attn_bwd = 2.5 * attn_fwd                     # S recompute, dP, dV, dK, dQ
    proj_fwd = 2.0 * B * T * d * (2 * H * hd)     # [B*T, d] x [d, 2D]
    proj_bwd = 2.0 * proj_fwd                     # dW and dm
    return {"attn_fwd": attn_fwd, "attn_bwd": attn_bwd, "proj_fwd": proj_fwd,
            "proj_bwd": proj_bwd, "total": attn_fwd + attn_bwd + proj_fwd + proj_bwd}


def stack_windows(c: dict):
    """Prefiller Q alternates sliding (W) and full (T) layers; decoder P is all W."""
    q = [c["W"] if l % 2 == 0 else c["T"] for l in range(c["L"])]
    return q, [c["W"]] * c["L"]


def stack_flops(c: dict) -> float:
    """Attention fwd+bwd of every Q and P layer plus one shared projection fwd+bwd."""
    B, T, H, hd = c["B"], c["T"], c["H"], c["hd"]
    d = H * hd
    q_w, p_w = stack_windows(c)
    tot = 0.0
    for w in q_w + p_w:
        f = layer_flops(B, T, H, hd, d, w)
        tot += f["attn_fwd"] + f["attn_bwd"]
    f = layer_flops(B, T, H, hd, d, c["W"])
    return tot + f["proj_fwd"] + f["proj_bwd"]


def kernel_work(name: str, cfg: dict) -> tuple[float, str]:
    """Algorithmic work of one launch of a traced kernel: (amount, unit)."""
    B, T, H, hd, d, W = (cfg[k] for k in ("B", "T", "H", "hd", "d", "W"))
    f = layer_flops(B, T, H, hd, d, W)
    D = H * hd
    table = {
        "mem_project_gemm": (f["proj_fwd"] / 2, "flop"),
        "mem_project_bwd_dm_gemm": (f["proj_fwd"], "flop"),
        "mem_project_bwd_dw_gemm": (f["proj_fwd"] / 2, "flop"),
        "attn_fwd": (f["attn_fwd"], "flop"),
        "attn_bwd_dq": (f["attn_bwd"] * 3 / 5, "flop"),
        "attn_bwd_dkdv": (f["attn_bwd"] * 4 / 5, "flop"),
        "attn_bwd": (f["attn_bwd"], "flop"),
        "attn_fwd_tc": (f["attn_fwd"], "flop"),
        "attn_bwd_tc": (f["attn_bwd"], "flop"),
        "mem_project_tc": (f["proj_fwd"], "flop"),
        "mem_project_bwd_dm_tc": (f["proj_fwd"], "flop"),
        "mem_project_bwd_dw_tc": (f["proj_fwd"], "flop"),
        "mem_project_bwd_tc": (2 * f["proj_fwd"], "flop"),  # dm and dW in one launch
        # reads q, k, v, R_k, R_v; writes q_rot, k_bar, v_bar (bf16)
        "inject_prep": (B * T * D * 2.0 * (5 + 3), "byte"),
        # reads dq_rot (fp32), dk_bar, dv_bar, k, v, R_k, R_v (bf16); writes dq, dk, dv, dR_k, dR_v
        "unmix": (B * T * D * (4 + 6 * 2 + 5 * 2.0), "byte"),
        # reads m, m', dm; writes dm (the layer step accumulates into dO)
        "consistency_loss": (B * T * D * 2.0 * 4, "byte"),
        # the same, plus the zeroed fp32 dQ accumulator (Delta itself is B*H*T floats)
        "consistency_loss_prep": (B * T * D * 12.0, "byte"),
        # reads O, dO (bf16); zeroes the fp32 dQ accumulator
        "attn_delta": (B * T * D * (2.0 * 2 + 4), "byte"),
    }
    return table.get(name, (0.0, "flop"))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_sha(fname: str) -> str:
    p = os.path.join(ROOT, "sliding_window_recurrent_b200", "csrc", fname)
    if not os.path.exists(p):
        return ""
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


# --------------------------------------------------------------------------- ranks
def max_over_ranks(dist, x: float, device) -> float:
    """The largest of every rank's x (identity without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest
    rank's time (weak scaling: each replica does the same work)."""
    return units_per_rank * world / (ms_max * 1e-3)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling (every 200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- our arm
def make_layer_inputs(torch, dev, seed):
    """Seeded inputs of the d20 layer, drawn on the host (synth) and copied once."""
    import synth
    wl = dict(synth.WORKLOADS["layer_bf16"])
    x = synth.layer_inputs(wl, seed)

    def to_dev(t):
        if isinstance(t, synth.Tensor):
            return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(t)).to(dev)

    return {k: to_dev(x[k]) for k in ("q", "k", "v", "gates", "m_shift", "w_mk", "w_mv", "target", "dout")}


class LayerStep:
    """One fwd + loss + bwd step of the d20 layer through the C ABI.

    The loss gradient is added in place to the upstream-gradient buffer, as a
    training step adds it to the dO it receives; the buffer is filled from the
    seeded dO once, outside the timed region (the added ~1e-6 per element is
    below half a bf16 ulp of the N(0,1) values, so steps do not drift)."""

    def __init__(self, torch, dev, inputs):
        from sliding_window_recurrent_b200.layer import InjectedSWALayer
        c = LAYER
        self.torch = torch
        self.x = inputs
        self.L = InjectedSWALayer(c["B"], c["T"], c["H"], c["hd"], c["d"], c["W"], dtype="bf16", device=dev)
        self.D = c["H"] * c["hd"]
        self.dout_total = inputs["dout"].clone()

    def __call__(self):
        x, L = self.x, self.L
        L.forward(x["q"], x["k"], x["v"], x["gates"], x["m_shift"], x["w_mk"], x["w_mv"])
        # the loss of the layer's own output, with the backward's first pass (Delta, dQ accumulator)
        L.consistency_prepare_bwd(x["target"], LAYER["lam"], self.dout_total)
        L.backward(x["k"], x["v"], self.dout_total, x["gates"], x["m_shift"], x["w_mk"], x["w_mv"], prepared=True)


def aggregate_profile(rows):
    agg: dict[str, list] = {}
    for name, k, ms in rows:
        a = agg.setdefault(name, [0, 0.0, 0])
        a[0] += 1
        a[1] += ms
        a[2] += k
    return agg


def capture_graph(torch, fn):
    """fn's launches captured once into a CUDA graph (after a side-stream run,
    as torch's graph capture wants)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def run_layer_bench(torch, dist, rank, world, dev, steps, warmup, peaks, peaks_src, gpu_uuid):
    """The step's launches are captured in a CUDA graph and replayed for the
    timed steps (no host gaps between the kernels). Right after the timed
    replays, the same number of eager steps run with the library's per-launch
    CUDA-event tracing on, on the launching stream: they give each kernel's
    average duration (a kernel's own duration does not depend on the gaps
    around it)."""
    import sliding_window_recurrent_b200 as mg
    c = LAYER
    x = make_layer_inputs(torch, dev, 1234 + rank)
    step = LayerStep(torch, dev, x)
    flops = layer_flops(c["B"], c["T"], c["H"], c["hd"], c["d"], c["W"])
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    n0 = mg.maglev_launch_count()
    graph = capture_graph(torch, step)
    per_step = (mg.maglev_launch_count() - n0) // 2  # the side-stream run and the capture
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    sampler = ClockSampler(gpu_uuid)
    sampler.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = per_step * steps
    clocks = sampler.stop()
    del graph
    mg.maglev_profile_report()  # drop any earlier records
    mg.maglev_profile_enable(True)
    for _ in range(steps):
        # the GPU waits ~2 ms first, so that the host has queued the whole step
        # and each event pair brackets its kernel alone, not a host gap
        torch.cuda._sleep(4_000_000)
        step()
    torch.cuda.synchronize()
    mg.maglev_profile_enable(False)
    prof = aggregate_profile(mg.maglev_profile_report())
    ms = e0.elapsed_time(e1) / steps
    ms_max = max_over_ranks(dist, ms, dev)
    if dist is not None:
        dist.barrier()
    # dominant kernel and its roofline
    dom = max(prof.items(), key=lambda kv: kv[1][1]) if prof else None
    roof = None
    if dom:
        name, (calls, tot_ms, nk) = dom
        work, unit = kernel_work(name, c)
        avg_ms = tot_ms / calls
        if unit == "flop":
            achieved = work / (avg_ms * 1e-3) / 1e12
            peak = peaks["bf16_tflops"]
            roof = {"kernel": name, "bound": "tensor", "achieved": round(achieved, 3), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 5)}
        else:
            achieved = work / (avg_ms * 1e-3) / 1e9
            peak = peaks["hbm_gbs"]
            roof = {"kernel": name, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                    "unit": "GB/s", "frac": round(achieved / peak, 5)}
        roof["traffic"] = stored_traffic(name)
        roof["traffic_source"] = "stored ncu capture of this kernel's current source" if roof["traffic"] else None
        roof["peak_source"] = f"{peaks_src} burst (MEASURED_PEAKS.json)" if peaks_src == "measured" else "fallback"
        key = "bf16_tflops" if unit == "flop" else "hbm_gbs"
        roof["spec_peak"] = SPEC_PEAKS[key]
        roof["frac_of_spec"] = round(roof["achieved"] / SPEC_PEAKS[key], 5)
        roof["avg_launch_ms"] = round(avg_ms, 5)
        roof["duration_source"] = "CUDA events around each launch, on its stream, over as many eager steps as timed"
        roof["work_per_launch"] = work
    kernels = {n: {"calls": v[0], "ms_total": round(v[1], 4), "share": round(v[1] / sum(w[1] for w in prof.values()), 4)}
               for n, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    return {"ms": ms_max, "ms_rank": ms, "flops": flops, "launches": launches, "clocks": clocks,
            "roofline": roof, "kernels": kernels, "step": step}


def run_layer_e2e(torch, dev, steps, warmup, step):
    """Same step with every step's inputs copied in from pinned host memory and
    the loss and parameter gradients copied out, inside the timed region. As an
    input pipeline that prefetches does, step i+1's inputs are copied on their
    own stream into a second set of device buffers while step i computes: each
    step waits for its own inputs, and a buffer set is refilled only after the
    step that last read it has finished. The results are read back after every
    step, on the compute stream."""
    names = ("q", "k", "v", "m_shift", "target", "dout", "w_mk", "w_mv", "gates")
    host = {n: step.x[n].cpu().pin_memory() for n in names}
    L = step.L
    outs = [L.loss, L.dw_mk, L.dw_mv, L.dgate]
    host_out = [o.cpu().pin_memory() for o in outs]
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = sum(o.numel() * o.element_size() for o in outs)
    compute = torch.cuda.current_stream()
    copy = torch.cuda.Stream(device=dev)
    sets = [dict(step.x), {n: torch.empty_like(t) for n, t in step.x.items()}]
    douts = [step.dout_total, torch.empty_like(step.dout_total)]
    ready = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]
    used = [False, False]
    x0, dout0 = step.x, step.dout_total

    def e2e_step(i):
        s = i % 2
        if used[s]:
            copy.wait_event(done[s])  # the step that last read this set has finished
        with torch.cuda.stream(copy):
            for n in names:  # this step's dO lands in the buffer the step accumulates into
                (douts[s] if n == "dout" else sets[s][n]).copy_(host[n], non_blocking=True)
            ready[s].record(copy)
        compute.wait_event(ready[s])
        step.x, step.dout_total = sets[s], douts[s]
        step()
        for o, h in zip(outs, host_out):
            h.copy_(o, non_blocking=True)
        done[s].record(compute)
        used[s] = True

    for i in range(max(1, warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    copy.wait_event(e0)  # every timed copy starts after e0
    for i in range(steps):
        e2e_step(i)
    e1.record(compute)
    torch.cuda.synchronize()
    step.x, step.dout_total = x0, dout0
    return e0.elapsed_time(e1) / steps, h2d, d2h


def run_layer_fwd_bench(torch, dev, steps, warmup, step):
    """Forward only (projection, injection, attention) of the same layer, as a
    replayed CUDA graph."""
    x, L = step.x, step.L

    def fwd():
        L.forward(x["q"], x["k"], x["v"], x["gates"], x["m_shift"], x["w_mk"], x["w_mv"])

    for _ in range(warmup):
        fwd()
    torch.cuda.synchronize()
    graph = capture_graph(torch, fwd)
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    c = LAYER
    f = layer_flops(c["B"], c["T"], c["H"], c["hd"], c["d"], c["W"])
    ms = e0.elapsed_time(e1) / steps
    return {"value": round((f["attn_fwd"] + f["proj_fwd"]) / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "gflop_per_step": round((f["attn_fwd"] + f["proj_fwd"]) / 1e9, 3),
            "workload": "d20 injected-SWA layer forward: B=4 T=2048 d=1280 H=10x128 W=512, bf16"}


def run_stack_bench(torch, dev, steps, warmup):
    """Prefiller Q (20 SLSL layers, no injection) + decoder P (20 injected
    layers) + shared projection + memory state + loss, fwd+bwd, B=8."""
    import sliding_window_recurrent_b200 as mg
    from sliding_window_recurrent_b200.stack import PrefillerDecoderStack
    c = STACK
    B, T, H, hd = c["B"], c["T"], c["H"], c["hd"]
    D = H * hd
    q_w, p_w = stack_windows(c)
    gen = torch.Generator(device=dev)
    gen.manual_seed(2468)
    bf = torch.bfloat16
    rn = lambda *s, std=1.0: (torch.randn(*s, generator=gen, device=dev) * std).to(bf)
    qi = [(rn(B, T, H, hd), rn(B, T, H, hd), rn(B, T, H, hd)) for _ in q_w]
    pi = [(rn(B, T, H, hd), rn(B, T, H, hd), rn(B, T, H, hd),
           torch.rand(4, H, generator=gen, device=dev) * 4 - 2) for _ in p_w]
    qd = [rn(B, T, H, hd) for _ in q_w]
    pd = [rn(B, T, H, hd) for _ in p_w]
    wk, wv = rn(D, D, std=D ** -0.5), rn(D, D, std=D ** -0.5)
    S = PrefillerDecoderStack(B, T, H, hd, q_w, p_w, lam=c["lam"], device=dev)
    step = lambda: S.step(qi, pi, qd, pd, wk, wv)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    n0 = mg.maglev_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    launches = mg.maglev_launch_count() - n0
    ms = e0.elapsed_time(e1) / steps
    mg.maglev_profile_enable(True)
    torch.cuda._sleep(20_000_000)  # the host queues the traced step while the GPU waits
    step()
    torch.cuda.synchronize()
    mg.maglev_profile_enable(False)
    prof = aggregate_profile(mg.maglev_profile_report())
    tot = sum(v[1] for v in prof.values())
    fl = stack_flops(c)
    out = {"value": round(fl / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 3),
           "gflop_per_step": round(fl / 1e9, 1), "gpu_launches": launches,
           "workload": f"prefiller Q 20 layers SLSL (W={c['W']}/{T}, no injection) + decoder P 20 injected "
                       f"layers (W={c['W']}) + shared projection + memory state + consistency loss, fwd+bwd, "
                       f"B={B} T={T} H={H}x{hd}, bf16",
           "kernels": {n: {"calls": v[0], "ms_total": round(v[1], 3), "share": round(v[1] / tot, 4)}
                       for n, v in sorted(prof.items(), key=lambda kv: -kv[1][1])}}
    del S, qi, pi, qd, pd
    torch.cuda.empty_cache()
    return out


def run_decode_bench(torch, dev, steps, warmup, peaks):
    """64 sequences x 20 layers; per layer the ring attention of the new token.
    The per-layer q/k/v come from a stand-in projection of RMSNorm(h_l) (torch
    matmul: the rest of the model is outside this path); the step is captured
    in a CUDA graph."""
    import sliding_window_recurrent_b200 as mg
    from sliding_window_recurrent_b200.layer import DecodeLayerState
    c = DECODE
    B, L, H, hd, d, W = c["B"], c["L"], c["H"], c["hd"], c["d"], c["W"]
    D = H * hd
    gen = torch.Generator(device=dev)
    gen.manual_seed(4321)
    bf = torch.bfloat16
    kr = [torch.randn(B, H, W, hd, generator=gen, device=dev, dtype=torch.float32).to(bf) for _ in range(L)]
    vr = [torch.randn(B, H, W, hd, generator=gen, device=dev, dtype=torch.float32).to(bf) for _ in range(L)]
    # per-layer stand-in projection weights, [3, d, D]: q | k | v = RMSNorm(h) W[i]
    wqkv = [(torch.randn(3, d, D, generator=gen, device=dev) / d ** 0.5).to(bf) for _ in range(L)]
    gates = [(torch.rand(4, H, generator=gen, device=dev) * 4 - 2) for _ in range(L)]
    wk = (torch.randn(D, d, generator=gen, device=dev) / d ** 0.5).to(bf)
    wv = (torch.randn(D, d, generator=gen, device=dev) / d ** 0.5).to(bf)
    h_bank = torch.randn(16, B, d, generator=gen, device=dev).to(bf)
    S = DecodeLayerState(B, H, hd, d, W, device=dev)
    pos = torch.full((B,), c["first_pos"], dtype=torch.int64, device=dev)
    m_prev = torch.zeros(B, d, dtype=bf, device=dev)
    it = torch.zeros((), dtype=torch.int64, device=dev)

    def one_step():
        S.mem_project(pos, m_prev, wk, wv)
        h = torch.index_select(h_bank, 0, torch.remainder(it, 16).view(1))[0].float()
        for l in range(L):
            xn = torch.nn.functional.rms_norm(h, (d,), eps=1e-6).to(bf)
            qkv = torch.matmul(xn, wqkv[l])          # [3, B, D], one batched GEMM
            o = S.step(pos, qkv[0].view(B, H, hd), qkv[1].view(B, H, hd), qkv[2].view(B, H, hd),
                       gates[l], kr[l], vr[l])
            h = h + o.view(B, D).float()
        m_prev.copy_(torch.nn.functional.rms_norm(h, (d,), eps=1e-6).to(bf))
        pos.add_(1)
        it.add_(1)

    # eager warm-up, then capture
    for _ in range(2):
        one_step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        one_step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        one_step()
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    # kernel-level roofline of decode_step from a traced eager step, queued
    # behind a GPU-side delay so that each event pair brackets its kernel alone
    mg.maglev_profile_enable(True)
    torch.cuda._sleep(4_000_000)
    one_step()
    torch.cuda.synchronize()
    mg.maglev_profile_enable(False)
    prof = aggregate_profile(mg.maglev_profile_report())
    del graph
    ring_bytes = 2.0 * B * H * W * hd * 2          # K and V rings read once per layer-step
    roof = None
    if "decode_step" in prof:
        calls, tot, _ = prof["decode_step"]
        avg = tot / calls
        gbs = ring_bytes / (avg * 1e-3) / 1e9
        traffic = stored_traffic("decode_step")
        roof = {"kernel": "decode_step", "bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4), "avg_launch_ms": round(avg, 5),
                "bytes_per_launch": ring_bytes, "traffic": traffic,
                "traffic_source": "stored ncu capture of this kernel's current source" if traffic else None,
                "spec_peak": SPEC_PEAKS["hbm_gbs"], "frac_of_spec": round(gbs / SPEC_PEAKS["hbm_gbs"], 4)}
    return {"tokens_per_s": B * 1000.0 / ms, "ms_per_step": ms, "roofline": roof,
            "kernels": {n: {"calls": v[0], "ms_total": round(v[1], 4)} for n, v in prof.items()},
            "workload": f"decode B={B} L={L} H={H}x{hd} d={d} ring W={W}, {steps} token steps from pos "
                        f"{c['first_pos']} (after {warmup + 3} warm-up steps), CUDA graph"}


def run_full_causal_bench(torch, dev, steps, warmup):
    """One of the prefiller's full-causal layers (SLSL 'L': W = T = 2048, no
    injection), B=8, 10 heads of 128: attention fwd + bwd as a replayed graph.
    Work: 2,098,176 causal pairs per (b, h) x 4 hd flops forward, 2.5x backward."""
    from sliding_window_recurrent_b200.layer import InjectedSWALayer
    B, T, H, hd = STACK["B"], STACK["T"], STACK["H"], STACK["hd"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(1357)
    rn = lambda: torch.randn(B, T, H, hd, generator=gen, device=dev).to(torch.bfloat16)
    q, k, v, dout = rn(), rn(), rn(), rn()
    L = InjectedSWALayer(B, T, H, hd, H * hd, T, dtype="bf16", inject=False, device=dev)

    def step():
        L.forward(q, k, v)
        L.backward(k, v, dout)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = capture_graph(torch, step)
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    ms = e0.elapsed_time(e1) / steps
    f = layer_flops(B, T, H, hd, H * hd, T)
    fl = f["attn_fwd"] + f["attn_bwd"]
    return {"value": round(fl / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "gflop_per_step": round(fl / 1e9, 2),
            "workload": f"prefiller full-causal layer (W = T = {T}, no injection) attention fwd+bwd incl. RoPE "
                        f"and delta/unmix passes, B={B} H={H}x{hd}, bf16, CUDA graph"}


def run_lm_head_bench(torch, dev, steps, warmup, peaks):
    """Softcapped LM head + CE, fwd+bwd: logits GEMM with the CE statistics in
    its epilogue, the loss and dz, then dm = dz U and dU = dz^T m."""
    import sliding_window_recurrent_b200 as mg
    c = LMHEAD
    N, d, V = c["N"], c["d"], c["V"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(97)
    bf = torch.bfloat16
    m = torch.randn(N, d, generator=gen, device=dev).to(bf)
    U = (torch.randn(V, d, generator=gen, device=dev) * (4.0 / d ** 0.5)).to(bf)
    y = torch.randint(0, V, (N,), generator=gen, device=dev)
    loss = torch.zeros((), device=dev)
    lse = torch.empty(N, device=dev)
    dm = torch.empty(N, d, dtype=bf, device=dev)
    dU = torch.empty(V, d, dtype=bf, device=dev)
    ws = torch.empty(mg.maglev_lm_head_workspace_bytes(N, d, V), dtype=torch.uint8, device=dev)
    step = lambda: mg.maglev_lm_head_ce(N, d, V, mg.MAGLEV_BF16, c["softcap"], 0.0, m, U, y, loss, lse, dm, dU, ws)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    mg.maglev_profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    mg.maglev_profile_enable(False)
    prof = aggregate_profile(mg.maglev_profile_report())
    ms = e0.elapsed_time(e1) / steps
    flops = 3 * 2.0 * N * d * V  # logits, dm, dU
    kern = {n: {"calls": v[0], "ms_total": round(v[1], 4)} for n, v in prof.items()}
    roof = None
    if "lm_logits_ce_tc" in prof:
        calls, tot, _ = prof["lm_logits_ce_tc"]
        tf = 2.0 * N * d * V / (tot / calls * 1e-3) / 1e12
        roof = {"kernel": "lm_logits_ce_tc", "bound": "tensor", "achieved": round(tf, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4)}
    del ws
    torch.cuda.empty_cache()
    return {"value": round(flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "gflop_per_step": round(flops / 1e9, 1), "roofline": roof, "kernels": kern,
            "workload": f"softcapped LM head + CE fwd+bwd: N={N} tokens, d={d}, V={V}, softcap 15, bf16"}


# --------------------------------------------------------------------------- oracle arm
def oracle_sample_step(x, c):
    """The oracle's fwd + loss + bwd on a bounded sample of the layer workload:
    batch row 0, head 0, the full T = 2048 sequence, that head's memory channels."""
    import oracle
    hd, T, W, d = c["hd"], c["T"], c["W"], c["d"]
    q, k, v = (x[n][:1, :, :1] for n in ("q", "k", "v"))
    m = x["m_shift"][:1]
    wk, wv = x["w_mk"][:hd], x["w_mv"][:hd]
    Rk, Rv = oracle.mem_project(m, wk, wv)
    f = oracle.inject_swa_forward(q, k, v, Rk, Rv, x["gates"][:, :1], W)
    loss, dm, _ = oracle.consistency_loss(f["out"].reshape(T, hd), x["target"][0, :, :hd], c["lam"])
    g = oracle.inject_swa_backward(q, k, v, Rk, Rv, x["gates"][:, :1], x["dout"][:1, :, :1] + dm.reshape(1, T, 1, hd), W)
    oracle.mem_project_backward(m, wk, wv, g["dR_k"], g["dR_v"])


def oracle_sample_inputs():
    import synth
    x = synth.layer_inputs(dict(synth.WORKLOADS["layer_bf16"]), 1234)
    out = {n: x[n].f64 for n in ("q", "k", "v", "m_shift", "w_mk", "w_mv", "target", "dout")}
    out["gates"] = x["gates"].astype(np.float64)
    return out


def sample_flops(c):
    f = layer_flops(1, c["T"], 1, c["hd"], c["d"], c["W"])
    return f["total"]


def oracle_threads() -> int:
    """Threads the oracle's numpy BLAS runs with (its only parallel part)."""
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return 1


def cpu_baseline(budget_s=12.0):
    c = LAYER
    x = oracle_sample_inputs()
    fl = sample_flops(c)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_sample_step(x, c)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 50:
            break
    return {"value": round(fl * n / el / 1e12, 6), "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"oracle fwd+loss+bwd of batch row 0, head 0 (T=2048, W=512, d=1280): {fl/1e9:.3f} GFLOP x {n} runs in {el:.1f} s"}


def layer_config(world: int) -> dict:
    """`config` of the headline line, the same for both arms."""
    c = LAYER
    return {"workload": "d20 injected-SWA layer fwd+consistency loss+bwd: B=4 T=2048 d=1280 H=10x128 "
                        "W=512 lambda=0.1, bf16 storage, fp32 accumulation",
            "global_batch": c["B"] * world, "seq_len": c["T"], "parallelism": f"replicas x{world} (no collective)",
            "l2": "no flush: each step touches ~0.4 GB > 126 MB L2",
            "gflop_per_step": round(layer_flops(c["B"], c["T"], c["H"], c["hd"], c["d"], c["W"])["total"] / 1e9, 3)}


def reference_arm(args, rank):
    if rank != 0:
        return
    c = LAYER
    x = oracle_sample_inputs()
    fl = sample_flops(c)
    for _ in range(args.warmup):
        oracle_sample_step(x, c)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(x, c)
    el = time.perf_counter() - t0
    val = fl * args.steps / el / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": layer_config(args.gpus),
            "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                             "sample": f"the CPU fp64 oracle's fwd+loss+bwd of batch row 0, head 0 of that "
                                       f"workload (T=2048, W=512, d=1280): {fl/1e9:.3f} GFLOP per step"},
            "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=4096)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--stack-steps", type=int, default=5)
    ap.add_argument("--no-stack", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-lm-head", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        reference_arm(args, rank)
        return

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    from sliding_window_recurrent_b200 import build as _build
    _build.build(quiet=True)
    import sliding_window_recurrent_b200 as mg

    peaks, peaks_src = load_peaks()
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        gpu_uuid = gpu_uuid if gpu_uuid.startswith("GPU-") else "GPU-" + gpu_uuid
    except Exception:
        gpu_uuid = None

    r = run_layer_bench(torch, dist, rank, world, dev, args.steps, args.warmup, peaks, peaks_src, gpu_uuid)
    value = job_rate(r["flops"]["total"], world, r["ms"]) / 1e12

    e2e = None
    if not args.no_e2e:
        ms_e2e, h2d, d2h = run_layer_e2e(torch, dev, args.steps, args.warmup, r["step"])
        ms_e2e = max_over_ranks(dist, ms_e2e, dev)
        e2e = {"value": round(job_rate(r["flops"]["total"], world, ms_e2e) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 4)}

    fwd = run_layer_fwd_bench(torch, dev, args.steps, args.warmup, r["step"])
    stack = None
    if not args.no_stack:
        stack = run_stack_bench(torch, dev, args.stack_steps, args.warmup)
        ms_stack = max_over_ranks(dist, stack["ms_per_step"], dev)
        stack["value"] = round(job_rate(stack_flops(STACK), world, ms_stack) / 1e12, 3)

    dec = None
    if not args.no_decode:
        dec = run_decode_bench(torch, dev, args.decode_steps, args.warmup, peaks)
        dec["tokens_per_s"] = job_rate(DECODE["B"], world, max_over_ranks(dist, dec["ms_per_step"], dev))

    full = None
    if not args.no_stack:
        full = run_full_causal_bench(torch, dev, args.steps, args.warmup)

    lmh = None
    if not args.no_lm_head:
        lmh = run_lm_head_bench(torch, dev, max(3, args.steps // 4), args.warmup, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(r["ms"], 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) inputs of the d20 shapes (stand-in for FineWeb-Edu activations)",
        "config": layer_config(world),
        "frac_of_bf16_peak": round(value / world / peaks["bf16_tflops"], 5),
        "frac_of_spec_bf16_peak": round(value / world / SPEC_PEAKS["bf16_tflops"], 5),
        "roofline": r["roofline"],
        "kernels": r["kernels"],
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
        "forward": fwd,
        "stack": stack,
        "prefiller_full_causal_layer": full,
        "lm_head": lmh,
        "decode": None if dec is None else {
            "value": round(dec["tokens_per_s"], 1), "unit": "tokens/s", "ms_per_step": round(dec["ms_per_step"], 4),
            "workload": dec["workload"], "roofline": dec["roofline"], "kernels": dec["kernels"]},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
