#!/usr/bin/env python
"""Benchmark: hybrid linear temporal attention forward on B200, 480P workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one call of hlta_hybrid_fwd over one 480P clip (B=1, 24 heads split 8 SWA / 8 DSWA
/ 8 GDN, d=128, T=21 frames of N=1560 tokens, L=32760), i.e. every branch of the operator on
one batch of seeded synthetic inputs already resident in HBM. `value` is tokens/s (B*L per
step, summed over ranks). The q/k/v inputs (603 MB) are larger than the 126 MB L2, so no L2
flush is done between steps.

Under torchrun with N > 1 ranks every rank runs an independent replica on its own GPU with
its own inputs (the operator has no exchange step between GPUs); the timing is taken on the
device, bracketed by barriers, and reduced as the max over ranks.

`--impl reference` times the CPU oracle (oracle/, fp64 plain definitions) on the host cores,
on bounded samples of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "hybrid temporal attention fwd tokens/s @480P; % of bf16 tensor / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="480p")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the training-pass measurement (detail.backward)")
    ap.add_argument("--no-stream", action="store_true",
                    help="skip the streaming-step measurement (detail.stream)")
    return ap.parse_args()


# ------------------------------------------------------------------------------------------
# work accounting (algorithmic: valid query-key pairs at 4*d FLOP, GDN q/k/v/o + gate bytes)
# ------------------------------------------------------------------------------------------
def window_pairs(T: int, N: int, w: int, r: int) -> int:
    frames = 0
    for f in range(T):
        frames += sum(1 for i in range(w) if f - r * i >= 0)
    return frames * N * N


def work(wl):
    ps = window_pairs(wl.T, wl.N, wl.w_swa, 1) * wl.B * wl.Hs
    pd = window_pairs(wl.T, wl.N, wl.w_dswa, wl.r) * wl.B * wl.Hd
    gdn_bytes = wl.B * wl.Hg * wl.L * (4 * wl.d * 2 + 2 * 4)
    return {"swa_flop": 4 * wl.d * ps, "dswa_flop": 4 * wl.d * pd, "gdn_bytes": gdn_bytes}


class Replicas:
    """The N > 1 plumbing: one independent replica per rank (no exchange on the data path);
    barriers bracket the timed region and the device-timed duration is reduced as the max
    over ranks. Works with any torch.distributed backend (NCCL on GPUs, gloo in CPU tests)."""

    def __init__(self, world: int, device):
        self.world, self.device = world, device

    def barrier(self):
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()

    def allmax(self, v: float) -> float:
        if self.world == 1:
            return v
        import torch
        import torch.distributed as dist
        t = torch.tensor([v], device=self.device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def job_value(self, units_per_rank: int, ms_max: float) -> float:
        """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
        return units_per_rank * self.world / (ms_max / 1e3)


def stream_step_flop(wl, f: int) -> int:
    """Algorithmic softmax FLOP of one streaming step at frame f (4*d per valid pair)."""
    taps_s = sum(1 for i in range(wl.w_swa) if f - i >= 0)
    taps_d = sum(1 for i in range(wl.w_dswa) if f - wl.r * i >= 0)
    return 4 * wl.d * wl.B * wl.N * wl.N * (taps_s * wl.Hs + taps_d * wl.Hd)


def stream_step_bytes(wl) -> dict:
    """Algorithmic HBM bytes of one steady-state streaming step (every tap frame cached).

    Per rollout: the new frame's q, k, v read and o written (all heads, bf16), the gates
    (fp32 a, b of the GDN heads), the fp32 GDN state read and written, the new K/V appended
    to the rings (written once; their read is the k, v read above) and the cached K/V of the
    window's earlier frames read (w_swa - 1 SWA frames, w_dswa - 1 DSWA taps). The GDN part is
    its heads' q, k, v, o, gates and state."""
    el = 2
    fr = wl.N * wl.d * el                       # one head's frame of one tensor
    qkvo = 4 * wl.H * fr
    gates = 2 * 4 * wl.Hg * wl.N
    state = 2 * 4 * wl.Hg * wl.d * wl.d
    ring_w = 2 * (wl.Hs + wl.Hd) * fr
    ring_r = 2 * fr * (wl.Hs * (wl.w_swa - 1) + wl.Hd * (wl.w_dswa - 1))
    gdn = 4 * wl.Hg * fr + gates + state
    return {"total": wl.B * (qkvo + gates + state + ring_w + ring_r), "gdn": wl.B * gdn}


def measure_stream(h, torch, dev, warm: int = 24, steps: int = 40) -> dict:
    """Steady-state step time of the streaming cache on the 8-rollout 480P stream workload.

    The first `warm` steps fill the rings (every tap frame exists from frame r*(w-1) on);
    `steps` further steps are timed with CUDA events, with the library's per-branch profile
    events inside each step. Inputs: 4 seeded frames, cycled."""
    import hlta_inputs as hi
    sw = hi.WORKLOADS["stream_480p"]
    x = hi.make_inputs(sw, seed=7, frames=4)
    fr = []
    for i in range(4):
        sl = slice(i * sw.N, (i + 1) * sw.N)
        fr.append({n: x[n][:, :, sl].contiguous().to(dev) for n in "qkvab"})
    o = torch.empty_like(fr[0]["q"])
    st = h.Stream(sw.B, sw.Hs, sw.Hd, sw.Hg, sw.N, sw.d, sw.w_swa, sw.w_dswa, sw.r, sw.chunk)
    for i in range(warm):
        f = fr[i % 4]
        st.step(f["q"], f["k"], f["v"], f["a"], f["b"], out=o)
    torch.cuda.synchronize()
    prof = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for evs in prof:
        for e in evs:
            e.record()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    n0 = h.hlta_kernel_launches()
    e0.record()
    for i in range(steps):
        f = fr[i % 4]
        h.hlta_set_profile_events(prof[i])
        st.step(f["q"], f["k"], f["v"], f["a"], f["b"], out=o)
    e1.record()
    torch.cuda.synchronize()
    h.hlta_set_profile_events(None)
    launches = (h.hlta_kernel_launches() - n0) / steps
    st.close()
    ms = e0.elapsed_time(e1) / steps
    gdn_ms = statistics.mean(p[3].elapsed_time(p[4]) for p in prof)
    sb = stream_step_bytes(sw)
    flop = stream_step_flop(sw, warm + steps)
    # the same rollout advanced 4 frames per call (hlta_stream_step_frames)
    F = 4
    big = {n: x[n].to(dev) for n in "qkvab"}          # [B, H, 4N, d], [B, Hg, 4N]
    o4 = torch.empty_like(big["q"])
    st4 = h.Stream(sw.B, sw.Hs, sw.Hd, sw.Hg, sw.N, sw.d, sw.w_swa, sw.w_dswa, sw.r, sw.chunk,
                   max_step_frames=F)
    for _ in range(warm // F):
        st4.step_frames(big["q"], big["k"], big["v"], big["a"], big["b"], F, out=o4)
    torch.cuda.synchronize()
    e0.record()
    calls = steps // F
    for _ in range(calls):
        st4.step_frames(big["q"], big["k"], big["v"], big["a"], big["b"], F, out=o4)
    e1.record()
    torch.cuda.synchronize()
    st4.close()
    ms4 = e0.elapsed_time(e1) / (calls * F)
    # the one-frame step captured into CUDA graphs (one per cycled input frame) and replayed:
    # the frame index comes from the cache's device counter, so replays advance the rollout
    stg = h.Stream(sw.B, sw.Hs, sw.Hd, sw.Hg, sw.N, sw.d, sw.w_swa, sw.w_dswa, sw.r, sw.chunk)
    graphs = []
    for f in fr:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, capture_error_mode="thread_local"):
            stg.step(f["q"], f["k"], f["v"], f["a"], f["b"], out=o)
        graphs.append(gr)
    for i in range(warm):
        graphs[i % 4].replay()
    torch.cuda.synchronize()
    e0.record()
    for i in range(steps):
        graphs[i % 4].replay()
    e1.record()
    torch.cuda.synchronize()
    msg = e0.elapsed_time(e1) / steps
    del graphs
    stg.close()
    return {"workload": f"{sw.name}: B={sw.B} new frame N={sw.N} heads {sw.Hs}/{sw.Hd}/{sw.Hg} "
                        f"SWA w={sw.w_swa} DSWA w={sw.w_dswa} r={sw.r}; steady state (frame >= {warm})",
            "ms_per_step": ms, "tokens_per_s": sw.B * sw.N / (ms / 1e3),
            "softmax_tflops": flop / (ms / 1e3) / 1e12, "launches_per_step": launches,
            "hbm_bytes_per_step": sb["total"], "gbs": sb["total"] / (ms / 1e3) / 1e9,
            "gdn_ms": gdn_ms, "gdn_bytes_per_step": sb["gdn"],
            "gdn_gbs": sb["gdn"] / (gdn_ms / 1e3) / 1e9,
            "four_frames_per_call": {"ms_per_frame": ms4, "tokens_per_s": sw.B * sw.N / (ms4 / 1e3),
                                     "note": "hlta_stream_step_frames with 4 frames per rollout "
                                             "per call, same rollout and steady state"},
            "graph_replay": {"ms_per_step": msg, "tokens_per_s": sw.B * sw.N / (msg / 1e3),
                             "note": "the one-frame step captured once per input frame into a "
                                     "CUDA graph and replayed; same rollout and steady state"}}


def measure_raw(h, torch, dev, wl, hi, steps: int) -> dict:
    """The hybrid step with the GDN prologue fused (raw q, k and gate inputs x, y for the GDN
    heads): same workload, timed like the main step (inputs resident, back to back)."""
    raw = hi.make_raw_inputs(wl, seed=11)
    q, k, v, x, y = (raw[n].to(dev) for n in ("q", "k", "v", "x", "y"))
    o = torch.empty_like(q)
    S = torch.empty((wl.B, wl.Hg, wl.d, wl.d), device=dev, dtype=torch.float32)
    ws = torch.empty(h.hlta_hybrid_workspace_bytes(wl.B, wl.Hg, wl.T, wl.N, wl.d, wl.chunk),
                     device=dev, dtype=torch.uint8)

    def step():
        h.hlta_hybrid_fwd_raw(q, k, v, x, y, wl.decay, o, None, S, wl.B, wl.Hs, wl.Hd, wl.Hg,
                              wl.T, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r, wl.chunk, 0.0, ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    # the softmax heads' prologue: rotary embedding of their q and k in place (within-frame
    # position), alone and in front of the raw step
    Hsm = wl.Hs + wl.Hd

    def rope():
        h.rope(q, k, wl.N, heads=(0, Hsm), pos_mode=0)

    for _ in range(3):
        rope()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        rope()
    e1.record()
    torch.cuda.synchronize()
    rope_ms = e0.elapsed_time(e1) / steps
    e0.record()
    for _ in range(steps):
        rope()
        step()
    e1.record()
    torch.cuda.synchronize()
    ms_rope = e0.elapsed_time(e1) / steps
    rope_bytes = 2 * 2 * wl.B * Hsm * wl.L * wl.d * q.element_size()   # q and k, read + write
    return {"ms_per_step": ms, "tokens_per_s": wl.B * wl.L / (ms / 1e3),
            "note": "hlta_hybrid_fwd_raw: the GDN heads' unit-norm q/k and gate activations "
                    "computed inside the chunk preparation",
            "with_rope": {"ms_per_step": ms_rope, "tokens_per_s": wl.B * wl.L / (ms_rope / 1e3),
                          "rope_ms": rope_ms, "rope_bytes": rope_bytes,
                          "rope_gbs": rope_bytes / (rope_ms / 1e3) / 1e9,
                          "note": "hlta_rope on the softmax heads' q and k (in place, position "
                                  "inside the frame), then hlta_hybrid_fwd_raw; rope_gbs against "
                                  "the HBM peak in hbm_peak_gbs"}}


def measure_fp8(h, torch, dev, wl, q, k, v, steps: int) -> dict:
    """The two softmax launches on E4M3 inputs (per-block q/k scales, per-channel v scales):
    attention alone on resident codes, and the three quantisations plus attention from the
    bf16 tensors. Same heads, windows and timing as attn_alone_*."""
    hs, hd = slice(0, wl.Hs), slice(wl.Hs, wl.Hs + wl.Hd)
    br = [(hs, wl.Hs, wl.w_swa, 1), (hd, wl.Hd, wl.w_dswa, wl.r)]
    src = [tuple(x_[:, s_].contiguous() for x_ in (q, k, v)) for s_, _, _, _ in br]
    codes = [h.fp8_quantize_window_inputs(*t, wl.T, wl.N) for t in src]
    outs = [torch.empty(t[0].shape, dtype=torch.bfloat16, device=dev) for t in src]

    def attn():
        for (_, _, w, r), c, o in zip(br, codes, outs):
            h.window_fp8(*c, wl.T, wl.N, w, r, out=o)

    def quant_attn():
        for (_, _, w, r), t, o in zip(br, src, outs):
            h.window_fp8(*h.fp8_quantize_window_inputs(*t, wl.T, wl.N), wl.T, wl.N, w, r, out=o)

    res = {}
    for name, fn in (("attn", attn), ("quantise_and_attn", quant_attn)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        res[name] = e0.elapsed_time(e1) / steps
    return res


def measure_backward(h, torch, dev, wl, q, k, v, a, b, steps: int) -> dict:
    """Training pass of the same workload: the softmax branches' forward with log-sum-exp and
    their backward, and the GDN heads' backward (chunk-start states recomputed inside), each
    timed back to back over `steps` repetitions with a seeded upstream gradient."""
    g0 = wl.Hs + wl.Hd
    gen = torch.Generator(device=dev).manual_seed(99)
    res = {}
    br = [(slice(0, wl.Hs), wl.w_swa, 1), (slice(wl.Hs, g0), wl.w_dswa, wl.r)]
    bf16 = q.dtype == torch.bfloat16          # the softmax training pair is bf16 only
    src = [tuple(x_[:, s_].contiguous() for x_ in (q, k, v)) for s_, _, _ in br if bf16 and s_.stop > s_.start]
    cfg = [(w, r) for s_, w, r in br if bf16 and s_.stop > s_.start]

    def timed(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    if src:
        outs = [h.window_fwd_lse(*t, wl.T, wl.N, w, r) for t, (w, r) in zip(src, cfg)]
        dOs = [torch.randn(t[0].shape, device=dev, generator=gen).to(t[0].dtype) for t in src]
        grads = [tuple(torch.empty_like(t[0]) for _ in range(3)) for t in src]
        wss = [torch.empty(h.hlta_window_bwd_workspace_bytes(wl.B, t[0].shape[1], wl.T, wl.N),
                           dtype=torch.uint8, device=dev) for t in src]

        def fwd():
            for t, (w, r), (o, ls) in zip(src, cfg, outs):
                h.window_fwd_lse(*t, wl.T, wl.N, w, r, out=o, lse=ls)

        def bwd():
            for t, (w, r), (o, ls), dO, gr, ws in zip(src, cfg, outs, dOs, grads, wss):
                h.window_bwd(*t, o, ls, dO, wl.T, wl.N, w, r, grads=gr, workspace=ws)

        res["attn_fwd_lse_ms"] = timed(fwd)
        res["attn_bwd_ms"] = timed(bwd)
        del outs, dOs, grads, wss
    if wl.Hg:
        qg, kg, vg = (x_[:, g0:].contiguous() for x_ in (q, k, v))
        dOg = torch.randn(qg.shape, device=dev, generator=gen).to(qg.dtype)
        wsg = torch.empty(h.hlta_gdn_bwd_workspace_bytes(wl.B, wl.Hg, wl.L), dtype=torch.uint8,
                          device=dev)
        res["gdn_bwd_ms"] = timed(lambda: h.gdn_bwd(qg, kg, vg, a, b, dOg, workspace=wsg))
        res["gdn_bwd_workspace_gb"] = wsg.numel() / 1e9
        del qg, kg, vg, dOg, wsg
    return res


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def traffic_record(kernel_src: str):
    """DRAM bytes per launch from a committed ncu summary, valid only for the same source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        with open(os.path.join(ROOT, "linear_video_world_b200", "csrc", kernel_src), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        r = rec.get(kernel_src)
        if r and r.get("src_sha") == sha:
            return r
    except (OSError, ValueError):
        pass
    return None


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", gpu_index],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ------------------------------------------------------------------------------------------
def oracle_sample(x, wl, rows: int, seed: int):
    """Time the oracle on `rows` query positions of every softmax head plus `rows`
    consecutive tokens of every GDN head; returns (tokens, seconds)."""
    import numpy as np
    import torch

    import oracle
    g = torch.Generator().manual_seed(seed)
    pos = torch.randint(0, wl.L, (rows,), generator=g).numpy()
    q, k, v = (x[n][0] for n in "qkv")          # [H, L, d] float32 numpy, batch 0
    Hs, Hd, Hg = wl.Hs, wl.Hd, wl.Hg
    t0 = time.perf_counter()
    if Hs:
        flat = (np.arange(Hs)[:, None] * wl.L + pos[None, :]).reshape(-1)
        oracle.swa(q[:Hs], k[:Hs], v[:Hs], wl.T, wl.N, wl.w_swa, rows=flat)
    if Hd:
        flat = (np.arange(Hd)[:, None] * wl.L + pos[None, :]).reshape(-1)
        s = slice(Hs, Hs + Hd)
        oracle.dswa(q[s], k[s], v[s], wl.T, wl.N, wl.w_dswa, wl.r, rows=flat)
    if Hg:
        s = slice(Hs + Hd, Hs + Hd + Hg)
        oracle.gdn(q[s, :rows], k[s, :rows], v[s, :rows], x["a"][0, :, :rows], x["b"][0, :, :rows])
    return rows, time.perf_counter() - t0


def host_f32(x):
    """The sampled inputs as float32 numpy arrays (bf16 values are exact in float32), converted
    once so that the timed oracle calls do not pay for the conversion."""
    import numpy as np
    return {n: np.ascontiguousarray(x[n].float().numpy()) for n in "qkvab"}


def calibrated_rows(x, wl, seconds: float, seed: int) -> int:
    """Sample size (tokens) whose oracle time is about `seconds`, at most the whole clip."""
    n0 = min(16, wl.L)
    _, t = oracle_sample(x, wl, n0, seed)
    n1 = min(wl.L, max(n0, int(n0 * min(seconds, 2.0) / max(t, 1e-3))))
    _, t1 = oracle_sample(x, wl, n1, seed + 1)
    return min(wl.L, max(n0, int(n1 * seconds / max(t1, 1e-3))))


def cpu_baseline(x, wl, seconds: float):
    import oracle
    oracle.build()
    x = host_f32(x)
    rows = calibrated_rows(x, wl, seconds, seed=123)
    tokens, sec = oracle_sample(x, wl, rows, seed=124)
    return {"value": tokens * wl.B / sec, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": (f"{rows} random query positions of the 480P clip on all {wl.Hs + wl.Hd} "
                       f"softmax heads (explicit fp64 softmax) plus {rows} consecutive tokens of "
                       f"all {wl.Hg} GDN heads (fp64 token recurrence); {sec:.1f} s")}


def run_reference(args, wl):
    import hlta_inputs as hi
    import oracle
    oracle.build()
    x = host_f32(hi.make_inputs(wl, seed=0))
    budget = min(20.0, 120.0 / max(1, args.steps + args.warmup))   # CPU seconds per step
    rows = calibrated_rows(x, wl, max(0.5, budget), seed=7)
    for i in range(args.warmup):
        oracle_sample(x, wl, rows, seed=1000 + i)
    times = []
    for i in range(args.steps):
        _, sec = oracle_sample(x, wl, rows, seed=2000 + i)
        times.append(sec)
    total = sum(times)
    value = rows * wl.B * args.steps / total
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"per step: {rows} random query positions on every softmax "
                                   f"head plus {rows} GDN tokens on every GDN head"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl):
    return {"workload": f"{wl.name}: B={wl.B} heads {wl.Hs}/{wl.Hd}/{wl.Hg} (SWA/DSWA/GDN) d={wl.d} "
                        f"T={wl.T} N={wl.N} L={wl.L} SWA w={wl.w_swa} DSWA w={wl.w_dswa} r={wl.r} "
                        f"GDN chunk {wl.chunk}",
            "global_batch": wl.B, "seq_len": wl.L, "parallelism": "replicas",
            "l2": "inputs larger than L2 (q,k,v 603 MB vs 126 MB); no flush between steps"}


# ------------------------------------------------------------------------------------------
def main():
    args = parse_args()
    import hlta_inputs as hi
    wl = hi.WORKLOADS[args.workload]
    assert not wl.streaming, "bench workloads: 480p, 480p_long, 720p_long, tiny_fp32"

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        return

    import torch
    import torch.distributed as dist

    import linear_video_world_b200 as h

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    rep = Replicas(world, dev)
    barrier, allmax = rep.barrier, rep.allmax

    x = hi.make_inputs(wl, seed=rank)
    q, k, v, a, b = (x[n].to(dev) for n in "qkvab")
    o = torch.empty_like(q)
    S_out = torch.empty((wl.B, wl.Hg, wl.d, wl.d), device=dev, dtype=torch.float32)
    ws = torch.empty(h.hlta_hybrid_workspace_bytes(wl.B, wl.Hg, wl.T, wl.N, wl.d, wl.chunk,
                                                   h.HLTA_BF16 if wl.dtype == "bf16" else h.HLTA_FP32),
                     device=dev, dtype=torch.uint8)

    def step():
        h.hlta_hybrid_fwd(q, k, v, a, b, o, None, S_out, wl.B, wl.Hs, wl.Hd, wl.Hg, wl.T, wl.N,
                          wl.d, wl.w_swa, wl.w_dswa, wl.r, wl.chunk, 0.0, ws)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert h.hlta_device_status() == 0

    # ---- device-resident timed region -----------------------------------------------------
    K = args.steps
    prof = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    for evs in prof:            # torch creates the CUDA event at its first record
        for e in evs:
            e.record()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    gpu_index = vis.split(",")[local_rank] if vis else str(local_rank)
    barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(gpu_index)
    time.sleep(0.3)
    n_launch0 = h.hlta_kernel_launches()
    ev0.record()
    for i in range(K):
        h.hlta_set_profile_events(prof[i])
        step()
    ev1.record()
    launches = h.hlta_kernel_launches() - n_launch0
    torch.cuda.synchronize()
    h.hlta_set_profile_events(None)
    barrier()
    clocks = clk.stop()
    total_ms = allmax(ev0.elapsed_time(ev1))
    ms = total_ms / K
    # SWA and DSWA heads share one attention launch: from its start (event 0, after the GDN
    # preparation it waits for) to the end of its last CTA (events 1 and 2)
    attn_span_ms = statistics.mean(max(p[0].elapsed_time(p[1]), p[0].elapsed_time(p[2])) for p in prof)
    gdn_ms = statistics.mean(p[3].elapsed_time(p[4]) for p in prof)
    assert h.hlta_device_status() == 0
    tokens = wl.B * wl.L
    value = rep.job_value(tokens, ms)

    # ---- end to end through the C ABI with host buffers -----------------------------------
    # Every step copies its inputs from pinned host memory and its output and final state back.
    # Serial: copy in, compute, copy out on one stream. Pipelined (the serving loop): two sets
    # of device buffers; step i's inputs go in on a copy stream while step i-1 computes and
    # step i-2's results go out on a second copy stream (both link directions at once). The
    # timed region runs from the first input copy to the last result copy.
    pin = {n: x[n].pin_memory() for n in "qkvab"}
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    S_host = torch.empty(S_out.shape, dtype=S_out.dtype, pin_memory=True)
    sets = [({"q": q, "k": k, "v": v, "a": a, "b": b}, o, S_out),
            ({n: torch.empty_like(t) for n, t in (("q", q), ("k", k), ("v", v), ("a", a), ("b", b))},
             torch.empty_like(o), torch.empty_like(S_out))]
    s_comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run_set(i, stream):
        d, o_, S_ = sets[i]
        h.hlta_hybrid_fwd(d["q"], d["k"], d["v"], d["a"], d["b"], o_, None, S_, wl.B, wl.Hs, wl.Hd,
                          wl.Hg, wl.T, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r, wl.chunk, 0.0, ws,
                          stream=stream)

    def e2e_serial():
        d, o_, S_ = sets[0]
        for n in "qkvab":
            d[n].copy_(pin[n], non_blocking=True)
        run_set(0, s_comp)
        o_host.copy_(o_, non_blocking=True)
        S_host.copy_(S_, non_blocking=True)

    def e2e_pipelined(nsteps, e_start, e_end):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_comp = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        s_in.wait_stream(s_comp)
        s_out.wait_stream(s_comp)
        e_start.record(s_in)
        for i in range(nsteps + 2):
            if i < nsteps:                       # inputs of step i (set i % 2, free once step i-2 ran)
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_comp[i - 2])
                    for n in "qkvab":
                        sets[i % 2][0][n].copy_(pin[n], non_blocking=True)
                    ev_in[i].record(s_in)
            j = i - 1
            if 0 <= j < nsteps:                  # step j (its outputs free once step j-2's went out)
                s_comp.wait_event(ev_in[j])
                if j >= 2:
                    s_comp.wait_event(ev_out[j - 2])
                run_set(j % 2, s_comp)
                ev_comp[j].record(s_comp)
            j = i - 2
            if 0 <= j < nsteps:                  # results of step j
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[j])
                    o_host.copy_(sets[j % 2][1], non_blocking=True)
                    S_host.copy_(sets[j % 2][2], non_blocking=True)
                    ev_out[j].record(s_out)
        e_end.record(s_out)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(max(3, args.warmup)):
        e2e_serial()
    torch.cuda.synchronize()
    barrier()
    e0.record()
    for _ in range(K):
        e2e_serial()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_serial_ms = allmax(e0.elapsed_time(e1)) / K
    e2e_pipelined(max(3, args.warmup), torch.cuda.Event(), torch.cuda.Event())
    torch.cuda.synchronize()
    barrier()
    e2e_pipelined(K, e0, e1)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = allmax(e0.elapsed_time(e1)) / K
    assert h.hlta_device_status() == 0
    h2d = sum(pin[n].numel() * pin[n].element_size() for n in "qkvab")
    d2h = o_host.numel() * o_host.element_size() + S_host.numel() * S_host.element_size()

    # ---- the softmax heads alone (no GDN branch sharing the SMs) ---------------------------
    # the SWA and DSWA heads as a hybrid call without GDN heads: the same single attention
    # launch the step makes
    hsd = slice(0, wl.Hs + wl.Hd)
    sub = {n: x_[:, hsd].contiguous() for n, x_ in (("q", q), ("k", k), ("v", v))}
    o_sd = torch.empty_like(sub["q"])

    def attn_only():
        h.hlta_hybrid_fwd(sub["q"], sub["k"], sub["v"], None, None, o_sd, None, None, wl.B, wl.Hs,
                          wl.Hd, 0, wl.T, wl.N, wl.d, wl.w_swa, wl.w_dswa, wl.r, wl.chunk, 0.0, None)

    for _ in range(3):
        attn_only()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(K):
        attn_only()
    a1.record()
    torch.cuda.synchronize()
    attn_alone_ms = a0.elapsed_time(a1) / K
    del sub, o_sd

    # ---- the GDN branch alone (its heads by themselves, all SMs to itself) -----------------
    gdn_alone_ms = None
    if wl.Hg > 0:
        hg = slice(wl.Hs + wl.Hd, wl.Hs + wl.Hd + wl.Hg)
        gq, gk, gv = (x_[:, hg].contiguous() for x_ in (q, k, v))
        go = torch.empty_like(gq)
        gS = torch.empty((wl.B, wl.Hg, wl.d, wl.d), device=dev, dtype=torch.float32)
        gws = torch.empty(h.hlta_gdn_workspace_bytes(wl.B, wl.Hg, wl.L, wl.d, wl.chunk,
                                                     h.HLTA_BF16 if wl.dtype == "bf16" else h.HLTA_FP32),
                          device=dev, dtype=torch.uint8)

        def gdn_only():
            h.hlta_gdn_chunk_fwd(gq, gk, gv, a, b, go, None, gS, wl.B, wl.Hg, wl.L, wl.d, wl.chunk, gws)

        for _ in range(3):
            gdn_only()
        torch.cuda.synchronize()
        a0.record()
        for _ in range(K):
            gdn_only()
        a1.record()
        torch.cuda.synchronize()
        assert h.hlta_device_status() == 0
        gdn_alone_ms = a0.elapsed_time(a1) / K
        del gq, gk, gv, go, gS, gws
    stream_detail = None if args.no_stream else measure_stream(h, torch, dev)
    raw_detail = None if args.no_stream else measure_raw(h, torch, dev, wl, hi, K)
    fp8_ms = (measure_fp8(h, torch, dev, wl, q, k, v, K)
              if not args.no_stream and wl.dtype == "bf16" and wl.Hs + wl.Hd > 0 else None)
    bwd_ms = (measure_backward(h, torch, dev, wl, q, k, v, a, b, max(2, min(K, 5)))
              if not args.no_stream and not args.no_backward and wl.d == 128 else None)

    # ---- roofline of the dominant kernel (windowed attention, both launches) --------------
    wk = work(wl)
    pk, pk_kind = peaks()
    attn_flop = wk["swa_flop"] + wk["dswa_flop"]
    attn_ms = attn_span_ms
    achieved = attn_flop / (attn_ms / 1e3) / 1e12
    # the timed region lasts K steps of ~2 ms (tens of ms): the burst peak applies, not the
    # seconds-long sustained one
    peak = float(pk.get("bf16_tflops"))
    tr = traffic_record("attn_tc2.cu")          # the bf16 window attention kernel
    tr8 = tr                                    # the E4M3 instantiation lives in the same file
    roofline = {"bound": "tensor", "kernel": "attn_tc2_kernel (the SWA and DSWA heads in one persistent "
                                              "launch beside the GDN chain: from its start, after the "
                                              "GDN preparation, to the end of its last CTA)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_kind": f"{pk_kind} bf16 dense, burst (the timed region is {total_ms:.0f} ms)",
                "traffic": tr.get("hybrid_bytes") if tr else None}
    hbm = float(pk.get("hbm_gbs"))
    gdn_gbs = wk["gdn_bytes"] / (gdn_ms / 1e3) / 1e9
    detail = {
        "attn_span_ms": attn_span_ms, "gdn_ms": gdn_ms,
        "gdn_gbs": gdn_gbs, "gdn_hbm_frac": gdn_gbs / hbm,
        "hbm_peak_gbs": hbm, "hbm_peak_kind": pk_kind,
        "attn_alone_ms": attn_alone_ms,
        "attn_alone_tflops": attn_flop / (attn_alone_ms / 1e3) / 1e12,
        "attn_alone_frac": attn_flop / (attn_alone_ms / 1e3) / 1e12 / float(pk.get("bf16_tflops")),
        "gdn_alone_ms": gdn_alone_ms,
        "gdn_alone_gbs": wk["gdn_bytes"] / (gdn_alone_ms / 1e3) / 1e9 if gdn_alone_ms else None,
        "gdn_alone_hbm_frac": wk["gdn_bytes"] / (gdn_alone_ms / 1e3) / 1e9 / hbm if gdn_alone_ms else None,
        "note": "the GDN branch runs on a high-priority stream beside one persistent attention "
                "launch over the SWA and DSWA heads, which starts after the GDN preparation and "
                "leaves the GDN chain its SMs; attn_span_ms runs from that launch's start to the "
                "end of its last CTA (the roofline's duration); attn_alone_* times the attention launch by itself "
                "against the burst bf16 peak; gdn_alone_* times hlta_gdn_chunk_fwd on the GDN "
                "heads by themselves (segment scan over all SMs). The GDN HBM fractions use "
                "the algorithmic q/k/v/o + gate bytes of the GDN heads",
    }
    if stream_detail is not None:
        stream_detail["softmax_frac"] = stream_detail["softmax_tflops"] / peak
        stream_detail["hbm_frac"] = stream_detail["gbs"] / hbm
        stream_detail["gdn_hbm_frac"] = stream_detail["gdn_gbs"] / hbm
        stream_detail["note"] = ("softmax_frac: algorithmic softmax FLOP of the step against the "
                                 "burst bf16 peak; hbm_frac: the step's algorithmic bytes (new "
                                 "q/k/v/o, gates, GDN state read and write, ring appends, cached "
                                 "window K/V) over the step time against the measured HBM copy "
                                 "bandwidth; gdn_hbm_frac: the GDN heads' q/k/v/o, gates and "
                                 "state over the GDN branch's event-timed duration inside the step")
        detail["stream"] = stream_detail
    if raw_detail is not None:
        detail["raw_prologue"] = raw_detail
    if bwd_ms is not None:
        bw = dict(bwd_ms)
        if "attn_bwd_ms" in bw:
            # five products of 2 d FLOP per valid pair (S, dP, dV, dK, dQ; the kernels
            # recompute S and dP once more, not counted)
            bflop = 2.5 * attn_flop
            bw["attn_bwd_tflops"] = bflop / (bw["attn_bwd_ms"] / 1e3) / 1e12
            bw["attn_bwd_frac"] = bw["attn_bwd_tflops"] / float(pk.get("bf16_tflops"))
        bw["note"] = ("training pass: hlta_window_fwd_lse + hlta_window_bwd for the SWA and DSWA "
                      "heads (tcgen05 dK/dV and dQ kernels), hlta_gdn_chunk_bwd for the GDN heads "
                      "(state passes on the tensor cores beside the chunk preparation, chunk "
                      "gradients through the pipelined block GEMM); frac against the burst "
                      "bf16 peak")
        detail["backward"] = bw
    if fp8_ms is not None:
        # E4M3 dense peak = the measured bf16 burst peak x 2 (nominal fp8:bf16 ratio 4.5:2.25)
        fp8_peak = 2.0 * float(pk.get("bf16_tflops"))
        elems = wl.B * (wl.Hs + wl.Hd) * wl.L * wl.d
        detail["fp8"] = {
            "attn_ms": fp8_ms["attn"],
            "attn_tflops": attn_flop / (fp8_ms["attn"] / 1e3) / 1e12,
            "attn_frac_of_fp8_peak": attn_flop / (fp8_ms["attn"] / 1e3) / 1e12 / fp8_peak,
            "fp8_peak_tflops": fp8_peak,
            "attn_bytes": 5 * elems,
            "quantise_and_attn_ms": fp8_ms["quantise_and_attn"],
            "attn_traffic": (tr8["fp8_swa_bytes"] + tr8["fp8_dswa_bytes"]) if tr8 and "fp8_swa_bytes" in tr8 else None,
            "note": "hlta_window_fp8_fwd for the SWA and DSWA heads back to back on resident E4M3 "
                    "codes (q, k, v 1 byte, o bf16: attn_bytes; attn_traffic: DRAM bytes of the two "
                    "launches from the committed ncu summary), then with the three "
                    "quantisations from bf16 in the timed region; peak = measured bf16 burst x 2",
        }

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic (seeded, per-rank seed)",
        "config": config_of(wl), "clocks": clocks,
        "e2e": {"value": rep.job_value(tokens, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "mode": "pipelined: step i's host-to-device copy and step i-2's device-to-host "
                        "copy on two copy streams beside step i-1's compute, two device buffer "
                        "sets; timed from the first input copy to the last result copy",
                "serial": {"value": rep.job_value(tokens, e2e_serial_ms), "ms_per_step": e2e_serial_ms,
                           "note": "copy in, compute, copy out on one stream"}},
        "gpu_launches": launches, "roofline": roofline, "detail": detail,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(x, wl, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
