#!/usr/bin/env python
"""Benchmark: HyQuant hybrid INT4/FP16 KV-cache decode attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: Llama-3.1-8B-shaped decode attention at 32K context (batch 1 per
GPU, 32 query / 8 KV heads, head_dim 128, window 128, 3% vertical-line
tokens).  One step = one decode step of one attention layer through the
library's C ABI: hyq_append (the token leaving the window is packed to INT4,
the new K/V enters the window, the query enters the detector ring) and
hyq_decode (fused dequant + attention, split-KV + combine); every 64 tokens
of a layer the step also re-selects its vertical lines (hyq_select_vl over
the cache + hyq_vl_apply).  Eight independent layer caches are cycled so the
working set (~360 MB) exceeds the 126 MB L2 between successive steps.

Metric: effective decode-attention HBM GB/s = algorithmic bytes of the
decode steps (packed codes + scales + FP16 vertical-line/window K/V + Q/O) /
time.  The timed region is one CUDA-graph replay of K steps, bracketed by
a barrier and synchronize; the decode kernel's average launch time comes
from CUDA events captured inside the graph around each run of back-to-back
step launches between two re-selections.

--impl reference times the CPU oracle (fp64, plain C) on a bounded sample of
the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention effective HBM GB/s (% of B200 peak); µs/step at 32K ctx"
L2_DEFEAT_BYTES = 360e6  # rotate layer caches until a pass over them is ~3x the 126 MB L2
RESELECT = 64
N_Q = 64
RESELECT_REPS = 4  # cache-mode re-selections timed on their own (the first untimed)


def algorithmic_bytes(B, Hq, Hkv, T, k, W=128):
    """Bytes one decode must move at length T: packed INT4 K/V + scale/zero
    (160 B per token per unit), FP16 K/V of vertical-line and window tokens
    (512 B), Q in and O out (fp16).  k: vertical-line rows, one count for
    every unit or a list with one count per unit."""
    n_old = max(0, T - W)
    ks = [k] * (B * Hkv) if isinstance(k, int) else list(k)
    return sum((n_old - ku) * 160 + ku * 512 + min(T, W) * 512 for ku in ks) + B * Hq * 128 * 2 * 2


def step_bytes(B, Hq, Hkv, T, k, W=128):
    """Bytes of one fused step that ends at length T: the decode's, plus the
    append's per unit (new K/V rows in, the leaving window row in, its INT4
    codes and scale/zero out, the new rows into the window) and the query
    into the detector ring."""
    append = (2 * 256 + 2 * 256 + 160 + 2 * 256) if T - 1 >= W else (2 * 256 + 2 * 256)
    return algorithmic_bytes(B, Hq, Hkv, T, k, W) + B * Hkv * append + B * Hq * 256


def decode_traffic(cid=2):
    """DRAM bytes per decode launch of workload `cid` from the committed ncu
    capture, or None once the decode kernel's sources differ from the
    captured ones."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json" if cid == 2 else f"decode_traffic_c{cid}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    h = hashlib.sha256()
    for name in ("hyq_decode.cu", "hyq_common.cuh", "hyq_quant.cuh"):
        with open(os.path.join(ROOT, "fp16_kv_cache_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return int(d["bytes_per_launch"]) if h.hexdigest() == d.get("source_sha256") else None


def upload_graph(torch, g):
    """Upload an instantiated CUDA graph to the device (cudaGraphUpload)
    before its timed replay.  A graph that was never uploaded is uploaded by
    its first launch, inside the timed region (about 2.5 us per step over a
    20-step graph, measured); the replay itself still runs every step."""
    import ctypes
    rt = ctypes.CDLL("libcudart.so.12")  # the runtime torch has loaded
    rt.cudaGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    rc = rt.cudaGraphUpload(ctypes.c_void_p(g.raw_cuda_graph_exec()),
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    if rc != 0:
        raise RuntimeError(f"cudaGraphUpload failed ({rc})")
    torch.cuda.synchronize()


def max_over_ranks(x: float, device) -> float:
    """The job's time is the slowest rank's: MAX all-reduce over the process
    group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense fp16/bf16 tensor TFLOP/s (burst): measured, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def prefill_attention_leg(torch, hyq, synth, cfg, layer, Kd, Vd):
    """hyq_prefill_attention over the workload's prompt (the layer's cache
    gives T and the vertical lines), timed with CUDA events after one
    untimed call.  Algorithmic work: 4 * 128 flop per causal (query row,
    key) pair and query head (Q K^T and P V), against the measured dense
    fp16/bf16 tensor peak."""
    B, Hq, T = cfg.B, cfg.Hq, cfg.T
    cap = layer.cap
    g = torch.Generator(device="cuda").manual_seed(cfg.seed & 0xFFFF)
    q = torch.randn(B, Hq, cap, 128, device="cuda", generator=g, dtype=torch.float32).to(torch.float16)
    o = torch.empty(B, Hq, cap, 128, dtype=torch.float32, device="cuda")
    ws = hyq.workspace(hyq.hyq_prefill_attention_workspace(layer))
    hyq.hyq_prefill_attention(layer, q, Kd, Vd, o, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    hyq.hyq_prefill_attention(layer, q, Kd, Vd, o, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    flops = 4 * 128 * B * Hq * T * (T + 1) / 2
    tc, tc_kind = measured_tensor_peak()
    rate = flops / (ms * 1e-3) / 1e12
    del q, o, ws
    torch.cuda.empty_cache()
    return {"us": round(1000 * ms, 1), "achieved": round(rate, 2), "unit": "TFLOP/s", "per_launch": int(flops),
            "peak": tc, "frac": round(rate / tc, 4), "peak_source": tc_kind,
            "how": "prepass (quantize + dequantize Q/K/V, transpose V) and the tcgen05 attention kernel, one call"}


def prefill_kernels(cfg, t_ms):
    """Rooflines of the prompt-side calls timed while the layer caches are
    built: hyq_prefill (HBM: per unit T rows of K and V in, 160 B of codes
    and scale/zero out per packed row, the window rows out), hyq_select_vl in
    prefill mode (tensor: 2 passes of 2*128 flop per causal (query row, key)
    pair) and hyq_vl_apply in prefill mode (HBM: 1028 B per selected row)."""
    U, G, T, W, k = cfg.B * cfg.Hkv, cfg.Hq // cfg.Hkv, cfg.T, 128, cfg.k
    hbm, hbm_kind = measured_peaks()
    tc, tc_kind = measured_tensor_peak()
    n_old, nwin = max(0, T - W), min(T, W)
    b_prefill = U * (T * 512 + n_old * 160 + nwin * 512)
    pairs = G * sum(max(0, T - 63 + i) for i in range(64))  # causal (row, key) pairs per unit
    f_select = 2 * 2 * 128 * pairs * U
    b_apply = U * k * 1028
    out = {}
    for name, ms, amount, unit, peak, kind in (
            ("hyq_prefill", t_ms[0], b_prefill, "GB/s", hbm, hbm_kind),
            ("hyq_select_vl (prefill mode)", t_ms[1], f_select, "TFLOP/s", tc, tc_kind),
            ("hyq_vl_apply (prefill mode)", t_ms[2], b_apply, "GB/s", hbm, hbm_kind)):
        rate = amount / (ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12) if ms > 0 else None
        out[name] = {"us": round(1000 * ms, 2), "achieved": None if rate is None else round(rate, 2),
                     "unit": unit, "per_launch": int(amount), "peak": peak,
                     "frac": None if rate is None else round(rate / peak, 4), "peak_source": kind}
    return out


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=128)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4],
                    help="workload (2: the headline Llama-3.1-8B 32K batch-1 decode; 1, 3 and 4 for profiling)")
    ap.add_argument("--no-prefill-attention", action="store_true",
                    help="skip timing hyq_prefill_attention over the prompt")
    ap.add_argument("--no-batched", action="store_true",
                    help="skip the batched 32K workload (batch 16) that the default run adds under 'batched'")
    return ap.parse_args()


# --------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": int(statistics.median(sm)), "sm_max_mhz": int(rows[0][2]), "samples": len(rows),
                "reasons": reasons}


# --------------------------------------------------------------- setup
def setup_layers(torch, hyq, synth, cfg, cap, n_layers):
    """Build n_layers hybrid caches from the workload's prompt, entirely with
    the library: prefill -> select_vl (prefill mode) -> vl_apply.  Returns the
    caches, the prompt's K/V on the device, and the CUDA-event times (ms) of
    the last layer's three calls (every kernel has run before by then).  That
    layer runs hyq_prefill and hyq_select_vl REP times back to back (both
    rebuild their outputs from the same inputs) and each time is the mean of
    the calls after the first, which queue behind a busy GPU, so the host's
    launch latency stays outside the events; hyq_vl_apply, shorter than that
    latency, is timed once."""
    K, V, _ = synth.kv_full(cfg, cap)
    Kd = torch.from_numpy(K).cuda()
    Vd = torch.from_numpy(V).cuda()
    qs = torch.from_numpy(np.stack([synth.qsel(cfg, b) for b in range(cfg.B)])).cuda()
    REP = 3
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * REP + 2)]
    layers = []
    for li in range(n_layers):
        timed = li == n_layers - 1
        c = hyq.HybridCache(cfg.B, cfg.Hq, cfg.Hkv, cap, cfg.k)
        c.seq_len.fill_(cfg.T)
        pos = torch.zeros(cfg.B, cfg.Hkv, cfg.k, dtype=torch.int32, device="cuda")
        ws = hyq.workspace(hyq.hyq_select_vl_workspace(c, N_Q))
        reps = REP if timed else 1
        for r in range(reps):
            if timed:
                ev[r].record()
            hyq.hyq_prefill(c, Kd, Vd)
        for r in range(reps):
            if timed:
                ev[REP + r].record()
            hyq.hyq_select_vl(c, qs, cfg.k, pos, ws, k_full=Kd)
        if timed:
            ev[2 * REP].record()
        hyq.hyq_vl_apply(c, pos, Kd, Vd)
        if timed:
            ev[2 * REP + 1].record()
        layers.append(c)
    torch.cuda.synchronize()

    def mean_after_first(i0):
        return sum(ev[i].elapsed_time(ev[i + 1]) for i in range(i0 + 1, i0 + REP)) / (REP - 1)

    t_ms = [mean_after_first(0), mean_after_first(REP), ev[2 * REP].elapsed_time(ev[2 * REP + 1])]
    return layers, Kd, Vd, t_ms


def bench_workload(torch, hyq, synth, cfg, K_steps, W_steps, e2e_steps, world, dev, clocks_on, fp16_on,
                   prefill_attn_on=False):
    """Build the workload's layer caches, capture K_steps fused steps in one
    CUDA graph and replay it (timed), time one cache-mode re-selection on
    its own, then the FP16 comparator and the end-to-end loop.  Returns the
    measurements; the caller composes the JSON line."""
    # enough layer caches that consecutive steps never find their data in L2
    n_layers = int(min(8, max(2, math.ceil(L2_DEFEAT_BYTES / algorithmic_bytes(cfg.B, cfg.Hq, cfg.Hkv, cfg.T, cfg.k)))))
    per_layer_tokens = (K_steps + W_steps + e2e_steps) // n_layers + 2 + RESELECT_REPS
    cap = ((cfg.T + per_layer_tokens + 127) // 128) * 128
    layers, Kd, Vd, t_setup = setup_layers(torch, hyq, synth, cfg, cap, n_layers)
    B, Hq, Hkv = cfg.B, cfg.Hq, cfg.Hkv
    pa = prefill_attention_leg(torch, hyq, synth, cfg, layers[-1], Kd, Vd) if prefill_attn_on else None

    # per-step inputs (device) and detector rings / workspaces
    q_in = torch.from_numpy(np.stack([synth.q(cfg, 10 + s) for s in range(64)])).to(dev)
    kv = [synth.step_kv(cfg, s) for s in range(64)]
    k_in = torch.from_numpy(np.stack([a for a, _ in kv])).to(dev)
    v_in = torch.from_numpy(np.stack([b for _, b in kv])).to(dev)
    # the detector's ring holds the last 64 queries of each layer: at the end
    # of the prompt these are the prompt's own last 64 (slot = position % 64)
    qs = np.stack([synth.qsel(cfg, b) for b in range(B)])
    ring0 = np.zeros_like(qs)
    for i in range(N_Q):
        ring0[:, :, (cfg.T - N_Q + i) % N_Q] = qs[:, :, i]
    rings = [torch.from_numpy(ring0).to(dev) for _ in layers]
    out = torch.empty(B, Hq, 128, dtype=torch.float16, device=dev)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    n_ctas = hyq.hyq_decode_default_ctas()
    dws = [hyq.workspace(hyq.hyq_decode_step_workspace(c, n_ctas)) for c in layers]
    sws = hyq.workspace(hyq.hyq_select_vl_workspace(layers[0], N_Q))
    sel_pos = torch.zeros(B, Hkv, cfg.k, dtype=torch.int32, device=dev)
    nunp = torch.zeros(1, dtype=torch.int32, device=dev)
    tokens = [cfg.T] * n_layers        # host mirror of each layer's length
    # Every layer re-selects after every 64 of its tokens.  The layers'
    # phases are staggered evenly (as if each had started decoding at a
    # different time), so that over a long run the re-selections are spread
    # through it at the steady-state rate instead of arriving together.
    appended = [(li * RESELECT) // n_layers for li in range(n_layers)]

    resel_at = {}  # layer -> step after which its first re-selection ran

    def step(s, before=None, after=None):
        """Enqueue step s; returns (launches, layer, T after the step's append,
        whether a re-selection followed).  before() runs before the decode
        launch, after(reselect) after it."""
        li = s % n_layers
        c = layers[li]
        i = s % 64
        if before is not None:
            before()
        hyq.hyq_decode_step(c, q_in[i], k_in[i], v_in[i], out, dws[li], q_ring=rings[li], lse=lse,
                            n_ctas=n_ctas)
        tokens[li] += 1
        appended[li] += 1
        launches = 1
        resel = appended[li] % RESELECT == 0
        if after is not None:
            after(resel)
        if resel:
            # the 64 queries of the ring are scored; the next decode of the
            # layer sees the new vertical-line set
            hyq.hyq_select_vl(c, rings[li], cfg.k, sel_pos, sws, q_is_ring=True)
            hyq.hyq_vl_apply(c, sel_pos, n_unpromoted=nunp)
            resel_at.setdefault(li, s)
            launches += 6  # select (cache mode): 5 kernels; vl_apply (cache mode): 1
        return launches, li, tokens[li], resel

    # warm-up (eager, untimed) -- also sets kernel attributes before capture
    for s in range(W_steps):
        step(s)
    torch.cuda.synchronize()

    # capture K steps; each run of back-to-back decode launches between two
    # re-selections is bracketed by one pair of events, so the launches inside
    # a run keep their programmatic overlap with the launch before them
    runs = []  # [start event, end event, [indices into `seen`]]

    def run_open():
        if not runs or runs[-1][1] is not None:
            e = torch.cuda.Event(enable_timing=True, external=True)
            e.record()
            runs.append([e, None, []])

    def run_close():
        e = torch.cuda.Event(enable_timing=True, external=True)
        e.record()
        runs[-1][1] = e

    g = torch.cuda.CUDAGraph()
    total_launches = 0
    n_resel_timed = 0
    seen = []  # (step, layer, T)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for j in range(K_steps):
                last = j == K_steps - 1

                def after(resel, j=j, last=last):
                    runs[-1][2].append(j)
                    if resel or last:
                        run_close()

                nl, li, T, resel = step(W_steps + j, run_open, after)
                total_launches += nl
                n_resel_timed += int(resel)
                seen.append((W_steps + j, li, T))
    torch.cuda.synchronize()
    upload_graph(torch, g)

    clocks = ClockSampler(dev.index or 0) if clocks_on else None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    g.replay()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), dev)
    # algorithmic bytes of every timed decode, with the VL count it saw
    # (a cache-mode re-selection keeps only rows still held in FP16)
    k_after = [c.vl_count.flatten().tolist() for c in layers]  # per unit, after the re-selection
    total_bytes = 0
    nbytes = []
    for j, (s_, li, T) in enumerate(seen):
        kk = cfg.k if (li not in resel_at or s_ <= resel_at[li]) else k_after[li]
        nb = step_bytes(B, Hq, Hkv, T, kk)
        total_bytes += nb
        nbytes.append(nb)
    run_ms = sum(r[0].elapsed_time(r[1]) for r in runs)
    run_n = sum(len(r[2]) for r in runs)
    dec_avg_ms = run_ms / run_n
    ev_bytes = [nbytes[j] for r in runs for j in r[2]]
    del g

    # one cache-mode re-selection (hyq_select_vl over the cache from the ring
    # + hyq_vl_apply), timed on its own with CUDA events, a few times
    resel_ms = []
    for r in range(RESELECT_REPS):
        c = layers[r % n_layers]
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        hyq.hyq_select_vl(c, rings[r % n_layers], cfg.k, sel_pos, sws, q_is_ring=True)
        hyq.hyq_vl_apply(c, sel_pos, n_unpromoted=nunp)
        e1.record()
        torch.cuda.synchronize()
        resel_ms.append(e0.elapsed_time(e1))
    resel_us = 1000 * float(np.median(resel_ms[1:] if len(resel_ms) > 1 else resel_ms))
    status = max(c.status() for c in layers)

    # hyq_decode alone (no fused append) over the same rotating caches,
    # back-to-back launches in one CUDA graph between one pair of events
    dec_only = decode_only_leg(torch, hyq, cfg, layers, q_in, out, lse, tokens, dev)

    # FP16 comparator (same kernel design over an all-FP16 cache), 3 copies > L2
    fp16 = fp16_comparator(torch, hyq, cfg, Kd, Vd, q_in, dev) if fp16_on else None

    # end to end through the public API with host buffers (eager loop)
    e2e = run_e2e(torch, hyq, cfg, layers, rings, dws, sws, sel_pos, nunp, n_ctas, tokens, appended,
                  e2e_steps, world, dev) if e2e_steps else None

    peak, peak_kind = measured_peaks()
    bytes_per_decode = float(np.mean(ev_bytes))
    achieved = bytes_per_decode / (dec_avg_ms * 1e-3) / 1e9
    us_step = 1000 * elapsed_ms / K_steps
    return {
        "cfg": cfg, "n_layers": n_layers, "n_ctas": n_ctas, "elapsed_ms": elapsed_ms,
        "total_bytes": total_bytes, "value": world * total_bytes / (elapsed_ms * 1e-3) / 1e9,
        "us_per_step": us_step, "dec_avg_ms": dec_avg_ms, "runs": len(runs), "run_n": run_n,
        "bytes_per_decode": bytes_per_decode, "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
        "n_resel_timed": n_resel_timed, "resel_us": resel_us, "k_after": k_after, "status": status,
        "fp16": fp16, "e2e": e2e, "clk": clk, "launches": total_launches, "t_setup": t_setup, "prefill_attn": pa,
        # the detector at the pages' cadence: one re-selection per 64 decode
        # steps of a layer, against 64 steps of this workload's decode
        "detector_share": resel_us / (64 * 1000 * dec_avg_ms + resel_us),
        "decode_only": dec_only,
    }


def workload_summary(r, world):
    """The per-workload keys of the JSON line."""
    cfg = r["cfg"]
    return {
        "workload": f"{cfg.name}: decode attention, B={cfg.B}/GPU, Hq={cfg.Hq}, Hkv={cfg.Hkv}, d=128, "
                    f"T={cfg.T}, window 128, VL {cfg.k}, INT4 g32",
        "step": f"hyq_decode_step (append + decode in one launch) on one of {r['n_layers']} layer caches; "
                f"every 64 tokens of a layer hyq_select_vl(cache) + hyq_vl_apply; "
                f"{r['n_resel_timed']} re-selections ran inside the timed region",
        "l2": f"inputs larger than L2: {r['n_layers']} rotating layer caches "
              f"(~{r['n_layers'] * r['bytes_per_decode'] / 1e6:.0f} MB) per GPU",
        "us_per_step": round(r["us_per_step"], 3),
        "decode_us_avg": round(1000 * r["dec_avg_ms"], 3),
        "decode_timed": f"CUDA events around {r['runs']} runs of back-to-back step launches "
                        f"({r['run_n']} launches, re-selections outside the runs)",
        "decode_bytes_per_step": int(r["bytes_per_decode"]),
        "pct_of_peak_step": round(100 * r["value"] / world / r["peak"], 1),
        "reselect": {"us": round(r["resel_us"], 1),
                     "how": "one cache-mode hyq_select_vl (from the 64-query ring) + hyq_vl_apply, CUDA events, "
                            f"median of {RESELECT_REPS - 1} after one untimed",
                     "share_at_64_token_cadence": round(r["detector_share"], 4)},
        "n_ctas": r["n_ctas"],
        "decode_only": r["decode_only"],
        "fp16_comparator": r["fp16"],
        "dev_status": r["status"],
        "vl_rows_after_reselect": [min(min(k) for k in r["k_after"]), max(max(k) for k in r["k_after"])],
        "parallelism": f"replicas x{world} (independent sequences, no collective)",
    }


def roofline_of(r):
    return {"bound": "hbm", "achieved": round(r["achieved"], 1), "peak": r["peak"], "unit": "GB/s",
            "frac": round(r["achieved"] / r["peak"], 4), "traffic": decode_traffic(r["cfg"].cid),
            "kernel": "hyq::decode_kernel<G,2> (hyq_decode_step)", "peak_source": f"{r['peak_kind']} hbm_gbs",
            "bytes_per_launch": int(r["bytes_per_decode"])}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import synth
    from fp16_kv_cache_b200 import build, hyq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    build.build()
    dev = torch.device("cuda", local)
    cfg = synth.config(args.config)
    r = bench_workload(torch, hyq, synth, cfg, args.steps, args.warmup, args.e2e_steps, world, dev,
                       not args.no_clocks, args.config == 2, prefill_attn_on=not args.no_prefill_attention)
    batched = None
    if args.config == 2 and not args.no_batched:
        # the batched long-context workload (batch 16, 32K each): its own
        # caches, graph and events, in the same run
        rb = bench_workload(torch, hyq, synth, synth.config(3), max(8, min(args.steps, 48)),
                            max(3, min(args.warmup, 8)), 0, world, dev, not args.no_clocks, False)
        batched = workload_summary(rb, world)
        batched.update({"value": round(rb["value"], 1), "unit": "GB/s", "steps": max(8, min(args.steps, 48)),
                        "roofline": roofline_of(rb), "gpu_launches": rb["launches"]})
        if rb["clk"]:
            batched["clocks"] = rb["clk"]
        torch.cuda.empty_cache()
    K_steps, W_steps = args.steps, args.warmup
    line = {
        "metric": METRIC, "value": round(r["value"], 1), "unit": "GB/s", "n_gpus": world,
        "steps": K_steps, "warmup": W_steps, "ms_per_step": round(r["elapsed_ms"] / K_steps, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
        "data": "synthetic (seeded N(0,1) fp16 Q/K/V, 4 K outlier channels x8, planted vertical lines)",
        "config": workload_summary(r, world),
        "roofline": roofline_of(r),
        "e2e": r["e2e"],
        "gpu_launches": r["launches"],
        "other_kernels": prefill_kernels(cfg, r["t_setup"]),
    }
    if r["prefill_attn"] is not None:
        line["other_kernels"]["hyq_prefill_attention"] = r["prefill_attn"]
    if batched is not None:
        line["batched"] = batched
    if r["clk"]:
        line["clocks"] = r["clk"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def decode_only_leg(torch, hyq, cfg, layers, q_in, out, lse, tokens, dev, reps=None):
    """hyq_decode (the decode without the fused append) timed like the step:
    back-to-back launches over the rotating layer caches in one CUDA graph,
    one pair of CUDA events around them.  The caches are only read."""
    n = len(layers)
    reps = reps or max(4 * n, 32 if cfg.B == 1 else 16)
    n_ctas = hyq.hyq_decode_default_ctas()
    ws = [hyq.workspace(hyq.hyq_decode_workspace(c, n_ctas)) for c in layers]
    for i in range(n):
        hyq.hyq_decode(layers[i], q_in[i % 64], out, ws[i], lse=lse, n_ctas=n_ctas)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            e0.record()
            for i in range(reps):
                hyq.hyq_decode(layers[i % n], q_in[i % 64], out, ws[i % n], lse=lse, n_ctas=n_ctas)
            e1.record()
    torch.cuda.synchronize()
    upload_graph(torch, g)
    g.replay()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    del g
    ks = [c.vl_count.flatten().tolist() for c in layers]
    nbytes = float(np.mean([algorithmic_bytes(cfg.B, cfg.Hq, cfg.Hkv, tokens[i % n], ks[i % n]) for i in range(reps)]))
    peak, kind = measured_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"us": round(1000 * ms, 3), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "bytes": int(nbytes),
            "launches": reps, "peak_source": f"{kind} hbm_gbs",
            "how": "hyq_decode alone (no fused append), back-to-back launches over the rotating caches, CUDA events"}


def fp16_comparator(torch, hyq, cfg, Kd, Vd, q_in, dev, copies=3, reps=60):
    Ks = [Kd] + [Kd.clone() for _ in range(copies - 1)]
    Vs = [Vd] + [Vd.clone() for _ in range(copies - 1)]
    seq = torch.full((cfg.B,), cfg.T, dtype=torch.int32, device=dev)
    o = torch.empty(cfg.B, cfg.Hq, 128, dtype=torch.float16, device=dev)
    ws = hyq.workspace(hyq.hyq_decode_fp16_workspace(cfg.B, cfg.Hq, cfg.Hkv))
    for i in range(6):
        hyq.hyq_decode_fp16(q_in[i], Ks[i % copies], Vs[i % copies], seq, o, ws)
    torch.cuda.synchronize()
    # timed like the hybrid step: one pair of events around back-to-back launches
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            e0.record()
            for i in range(reps):
                hyq.hyq_decode_fp16(q_in[i % 64], Ks[i % copies], Vs[i % copies], seq, o, ws)
            e1.record()
    torch.cuda.synchronize()
    upload_graph(torch, g)
    g.replay()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = cfg.B * cfg.Hkv * cfg.T * 512 + cfg.B * cfg.Hq * 128 * 4
    del g
    return {"us": round(1000 * ms, 3), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "bytes": nbytes}


def run_e2e(torch, hyq, cfg, layers, rings, dws, sws, sel_pos, nunp, n_ctas, tokens, appended, n, world, dev):
    """Same metric through the public API with host buffers: each step copies
    its q / k_new / v_new from pinned host memory and reads o back."""
    B, Hq, Hkv = cfg.B, cfg.Hq, cfg.Hkv
    rng = np.random.default_rng(0)
    # a step's inputs are staged together in pinned memory: q, then k_new,
    # then v_new (one host->device copy per step)
    nq, nk = B * Hq * 128, B * Hkv * 128
    hin = torch.from_numpy(rng.standard_normal((n, nq + 2 * nk)).astype(np.float16)).pin_memory()
    ho = torch.empty(n, B, Hq, 128, dtype=torch.float16).pin_memory()
    din = torch.empty(nq + 2 * nk, dtype=torch.float16, device=dev)
    dq = din[:nq].view(B, Hq, 128)
    dk = din[nq:nq + nk].view(B, Hkv, 128)
    dv = din[nq + nk:].view(B, Hkv, 128)
    do = torch.empty(B, Hq, 128, dtype=torch.float16, device=dev)
    k_before = [c.vl_count.flatten().tolist() for c in layers]  # vertical-line rows per unit
    seen = []  # (layer, T after the step, whether the layer has re-selected during this loop)
    resel = set()
    # the binding's prepared call per layer (arguments marshalled once) and
    # the per-step host views, made before the timed loop
    calls = [hyq.DecodeStepCall(c, dq, dk, dv, do, dws[li], q_ring=rings[li], n_ctas=n_ctas)
             for li, c in enumerate(layers)]
    h_in = [hin[s] for s in range(n)]
    h_out = [ho[s] for s in range(n)]
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for s in range(n):
        li = s % len(layers)
        c = layers[li]
        hyq.hyq_copy(din, h_in[s])
        calls[li]()
        hyq.hyq_copy(h_out[s], do)
        tokens[li] += 1
        appended[li] += 1
        seen.append((li, tokens[li], li in resel))
        if appended[li] % RESELECT == 0:
            hyq.hyq_select_vl(c, rings[li], cfg.k, sel_pos, sws, q_is_ring=True)
            hyq.hyq_vl_apply(c, sel_pos, n_unpromoted=nunp)
            resel.add(li)
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    k_after = [c.vl_count.flatten().tolist() for c in layers]
    total = sum(step_bytes(B, Hq, Hkv, T, k_after[li] if late else k_before[li]) for li, T, late in seen)
    return {"value": round(world * total / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
            "h2d_bytes_per_step": (B * Hq + 2 * B * Hkv) * 256, "d2h_bytes_per_step": B * Hq * 256,
            "us_per_step": round(1000 * ms / n, 3), "steps": n,
            "how": "eager loop of C-ABI calls via the ctypes binding (hyq.DecodeStepCall: arguments marshalled "
                   "once per layer); each step copies its q, k_new, v_new (staged together in pinned memory) to "
                   "the device and o back to pinned memory with hyq_copy (the library's copy kernel)"}


# --------------------------------------------------------------- CPU oracle
def cpu_baseline(seconds, cid=2):
    """The fp64 oracle as it stands, on the host cores, on a bounded sample:
    whole decode steps of the same workload (all 8 units, 32K positions),
    repeated until `seconds` of wall time; GB/s on the same algorithmic
    bytes."""
    import oracle
    import synth
    cfg = synth.config(cid)
    K, V, planted = synth.kv_full(cfg)
    c = oracle.OracleCache(cfg.B, cfg.Hq, cfg.Hkv, cfg.T, cfg.k)
    c.load_prompt(K, V, [cfg.T] * cfg.B)
    c.apply_vl(planted, K, V)
    nbytes = algorithmic_bytes(cfg.B, cfg.Hq, cfg.Hkv, cfg.T, cfg.k)
    steps = 0
    t0 = time.perf_counter()
    while True:
        oracle.decode(c, synth.q(cfg, steps))
        steps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": round(steps * nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{steps} full decode steps of llama3.1-8b-32k-b1 (8 units x 32768 positions), "
                      f"{dt:.1f} s wall, OpenMP over units",
            "us_per_step": round(1e6 * dt / steps, 1)}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import synth
    cfg = synth.config(2)
    K, V, planted = synth.kv_full(cfg)
    c = oracle.OracleCache(cfg.B, cfg.Hq, cfg.Hkv, cfg.T, cfg.k)
    c.load_prompt(K, V, [cfg.T] * cfg.B)
    c.apply_vl(planted, K, V)
    # bounded sample per step: 2 of the 8 units (1/4 of a decode step)
    units = [0, 5]
    frac = len(units) / cfg.units
    nbytes = algorithmic_bytes(cfg.B, cfg.Hq, cfg.Hkv, cfg.T, cfg.k) * frac
    for s in range(args.warmup):
        oracle.decode(c, synth.q(cfg, s), units=units)
    t0 = time.perf_counter()
    for s in range(args.steps):
        oracle.decode(c, synth.q(cfg, 100 + s), units=units)
    dt = time.perf_counter() - t0
    value = args.steps * nbytes / dt / 1e9
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * dt / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": "llama3.1-8b-32k-b1 (sample: 2 of 8 units per step)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": "each step decodes units 0 and 5 of the 32K workload (1/4 of a step)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse_args()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
