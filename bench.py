#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200: chunked prefill and recurrent decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One bench step is one chunked prefill of the ``prefill_32k`` workload (B=1,
H=32, T=32768, d=128, chunk 64, bf16 q/k/v, fp32 gates and state), i.e. every
prefill row of the hot path over one batch; ``value`` is prefill tokens/s
over all ranks. The decode row is timed in the same run on the ``decode_256``
workload (256 sequences x 32 heads, 128x128 fp32 states, 1000 consecutive
steps) and reported under ``"decode"`` as state GB/s. Outside the timed region
the same run also times, each with its own roofline fraction: the prefill with
the layer prologue fused in (``"fused_prologue"``), the whole layer between
its projections with seeded synthetic weights (``"layer"``), the backward pass on
prefill_4k's shape (``"backward"``), the packed variable-length prefill into
a state cache (``"varlen"``) and KDA against the general DPLR recurrence on the
same CUDA-core engine design (``"dplr_comparator"``).

Heads and batches are independent, so with N GPUs every rank runs its own copy
of the workload (weak scaling, no collective on the data path); the timed
region is bracketed by a barrier and a device synchronisation and the slowest
rank's time is reported. Rank 0 prints one JSON line.

``--impl reference`` times the fp64 CPU oracle (the checker, never tuned) on a
bounded sample of the same workload on this machine's host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import itertools
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_inputs as I  # noqa: E402

METRIC = "KDA prefill tokens/s (H=32,d=128,T=32K) and decode state GB/s vs HBM peak"
PREFILL = "prefill_32k"
DECODE = "decode_256"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2**20


# ---------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def prefill_bytes(w) -> int:
    """Algorithmic HBM bytes of one prefill: inputs read once, outputs written once.

    Per token-head: q, k, v (3*2*d bytes bf16) + log_alpha (4*dk) + beta (4)
    + out (2*dv) = 1540 B at d = 128; per head: S0 read (if given) + S_T written.
    """
    e = 2 if w.dtype == torch.bfloat16 else 4
    per_tok_head = 2 * w.dk * e + w.dv * e + 4 * w.dk + 4 + w.dv * e
    per_head = 4 * w.dk * w.dv * (2 if w.s0_std > 0 else 1)
    return w.B * w.T * w.H * per_tok_head + w.B * w.H * per_head


def prefill_flops(w) -> int:
    """Algorithmic flops of the chunked form per token-head (causal masks honoured):
    6 d^2 (state products Q~S, WS, K_bar^T U) + 5 C d (intra-chunk products and
    WY/UT applications), counted at d = dk = dv."""
    d, C = w.dk, w.chunk
    return w.B * w.T * w.H * (6 * d * d + 5 * C * d)


def decode_state_bytes(w) -> int:
    """State bytes one decode step moves: every 128x128 fp32 state read and written once."""
    return 2 * w.N * w.H * w.dk * w.dv * 4


def source_hash(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "gated_delta_rule_116_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel_key: str) -> float | None:
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json),
    or None if the kernel's sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel_key)
    if not rec or rec.get("source_hash") != source_hash(*rec.get("sources", [])):
        return None
    return float(rec["dram_bytes_per_launch"])


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], None, set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        loaded = [s for s in sm if s >= 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- our arm

def time_events(fn, n, stream):
    """Device time of n calls of fn on `stream`, one pair of events around each call (ms)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for s, e in evs:
        s.record(stream)
        fn()
        e.record(stream)
    return evs


def run_ours(args, rank, world, device):
    import gated_delta_rule_116_b200 as kda

    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    w = I.WORKLOADS[PREFILL]
    inp = I.prefill_inputs(w, device=device)
    q, k, v, la, beta, S0 = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta", "S0"))
    engine = next(e for e in ("tc_cluster", "generic")
                  if kda.engine_supported(e, w.dk, w.dv, w.chunk, w.dtype))
    out = torch.empty(w.B, w.T, w.H, w.dv, device=device, dtype=w.dtype)
    S_T = torch.empty(w.B, w.H, w.dk, w.dv, device=device, dtype=torch.float32)
    ws_n = kda.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.dtype)
    ws = torch.empty(max(ws_n, 1), device=device, dtype=torch.uint8) if ws_n else None

    def step():
        kda.chunk_fwd(q, k, v, la, beta, S0, w.chunk, out=out, S_T=S_T, engine=engine,
                      workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    barrier(world)
    torch.cuda.synchronize(device)
    with Clocks(device.index if device.index is not None else 0) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        evs = time_events(step, args.steps, stream)
        t1.record(stream)
        torch.cuda.synchronize(device)
    barrier(world)
    ms_kernel = statistics.mean(s.elapsed_time(e) for s, e in evs)
    value, ms_step = weak_scaling_rate(w.tokens, t0.elapsed_time(t1), world, device, args.steps)

    # roofline of the dominant kernel (the prefill kernel; one launch per step)
    hbm, hbm_src = peaks()
    bytes_alg = prefill_bytes(w)
    achieved = bytes_alg / (ms_kernel / 1e3) / 1e9
    traffic = traffic_from_profiles(f"prefill_{engine}")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": traffic,
                "peak_source": hbm_src, "kernel": f"prefill ({engine} engine)",
                "bytes_per_launch": bytes_alg, "kernel_ms": round(ms_kernel, 4),
                "flops_per_launch": prefill_flops(w),
                "tensor_tflops_achieved": round(prefill_flops(w) / (ms_kernel / 1e3) / 1e12, 2)}

    fused = run_fused(kda, w, ws, args, device, stream) if engine == "tc_cluster" else None
    layer = run_layer(kda, w, ws, args, device, stream) if engine == "tc_cluster" else None
    backward = run_backward(kda, args, device, stream) if not args.skip_extra_legs else None
    dplr = run_dplr(kda, args, device, stream) if not args.skip_extra_legs else None
    varlen = run_varlen(kda, args, device, stream) if not args.skip_extra_legs else None
    e2e = run_e2e(kda, w, inp, engine, ws, args, device, stream, world)
    decode = run_decode(kda, args, device, stream, world)
    clocks = clk.summary()
    launches = args.steps  # one prefill kernel per step (the fused leg's launches are outside the timed region)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        cpu = cpu_baseline(args, gpu_inputs=inp, gpu_out=out, gpu_st=S_T)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if engine == "generic" else "bf16",
            "data": "synthetic (seeded; recipe in kda_inputs.py)",
            "config": {"workload": PREFILL, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "chunk": w.chunk, "inputs": "bf16 q/k/v, fp32 gates, fp32 S0/S_T",
                       "engine": engine, "per_rank": "one full workload per GPU",
                       "l2": f"inputs larger than L2 ({bytes_alg / 1e9:.2f} GB moved per step)"},
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches + decode.pop("launches"),
            "clocks": clocks, "decode": decode, "fused_prologue": fused, "layer": layer, "backward": backward,
            "varlen": varlen, "dplr_comparator": dplr, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def run_fused(kda, w, ws, args, device, stream):
    """The same prefill with the layer prologue fused in (kda_chunk_fwd_fused): raw q, k
    and the gate's pre-activation (bf16) instead of unit q, k and fp32 log alpha. Its
    algorithmic bytes per token-head are 3*2*d + 2*d + 4 + 2*d = 1284 at d = 128."""
    lw = I.prefill_layer_inputs(w, device=device)
    out = torch.empty(w.B, w.T, w.H, w.dv, device=device, dtype=w.dtype)
    S_T = torch.empty(w.B, w.H, w.dk, w.dv, device=device, dtype=torch.float32)

    def step():
        kda.chunk_fwd_fused(lw["q"], lw["k"], lw["v"], lw["gate"], lw["beta"], lw["S0"], w.chunk,
                            out=out, S_T=S_T, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    evs = time_events(step, args.steps, stream)
    torch.cuda.synchronize(device)
    ms = statistics.mean(s.elapsed_time(e) for s, e in evs)
    e = 2 if w.dtype == torch.bfloat16 else 4
    bytes_alg = (w.B * w.T * w.H * (2 * w.dk * e + w.dv * e + w.dk * e + 4 + w.dv * e)
                 + w.B * w.H * 4 * w.dk * w.dv * (2 if w.s0_std > 0 else 1))
    hbm, src = peaks()
    gbs = bytes_alg / (ms / 1e3) / 1e9
    return {"entry": "kda_chunk_fwd_fused", "kernel_ms": round(ms, 4),
            "tokens_per_s": round(w.tokens / (ms / 1e3), 1), "bytes_per_launch": bytes_alg,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "peak_source": src}}


def run_layer(kda, w, ws, args, device, stream):
    """The layer between its projections on the bench workload's shape, with seeded
    synthetic weights (kda_inputs.layer_extras): ShortConv + Swish on the projected q,
    k and v (three kda_short_conv_swish launches, W = 4), then kda_layer_fwd (L2 norm,
    gate, recurrence, per-head RMSNorm, sigmoid output gate). Algorithmic bytes per
    token-head at d = 128, bf16: ShortConv 3 x (256 read + 256 written) = 1536; the
    layer kernel 3 x 256 (q, k, v) + 256 (gate) + 4 (beta) + 256 (output gate) + 256
    (out) = 1540, plus S0 read and S_T written per head."""
    lw = I.prefill_layer_inputs(w, device=device)
    ex = I.layer_extras(w, device=device)
    conv = {n: torch.empty_like(ex[f"x_{n}"]) for n in ("q", "k", "v")}
    out = torch.empty(w.B, w.T, w.H, w.dv, device=device, dtype=w.dtype)
    S_T = torch.empty(w.B, w.H, w.dk, w.dv, device=device, dtype=torch.float32)

    def convs():
        for n in ("q", "k", "v"):
            kda.short_conv_swish(ex[f"x_{n}"], ex[f"conv_{n}"], out=conv[n], stream=stream)

    def core():
        kda.layer_fwd(conv["q"], conv["k"], conv["v"], lw["gate"], lw["beta"], ex["out_gate"],
                      ex["norm_weight"], lw["S0"], out=out, S_T=S_T, workspace=ws, stream=stream)

    for _ in range(max(1, args.warmup)):
        convs()
        core()
    torch.cuda.synchronize(device)
    n = max(1, min(args.steps, 5))
    ev_c = time_events(convs, n, stream)
    ev_l = time_events(core, n, stream)
    torch.cuda.synchronize(device)
    ms_c = statistics.mean(a.elapsed_time(b) for a, b in ev_c)
    ms_l = statistics.mean(a.elapsed_time(b) for a, b in ev_l)
    th = w.tokens * w.H
    heads_state = w.B * w.H * 4 * w.dk * w.dv * (2 if w.s0_std > 0 else 1)
    b_conv, b_core = th * 1536, th * 1540 + heads_state
    hbm, src = peaks()

    def roof(b, ms):
        gbs = b / (ms / 1e3) / 1e9
        return {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(gbs / hbm, 4), "peak_source": src}
    return {"entries": "3 x kda_short_conv_swish + kda_layer_fwd", "weights": "seeded synthetic (kda_inputs.layer_extras)",
            "ms": round(ms_c + ms_l, 4), "tokens_per_s": round(w.tokens / ((ms_c + ms_l) / 1e3), 1),
            "short_conv": {"kernel_ms": round(ms_c, 4), "bytes": b_conv, "roofline": roof(b_conv, ms_c)},
            "layer_fwd": {"kernel_ms": round(ms_l, 4), "bytes": b_core, "roofline": roof(b_core, ms_l)}}


def run_dplr(kda, args, device, stream):
    """KDA against the general DPLR recurrence on the same CUDA-core engine design
    (kda_chunk_fwd_engine with KDA_ENGINE_GENERIC vs kda_dplr_chunk_fwd; chunk 32, the
    largest both fit in shared memory at d = 128), per input length: B x T = 16384
    tokens of H = 32 heads, bf16 inputs, T = 2048 and 8192. The ratio DPLR time / KDA
    time re-measures the operator-efficiency comparison of the pages on B200."""
    res = []
    for T in (2048, 8192):
        inp = I.dplr_inputs("prefill_4k", device=device, B=16384 // T, T=T)
        w = inp["w"]
        out = torch.empty(w.B, w.T, w.H, w.dv, device=device, dtype=w.dtype)

        def kda_step():
            kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None, 32,
                          out=out, engine="generic", output_final_state=False, stream=stream)

        def dplr_step():
            kda.dplr_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["log_alpha"], None,
                               32, out=out, output_final_state=False, stream=stream)

        ms = {}
        for name, fn in (("kda", kda_step), ("dplr", dplr_step)):
            fn()
            torch.cuda.synchronize(device)
            evs = time_events(fn, max(1, min(args.steps, 3)), stream)
            torch.cuda.synchronize(device)
            ms[name] = statistics.mean(a.elapsed_time(b) for a, b in evs)
        res.append({"T": T, "B": w.B, "kda_generic_ms": round(ms["kda"], 3), "dplr_ms": round(ms["dplr"], 3),
                    "dplr_over_kda": round(ms["dplr"] / ms["kda"], 3)})
    return {"engines": "fp32 CUDA cores, chunk 32, H=32, d=128, bf16 inputs", "by_length": res}


def run_backward(kda, args, device, stream):
    """The backward pass (kda_chunk_bwd) on prefill_4k's shape: gradients of q, k, v, log
    alpha, beta and S0 from dL/d(out) (bf16, seeded N(0,1)) and dL/d(S_T) (fp32). Its
    algorithmic bytes per token-head are 2824 at d = 128 with bf16 inputs (the forward's
    inputs and dL/d(out) read, six gradients written), plus S0, dL/d(S_T) and dL/d(S0) per
    head; the states it stores for the reverse chain are extra traffic, not counted."""
    w = I.WORKLOADS["prefill_4k"]
    inp = I.prefill_inputs(w, device=device, s0_std=0.05)
    g = torch.Generator(device=device).manual_seed(11)
    gout = torch.randn(w.B, w.T, w.H, w.dv, device=device, generator=g).to(w.dtype)
    gst = torch.randn(w.B, w.H, w.dk, w.dv, device=device, generator=g)
    ws = torch.empty(max(1, kda.bwd_workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.dtype)),
                     device=device, dtype=torch.uint8)

    def step():
        kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], gout, inp["S0"],
                      gst, workspace=ws, stream=stream)

    step()
    torch.cuda.synchronize(device)
    evs = time_events(step, max(1, min(args.steps, 3)), stream)
    torch.cuda.synchronize(device)
    ms = statistics.mean(s.elapsed_time(e) for s, e in evs)
    bytes_alg = w.tokens * w.H * 2824 + w.B * w.H * 3 * w.dk * w.dv * 4
    hbm, src = peaks()
    gbs = bytes_alg / (ms / 1e3) / 1e9
    return {"entry": "kda_chunk_bwd", "workload": "prefill_4k (B=8, H=32, T=4096, d=128, bf16, S0 ~ N(0,0.05))",
            "kernel_ms": round(ms, 3), "tokens_per_s": round(w.tokens / (ms / 1e3), 1),
            "bytes_per_launch": bytes_alg, "kernels": "bwd_states_kernel + bwd_chunk_kernel (16-token chunks, dense products as warp-level 3xTF32 tensor-core tiles, pairwise decays on CUDA cores)",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "peak_source": src}}


def run_varlen(kda, args, device, stream):
    """Packed variable-length prefill (kda_chunk_fwd_varlen_engine) into a state cache through a
    slot map: 32 sequences of 256..4096 tokens (kda_inputs.packed_lengths), H = 32,
    d = 128, bf16, prefill_4k's distributions; a 64-slot fp32 cache ~ N(0, 0.05), the
    sequences on every other slot, updated in place. Algorithmic bytes: 1540 per
    token-head plus each sequence's state read and written."""
    H, d = 32, 128
    lens = I.packed_lengths(32, 256, 4096)
    total = sum(lens)
    x = I.prefill_inputs("prefill_4k", device=device, B=1, T=total)
    flat = {n: x[n][0] for n in ("q", "k", "v", "log_alpha", "beta")}
    cu = torch.tensor([0] + list(itertools.accumulate(lens)), device=device, dtype=torch.int32)
    g = torch.Generator(device=device).manual_seed(12)
    cache = 0.05 * torch.randn(64, H, d, d, device=device, generator=g)
    slot = torch.arange(0, 64, 2, device=device, dtype=torch.int32)
    out = torch.empty(total, H, d, device=device, dtype=torch.bfloat16)
    engine = "tc_cluster" if kda.engine_supported("tc_cluster", d, d, 64, torch.bfloat16) else "generic"
    ws = torch.empty(max(1, kda.varlen_workspace_bytes(len(lens), H, d, d)), device=device, dtype=torch.uint8)

    def step():
        kda.chunk_fwd_varlen(flat["q"], flat["k"], flat["v"], flat["log_alpha"], flat["beta"], cu,
                             cache, slot=slot, out=out, engine=engine, workspace=ws, stream=stream)

    step()
    torch.cuda.synchronize(device)
    evs = time_events(step, max(1, min(args.steps, 5)), stream)
    torch.cuda.synchronize(device)
    ms = statistics.mean(s.elapsed_time(e) for s, e in evs)
    bytes_alg = total * H * (3 * 2 * d + 4 * d + 4 + 2 * d) + len(lens) * H * 2 * d * d * 4
    hbm, src = peaks()
    gbs = bytes_alg / (ms / 1e3) / 1e9
    return {"entry": "kda_chunk_fwd_varlen", "sequences": len(lens), "tokens": total,
            "lengths": "uniform 256..4096, seed 5", "slots": 64,
            "kernel_ms": round(ms, 3), "tokens_per_s": round(total / (ms / 1e3), 1),
            "bytes_per_launch": bytes_alg, "engine": engine,
            "kernel": ("chunk_cluster_kernel (tensor cores, one 4-CTA cluster per sequence and head)"
                       if engine == "tc_cluster" else "varlen_kernel (fp32 CUDA cores, 16-token chunks)"),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "peak_source": src}}


def run_e2e(kda, w, inp, engine, ws, args, device, stream, world):
    """Same metric through the public call with pinned host buffers: H2D of the
    step's inputs, the prefill, D2H of out and S_T, all inside the timed region."""
    names = ("q", "k", "v", "log_alpha", "beta", "S0")
    host = {n: inp[n].cpu().pin_memory() for n in names if inp[n] is not None}
    dev = {n: torch.empty_like(inp[n]) for n in host}
    out_h = torch.empty(w.B, w.T, w.H, w.dv, dtype=w.dtype).pin_memory()
    st_h = torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32).pin_memory()
    out_d = torch.empty(w.B, w.T, w.H, w.dv, device=device, dtype=w.dtype)
    st_d = torch.empty(w.B, w.H, w.dk, w.dv, device=device, dtype=torch.float32)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + st_h.numel() * st_h.element_size()

    def step():
        for n in host:
            dev[n].copy_(host[n], non_blocking=True)
        kda.chunk_fwd(dev["q"], dev["k"], dev["v"], dev["log_alpha"], dev["beta"], dev.get("S0"),
                      w.chunk, out=out_d, S_T=st_d, engine=engine, workspace=ws, stream=stream)
        out_h.copy_(out_d, non_blocking=True)
        st_h.copy_(st_d, non_blocking=True)

    n = max(1, min(args.steps, 5))
    for _ in range(2):
        step()
    torch.cuda.synchronize(device)
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(n):
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    rate, ms = weak_scaling_rate(w.tokens, t0.elapsed_time(t1), world, device, n)
    return {"value": round(rate, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3),
            "steps": n}


def run_decode(kda, args, device, stream, world):
    """decode_256: state cache [256,32,128,128] fp32 in place, fresh inputs per step."""
    w = I.WORKLOADS[DECODE]
    n_steps = args.decode_steps
    state = I.decode_state(w, device=device)
    steps = [I.decode_step_inputs(w, s, device=device) for s in range(n_steps)]
    out = torch.empty(w.N, w.H, w.dv, device=device, dtype=w.dtype)

    def run(s):
        x = steps[s]
        kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state, out=out,
                           stream=stream)

    for s in range(min(args.warmup, n_steps)):
        run(s)
    torch.cuda.synchronize(device)
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    per = []
    t0.record(stream)
    for s in range(n_steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run(s)
        b.record(stream)
        per.append((a, b))
    t1.record(stream)
    torch.cuda.synchronize(device)
    tok_rate, ms_loop = weak_scaling_rate(w.N, t0.elapsed_time(t1), world, device, n_steps)
    kern = sorted(a.elapsed_time(b) for a, b in per)
    med = kern[len(kern) // 2]
    hbm, src = peaks()
    bytes_step = decode_state_bytes(w)
    gbs = bytes_step / (med / 1e3) / 1e9
    return {"workload": DECODE, "steps": n_steps, "us_per_step_median": round(med * 1e3, 2),
            "us_per_step_p10": round(kern[len(kern) // 10] * 1e3, 2),
            "us_per_step_p90": round(kern[(9 * len(kern)) // 10] * 1e3, 2),
            "us_per_step_loop": round(ms_loop * 1e3, 2),
            "state_bytes_per_step": bytes_step, "state_GBps": round(gbs, 1),
            "frac_of_8TBps": round(gbs / NOMINAL_HBM_GBS, 4),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "peak_source": src,
                         "traffic": traffic_from_profiles("decode")},
            "tokens_per_s": round(tok_rate, 1),
            "launches": n_steps}


def run_only(args, device):
    """Profiling mode: warm-up + timed launches of one kernel, no extra work around them."""
    import gated_delta_rule_116_b200 as kda

    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    if args.only == "prefill":
        w = I.WORKLOADS[args.workload or PREFILL]
        inp = I.prefill_inputs(w, device=device)
        q, k, v, la, beta, S0 = (inp[x] for x in ("q", "k", "v", "log_alpha", "beta", "S0"))
        out = torch.empty(w.B, w.T, w.H, w.dv, device=device, dtype=w.dtype)
        S_T = torch.empty(w.B, w.H, w.dk, w.dv, device=device, dtype=torch.float32)
        ws_n = kda.workspace_bytes(w.B, w.T, w.H, w.dk, w.dv, w.chunk, w.dtype)
        ws = torch.empty(max(ws_n, 1), device=device, dtype=torch.uint8) if ws_n else None
        eng = args.engine or "auto"
        fn = lambda: kda.chunk_fwd(q, k, v, la, beta, S0, w.chunk, out=out, S_T=S_T, engine=eng,
                                   workspace=ws, stream=stream)
    else:
        w = I.WORKLOADS[DECODE]
        state = I.decode_state(w, device=device)
        x = I.decode_step_inputs(w, 0, device=device)
        out = torch.empty(w.N, w.H, w.dv, device=device, dtype=w.dtype)
        fn = lambda: kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state,
                                        out=out, stream=stream)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize(device)
    evs = time_events(fn, args.steps, stream)
    torch.cuda.synchronize(device)
    ms = [s.elapsed_time(e) for s, e in evs]
    print(f"{args.only} {w.name}: {len(ms)} launches, median {sorted(ms)[len(ms) // 2]:.4f} ms",
          flush=True)


# ---------------------------------------------------------------------------- CPU oracle

def cpu_baseline(args, gpu_inputs=None, gpu_out=None, gpu_st=None):
    """The fp64 oracle, as it stands, on a bounded sample of prefill_32k.

    With the bench's own device inputs and results, the oracle runs on exactly
    those inputs (copied to the host) and its output is compared element by
    element with the GPU's over the whole sample: the line then reports the
    parity margin of the timed workload itself (max-abs, max-rel and worst
    error / bound for the bf16 bound |x - ref| <= 2e-3 + 1e-2 |ref|)."""
    import numpy as np
    import oracle

    w = I.WORKLOADS[PREFILL]
    cores = os.cpu_count() or 1
    threads = max(1, min(cores, args.cpu_threads or cores))
    n_heads = w.H
    T_s = min(w.T, args.cpu_tokens)
    if gpu_inputs is not None:
        cut = lambda x: None if x is None else x[:, :T_s].cpu()
        inp = {n: cut(gpu_inputs[n]) for n in ("q", "k", "v", "log_alpha", "beta")}
        inp["S0"] = None if gpu_inputs["S0"] is None else gpu_inputs["S0"].cpu()
    else:
        inp = I.prefill_inputs(w, T=T_s, H=n_heads)
    t = time.perf_counter()
    ref_o, ref_s = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                  inp["S0"], nthreads=threads)
    dt = time.perf_counter() - t
    tok_s = T_s * (n_heads / w.H) / dt
    used = min(threads, n_heads)
    res = {"value": round(tok_s, 2), "unit": "tokens/s", "cores": used, "kind": "oracle",
           "sample": f"fp64 oracle on {n_heads} of {w.H} heads x first {T_s} tokens of {PREFILL} "
                     f"({dt:.1f} s); tokens/s scaled by heads/{w.H}",
           "host_cores": cores}
    if gpu_out is not None:
        def margin(x, ref):
            x = x.double().cpu().numpy()
            err = np.abs(x - ref)
            return {"max_abs": float(err.max()),
                    "max_rel": float((err / np.maximum(np.abs(ref), 1e-30)).max()),
                    "worst_err_over_bound": float((err / (2e-3 + 1e-2 * np.abs(ref))).max())}
        par = {"out": margin(gpu_out[:, :T_s], ref_o), "elements": int(ref_o.size)}
        if T_s == w.T:
            par["S_T"] = margin(gpu_st, ref_s)
        par["bound"] = "|x - ref| <= 2e-3 + 1e-2 |ref| (bf16 inputs, fp32 state)"
        res["parity"] = par
    return res


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle

    w = I.WORKLOADS[PREFILL]
    cores = os.cpu_count() or 1
    n_heads = max(1, min(w.H, cores))
    T_s = min(w.T, args.cpu_tokens_ref)
    inp = I.prefill_inputs(w, T=T_s, H=n_heads)

    def step():
        oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                       nthreads=cores)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t) / args.steps
    tok_s = T_s * (n_heads / w.H) / dt
    sample = (f"fp64 oracle on {n_heads} of {w.H} heads x first {T_s} tokens of {PREFILL} per "
              f"step; tokens/s scaled by heads/{w.H}")
    line = {"impl": "reference", "metric": METRIC, "value": round(tok_s, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; recipe in kda_inputs.py)",
            "config": {"workload": PREFILL, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "chunk": w.chunk},
            "cpu_baseline": {"value": round(tok_s, 2), "unit": "tokens/s",
                             "cores": min(cores, n_heads), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(tok_s, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------- plumbing

def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank, ms_local, world, device, steps=1):
    """Whole-job rate when every rank does the same work: the units of all ranks
    over the slowest rank's time. Returns (units per second, slowest ms per step)."""
    ms_step = max_over_ranks(ms_local, world, device) / steps
    return units_per_rank * world / (ms_step / 1e3), ms_step


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--cpu-tokens", type=int, default=32768,
                    help="tokens per head of the CPU oracle sample")
    ap.add_argument("--cpu-tokens-ref", type=int, default=2048,
                    help="tokens per head per step of the reference arm")
    ap.add_argument("--cpu-threads", type=int, default=0)
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-extra-legs", action="store_true",
                    help="skip the backward and variable-length legs")
    ap.add_argument("--only", choices=["prefill", "decode"],
                    help="profiling mode: run just this kernel's workload (warm-up + steps), "
                         "print its time, no JSON line")
    ap.add_argument("--engine", default=None, choices=["auto", "generic", "tc_cluster"],
                    help="with --only prefill: the prefill engine (default auto)")
    ap.add_argument("--workload", default=None,
                    help="with --only prefill: the prefill workload to run (default prefill_32k)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        print("note: at least 3 warm-up steps are used", file=sys.stderr)
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)

    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.cuda.set_device(device)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        if args.only:
            run_only(args, device)
            return 0
        run_ours(args, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
