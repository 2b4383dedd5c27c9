#!/usr/bin/env python3
"""Throughput of the quantized latent-MoE layer on B200.

One step = one call of the whole layer (activation quantiser, D projection,
router + top-k + bucketing, grouped gate/up + SwiGLU + requant, grouped down,
weighted combine + requant, U projection) on one batch of synthetic input.
The default workload is single-token decode: T=1, H=4096, latent L=1792, 128
experts top-8, expert FFN I=1024, Q8_0 weights, bf16 input, router bias
N(0, 1) per expert.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl elq|reference]
                  [--workload decode|verify|prefill|prefill_nvfp4|decode_nvfp4|decode_q4_k|decode_q3_k|stack|tiny]
                  [--f16 auto|on|off]

--f16: the layers also hold their Q8_0 codes widened to fp16, so that calls
taking the tensor-core path (T >= 16) multiply fp16 operands into exact fp32
accumulators (the same results); auto = on for the workloads with T >= 16
except the 48-layer stack (whose copies would take ~70 GB more).

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
synchronize on both sides, timed with CUDA events on the launching stream; the
max over ranks is taken.  Each rank runs its own replica on its own inputs
(no data-path collective).  The working set per step is ~63 MB, below the
126 MB L2, so the steps rotate over 8 distinct layer copies and 64 inputs:
between two uses of the same weights 7 other layers' weights (~440 MB) pass
through L2.

--impl reference times the CPU oracle (the test-suite's scalar C statement of
the layer) on the host cores on the same workload, one token per step.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "latent-MoE layer tokens/s; expert-weight HBM GB/s and % of B200 peak"
KERNELS_SMALL_T = ["proj_D", "router", "gate_up", "down", "proj_U"]
KERNELS_LARGE_T = ["quant_x", "proj_D", "router", "gate_up", "down", "proj_U"]
KERNELS_TC = ["quant_x", "pack_x", "proj_D", "router", "slot_map", "pack_z", "gate_up", "down", "combine",
              "proj_U"]
KERNELS_NVTC = ["quant_x", "pack_x", "proj_D", "quant_z", "router", "slot_map", "pack_z", "gate_up", "down",
                "combine", "proj_U"]
KERNELS_FUSED = ["layer"]
KERNEL_NAMES = {"gate_up": {5: "k_sgemv<{fmt}> gate/up (cluster GEMV, +SwiGLU, {afmt})",
                            6: "k_wgemv<{fmt}> gate/up (+SwiGLU, Q8_1)",
                            10: "k_tcgemm gate/up (tcgen05 kind::{kind}, +SwiGLU)",
                            11: "k_nvgemm gate/up (tcgen05 kind::mxf4nvf4 block-scaled, +SwiGLU, NVFP4)"},
                "layer": {1: "k_decode_layer (the whole layer: D, router, gate/up, down + combine, U; one launch)"}}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 4096; the stack: 64)")
    ap.add_argument("--warmup", type=int, default=None, help="warm-up steps (default 64; the stack: 4)")
    ap.add_argument("--impl", default="elq", choices=["elq", "reference"])
    ap.add_argument("--workload", default="decode")
    ap.add_argument("--copies", type=int, default=8, help="distinct layer copies rotated over")
    ap.add_argument("--inputs", type=int, default=64, help="distinct inputs rotated over")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="bounded CPU-baseline sample")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--f16", default="auto", choices=["auto", "on", "off"],
                    help="fp16 codes for the tensor-core GEMMs (auto: on for T >= 16)")
    ap.add_argument("--fused", action="store_true",
                    help="small T as the single persistent kernel instead of the separate-kernel sequence")
    ap.add_argument("--no-clocks", action="store_true",
                    help="no nvidia-smi sampling (for runs under a profiler; the line is then not a bench value)")
    ap.add_argument("--no-long", action="store_true",
                    help="skip the long-run median (for runs under a profiler)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def workload_desc(wl):
    wfmt = wl.fmt.upper() if wl.expert_fmt == wl.fmt else "%s D/U and %s expert" % (wl.fmt.upper(),
                                                                                  wl.expert_fmt.upper())
    return ("T=%d, H=%d, L=%d, E=%d, top-%d, I=%d, %s weights, %s input, router bias %s"
            % (wl.T, wl.H, wl.L, wl.E, wl.k, wl.I, wfmt, wl.x_dtype, wl.bias))


def nvfp4_globals(w):
    """Per-matrix NVFP4 global scales of w [n, ...]: amax / 2688 in fp32 (1 if all zero)."""
    import torch
    amax = w.reshape(w.shape[0], -1).abs().amax(dim=1)
    g = amax / torch.tensor(2688.0, dtype=torch.float32, device=w.device)
    return torch.where(amax > 0, g, torch.ones_like(g))


def use_f16(args, wl):
    """The fp16-operand tensor-core GEMMs: on for the workloads whose calls
    take the tensor-core path (T >= 16), unless --f16 says otherwise."""
    if args.f16 != "auto":
        return args.f16 == "on"
    return wl.T >= 16


def build_layer(elq, synth, wl, li, dev, fused=False, batch=32, f16=False):
    """Layer li of the workload on device dev, quantised by the library
    (f16: also the fp16 codes of its Q8_0 matrices, for the fp16-operand
    tensor-core GEMMs)."""
    import torch
    fmt, efmt = elq.FMT[wl.fmt], elq.FMT[wl.expert_fmt]
    dw = synth.dense_weights(wl, li, device=dev)
    rb = dw["router_bias"]
    ly = elq.Layer.allocate(wl.H, wl.L, wl.E, wl.k, wl.I, fmt, efmt, dw["router_w"],
                            None if rb is None else rb.to(dev), device=dev)
    ly.set_dense(dw["D"], dw["U"])
    if fused:
        ly.flags = elq.LAYER_FUSED
    if efmt == elq.NVFP4:
        ly.act_gz = ly.act_gh = synth.NVFP4_ACT_GSCALE
    for e0 in range(0, wl.E, batch):
        n = min(batch, wl.E - e0)
        if wl.expert_fmt in ("q5_1", "q3_k", "q4_k", "q5_k"):
            # pre-quantised GGUF blocks, packed into the arena
            bs = [synth.expert_blocks(wl, e, li) for e in range(e0, e0 + n)]
            ly.set_expert_blocks(e0, *(torch.stack([b[i] for b in bs]).to(dev) for i in range(3)))
            del bs
            continue
        ws_ = [synth.expert_weights(wl, e, li, device=dev) for e in range(e0, e0 + n)]
        g, u, d = (torch.stack([w[i] for w in ws_]) for i in range(3))
        if efmt == elq.NVFP4:
            ly.set_experts_nvfp4(e0, g, u, d, nvfp4_globals(torch.cat([g, u], dim=1)), nvfp4_globals(d))
        else:
            ly.set_experts(e0, g, u, d)
        del ws_, g, u, d
    if f16:
        ly.enable_f16()
    return ly


# ---------------------------------------------------------------------------
# clocks during the timed region

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.rows = []
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), "--query-gpu=" + self.Q, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self, t0, t1):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r for (t, r) in self.rows if t0 - 0.15 <= t <= t1 + 0.15] or [r for (_, r) in self.rows[-3:]]
        sm = [float(r[1]) for r in rows if len(r) > 2 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) > 2 and r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for i, n in enumerate(names):
                if len(r) > 5 + i and r[5 + i].lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the CPU oracle (cpu_baseline and the reference arm)

CPU_TOKENS = 4          # tokens per oracle call in the CPU samples (the oracle's cost is linear in tokens)


def oracle_setup(wl, n_tokens, gen_device, tokens=None):
    """Oracle layer with the experts that n_tokens distinct inputs of
    `tokens` tokens each (default: the workload's T) route to."""
    import numpy as np
    import oracle
    from quantized_latent_moe_b200 import synth
    fmts = {"q8_0": oracle.Q8_0, "q4_0": oracle.Q4_0, "nvfp4": oracle.NVFP4, "q5_1": oracle.Q5_1,
            "q3_k": oracle.Q3_K, "q4_k": oracle.Q4_K, "q5_k": oracle.Q5_K}

    def g(t):
        return t.to("cpu").numpy()

    dw = synth.dense_weights(wl, 0, device=gen_device)
    w = {k: (None if v is None else g(v)) for k, v in dw.items()}
    w["gate"] = None
    if wl.expert_fmt == synth.NVFP4:
        w["act_gz"] = w["act_gh"] = synth.NVFP4_ACT_GSCALE
    ly = oracle.Layer(wl.H, wl.L, wl.E, wl.k, wl.I, fmts[wl.fmt], fmts[wl.expert_fmt], w)
    xs = [g(synth.make_x(wl, step=s, T=tokens, device=gen_device).float()) for s in range(n_tokens)]
    need = set()
    for x in xs:
        idx, _ = ly.route(x)
        need |= set(idx.reshape(-1).tolist())
    gate, up, down = [None] * wl.E, [None] * wl.E, [None] * wl.E
    for e in sorted(need):
        if wl.expert_fmt in ("q5_1", "q3_k", "q4_k", "q5_k"):
            a, b, c = synth.expert_blocks(wl, e, 0)
        else:
            a, b, c = synth.expert_weights(wl, e, 0, device=gen_device)
        gate[e], up[e], down[e] = g(a), g(b), g(c)
    ly.set_experts({"gate": gate, "up": up, "down": down}, sorted(need))
    return ly, xs


def oracle_run(ly, xs, steps, threads):
    """Run `steps` oracle layer calls (token s % len(xs) each) over `threads`
    host threads (the C calls release the GIL); returns wall seconds."""
    n = max(1, threads)
    share = [steps // n + (1 if i < steps % n else 0) for i in range(n)]
    start = [sum(share[:i]) for i in range(n)]

    def work(i):
        for s in range(start[i], start[i] + share[i]):
            ly.forward(xs[s % len(xs)])

    ths = [threading.Thread(target=work, args=(i,)) for i in range(n)]
    t0 = time.perf_counter()
    for t in ths:
        t.start()
    for t in ths:
        t.join()
    return time.perf_counter() - t0


def host_threads():
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(n, 32))


def cpu_baseline(wl, seconds, gen_device):
    tok = min(wl.T, CPU_TOKENS)
    ly, xs = oracle_setup(wl, 2, gen_device, tok)
    threads = host_threads()
    t1 = oracle_run(ly, xs, threads, threads)          # calibration: one call per thread
    steps = max(threads, int(seconds / max(t1, 1e-6) * threads))
    dt = oracle_run(ly, xs, steps, threads)
    return {"value": steps * tok / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": "%d %s layer calls of %d token(s) each (2 distinct inputs, their %d experts "
                      "pre-quantised by the oracle), %.1f s wall on %d host threads"
                      % (steps, wl.name, tok, sum(g is not None for g in ly.gate), dt, threads)}


def run_reference(args):
    from quantized_latent_moe_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    gen = "cpu"
    try:
        import torch
        if torch.cuda.is_available():
            gen = "cuda"
    except Exception:
        pass
    tok = min(wl.T, CPU_TOKENS)
    ly, xs = oracle_setup(wl, 2, gen, tok)
    threads = host_threads()
    oracle_run(ly, xs, args.warmup, threads)
    dt = oracle_run(ly, xs, args.steps, threads)
    value = args.steps * tok / dt / wl.layers      # a stack step runs every layer
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic", "config": {"workload": "%s: %s" % (wl.name, workload_desc(wl)),
                                        "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": "each step: one layer call of %d token(s) on the scalar C oracle "
                                   "(2 distinct inputs alternating), steps spread over %d host threads%s"
                                   % (tok, threads, "" if wl.layers == 1 else
                                      "; tokens/s of the %d-layer stack = one layer's rate / %d"
                                      % (wl.layers, wl.layers))},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA path

_INT8_PEAK = None


def tensor_peak_int8():
    """Dense int8 tensor-core peak (TOPS), measured on this GPU: one CTA per
    SM issuing back-to-back tcgen05.mma kind::i8 (M=128, N=256, K=32) from
    shared memory into TMEM (elq_test_mma_i8_rate), timed with CUDA events
    on the launching stream after a warm-up launch; the best of five launches
    (a burst figure, like the measured bf16 peak)."""
    global _INT8_PEAK
    if _INT8_PEAK is not None:
        return _INT8_PEAK
    import torch
    from quantized_latent_moe_b200 import elq
    stream = torch.cuda.current_stream()
    n_mma = 32768
    ops = 2.0 * 128 * 256 * 32 * n_mma * elq.sm_count()
    elq.test_mma_i8_rate(256)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        _, err = elq.test_mma_i8_rate(n_mma)
        e1.record(stream)
        e1.synchronize()
        if int(err.item()) != 0:
            raise RuntimeError("int8 rate kernel: a bounded wait ran out")
        best = max(best, ops / (e0.elapsed_time(e1) / 1e3) / 1e12)
    _INT8_PEAK = (best, "measured int8 (tcgen05.mma kind::i8 M128 N256 K32 loop, one CTA per SM, best of 5)")
    return _INT8_PEAK


_F16_PEAK = None


def tensor_peak_f16():
    """Dense fp16 tensor-core peak (TFLOP/s), measured as tensor_peak_int8 is,
    with tcgen05.mma kind::f16 (M=128, N=256, K=16; elq_test_mma_f16_rate)."""
    global _F16_PEAK
    if _F16_PEAK is not None:
        return _F16_PEAK
    import torch
    from quantized_latent_moe_b200 import elq
    stream = torch.cuda.current_stream()
    n_mma = 32768
    ops = 2.0 * 128 * 256 * 16 * n_mma * elq.sm_count()
    elq.test_mma_f16_rate(256)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        _, err = elq.test_mma_f16_rate(n_mma)
        e1.record(stream)
        e1.synchronize()
        if int(err.item()) != 0:
            raise RuntimeError("fp16 rate kernel: a bounded wait ran out")
        best = max(best, ops / (e0.elapsed_time(e1) / 1e3) / 1e12)
    _F16_PEAK = (best, "measured fp16 (tcgen05.mma kind::f16 M128 N256 K16 loop, one CTA per SM, best of 5)")
    return _F16_PEAK


_FP4_PEAK = None


def tensor_peak_fp4():
    """Dense fp4 block-scaled tensor-core peak (TFLOP/s), measured on this GPU:
    one CTA per SM issuing back-to-back tcgen05.mma kind::mxf4nvf4 (M=128,
    N=256, K=64) from shared memory into TMEM (elq_test_mma_nvf4_rate); the
    best of five launches after a warm-up one (a burst figure)."""
    global _FP4_PEAK
    if _FP4_PEAK is not None:
        return _FP4_PEAK
    import torch
    from quantized_latent_moe_b200 import elq
    stream = torch.cuda.current_stream()
    n_mma = 32768
    flops = 2.0 * 128 * 256 * 64 * n_mma * elq.sm_count()
    elq.test_mma_nvf4_rate(256)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        _, err = elq.test_mma_nvf4_rate(n_mma)
        e1.record(stream)
        e1.synchronize()
        if int(err.item()) != 0:
            raise RuntimeError("fp4 rate kernel: a bounded wait ran out")
        best = max(best, flops / (e0.elapsed_time(e1) / 1e3) / 1e12)
    _FP4_PEAK = (best, "measured fp4 (tcgen05.mma kind::mxf4nvf4 block-scaled M128 N256 K64 loop, one CTA per SM, "
                       "best of 5)")
    return _FP4_PEAK


_F32X2_RATE = None


def f32x2_rate():
    """Packed fp32 instructions per second (fma.rn.f32x2, each two fused
    multiply-adds), measured on this GPU: 2 CTAs of 1024 threads per SM, 8
    independent chains per thread (elq_test_f32x2_rate), timed with CUDA
    events on the launching stream; the best of five launches."""
    global _F32X2_RATE
    if _F32X2_RATE is not None:
        return _F32X2_RATE
    import torch
    from quantized_latent_moe_b200 import elq
    stream = torch.cuda.current_stream()
    n = 4096
    instr = 2.0 * elq.sm_count() * 1024 * n * 8
    elq.test_f32x2_rate(64)
    torch.cuda.synchronize()
    best = 0.0
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        elq.test_f32x2_rate(n)
        e1.record(stream)
        e1.synchronize()
        best = max(best, instr / (e0.elapsed_time(e1) / 1e3))
    _F32X2_RATE = best
    return best


def source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_latent_moe_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """dram bytes per launch of `kernel` from the committed ncu summary, only if
    it was taken on the current kernel sources and on this workload."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get("%s@%s" % (kernel, workload)) or d.get(kernel)
    if not e or e.get("source_hash") != source_hash() or e.get("workload") != workload:
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(values, world, device):
    """Each rank's device times -> the max over ranks (every rank gets it);
    the job is as slow as its slowest rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


class GraphSet:
    """CUDA graphs of n consecutive steps, keyed by (n, first step mod period):
    step(i) depends on i only through i mod period, so one graph serves every
    run of n steps starting at the same phase.  prepare() captures (and
    replays once) every graph a later run() will use, so that a timed run()
    replays graphs and never captures one."""

    def __init__(self, G, step, period=None):
        self.G, self.step = G, step
        self.period = G if period is None else period
        self.graphs = {}

    def keys(self, k, start):
        out, done = [], 0
        while done < k:
            n = min(self.G, k - done)
            out.append((n, (start + done) % self.period))
            done += n
        return out

    def _get(self, key):
        import torch
        g = self.graphs.get(key)
        if g is None:
            n, ph = key
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(ph, ph + n):
                    self.step(i)
            self.graphs[key] = g
        return g

    def prepare(self, k, start):
        for key in dict.fromkeys(self.keys(k, start)):
            if key not in self.graphs:
                self._get(key).replay()

    def run(self, k, start=0):
        for key in self.keys(k, start):
            self._get(key).replay()
        return start + k

    def long_run(self, stream, start, min_ms=300.0, min_steps=400):
        """Device time per step over a long run of full graphs: replays for at
        least min_ms of warm-up, then at least min_steps steps and min_ms,
        each replay timed with CUDA events on the launching stream; the
        median over replays (ms per step)."""
        import torch
        key = (self.G, start % self.period)
        g = self._get(key)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        t0 = time.perf_counter()
        while (time.perf_counter() - t0) * 1e3 < min_ms:
            g.replay()
            torch.cuda.synchronize()
        per, steps, total = [], 0, 0.0
        while steps < min_steps or total < min_ms:
            ev[0].record(stream)
            g.replay()
            ev[1].record(stream)
            ev[1].synchronize()
            ms = ev[0].elapsed_time(ev[1])
            per.append(ms / self.G)
            steps += self.G
            total += ms
        return {"ms_per_step_median": statistics.median(per), "ms_per_step_mean": total / steps,
                "steps": steps, "replays": len(per), "warmup_ms": min_ms,
                "note": "median over replays of %d-step graphs after at least %.0f ms of warm-up"
                        % (self.G, min_ms)}

    def clear(self):
        self.graphs.clear()


def run_elq(args):
    import torch
    import torch.distributed as dist

    from quantized_latent_moe_b200 import build, elq, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    elq.lib()
    wl = synth.WORKLOADS[args.workload]
    stream = torch.cuda.current_stream()

    # distinct layer copies (layer index = copy + 8 * rank) and inputs
    layers = [build_layer(elq, synth, wl, c + args.copies * rank, dev, args.fused, f16=use_f16(args, wl))
              for c in range(args.copies)]
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    S = args.inputs
    xs = [synth.make_x(wl, step=s + 1000 * rank, device=dev) for s in range(S)]
    ys = [torch.empty(wl.T, wl.H, dtype=torch.float32, device=dev) for _ in range(2)]
    ws = layers[0].workspace(wl.T)
    for ly in layers[1:]:
        ly.share_workspace(wl.T, ws)   # steps are serial on the stream: one workspace serves all

    def step(i, y=None):
        elq.moe_layer(layers[i % args.copies], xs[i % S], ys[i % 2] if y is None else y, ws)

    # eager warm-up of every (layer, input) pairing used, then a graph of G steps
    for i in range(max(args.copies, 2)):
        step(i)
    torch.cuda.synchronize()
    assert elq.workspace_status(ws) == 0
    G = math.lcm(args.copies, S, 2)
    if wl.T > 64:
        G = min(G, 16)
    graphs = GraphSet(G, step)

    launches_per_step = layers[0].kernel_count(wl.T)
    KERNELS = {1: KERNELS_FUSED, 5: KERNELS_SMALL_T, 6: KERNELS_LARGE_T, 10: KERNELS_TC,
               11: KERNELS_NVTC}[launches_per_step]
    pos = graphs.run(args.warmup)
    # every graph the timed steps replay is captured, instantiated and
    # replayed once here: the timed region holds replays only
    graphs.prepare(args.steps, pos)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = None if args.no_clocks else Clocks(local)
    time.sleep(0.3)
    t_wall0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record(stream)
    pos = graphs.run(args.steps, pos)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    dev_ms = e0.elapsed_time(e1)
    long_run = None if args.no_long else graphs.long_run(stream, pos)

    # end to end through the C ABI with host buffers: pinned x in, y out, every step
    x_host = [x.cpu().pin_memory() for x in xs[:8]]
    nh = len(x_host)
    y_host = torch.empty(wl.T, wl.H, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(xs[0])
    y_dev = torch.empty(wl.T, wl.H, dtype=torch.float32, device=dev)
    for i in range(8):
        x_dev.copy_(x_host[i % nh], non_blocking=True)
        elq.moe_layer(layers[i % args.copies], x_dev, y_dev, ws)
        y_host.copy_(y_dev, non_blocking=True)
        stream.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(args.steps):
        x_dev.copy_(x_host[i % nh], non_blocking=True)
        elq.moe_layer(layers[i % args.copies], x_dev, y_dev, ws)
        y_host.copy_(y_dev, non_blocking=True)
        stream.synchronize()
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1)

    # per-kernel device time: the same steps with an event after every kernel.
    # Eager launches behind a queued GPU sleep, so the host runs ahead and the
    # kernels execute back to back (events cannot be timed inside a graph).
    nk = launches_per_step
    prof_steps = min(args.steps, 1024)
    per = [[] for _ in range(nk)]
    GP = 32
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(GP)]
    for row in evs:             # torch creates the CUDA event at its first record
        for ev in row:
            ev.record(stream)
    torch.cuda.synchronize()
    done = 0
    while done < prof_steps:
        n = min(GP, prof_steps - done)
        torch.cuda._sleep(20_000_000)
        for i in range(n):
            j = done + i
            elq.moe_layer_profiled(layers[j % args.copies], xs[j % S], ys[j % 2], evs[i], ws)
        torch.cuda.synchronize()
        for i in range(n):
            for j in range(nk):
                per[j].append(evs[i][j].elapsed_time(evs[i][j + 1]))
        done += n
    t_wall1 = time.time()
    clocks = {"sampled": False} if clk is None else clk.stop(t_wall0, t_wall1)
    kern_ms = [statistics.mean(v) for v in per]

    # routed experts per step (for the algorithmic bytes of the expert kernels)
    n_act = []
    for i in range(min(S, 64)):
        elq.moe_layer(layers[0], xs[i], ys[0], ws)
        torch.cuda.synchronize()
        n_act.append(int(elq.workspace_view(layers[0], wl.T, "n_act", ws).item()))
    act = statistics.mean(n_act)

    # max over ranks
    dev_ms, e2e_ms = max_over_ranks([dev_ms, e2e_ms], world, dev)

    if rank == 0:
        blk = 34 if wl.fmt == "q8_0" else 18              # D and U blocks
        # expert bytes per 32 values as the kernels read them (GGUF sizes; the
        # K-quants' arena carries 20 B per 32 values: 16 codes + a scale word)
        eblk = {"q8_0": 34, "q4_0": 18, "nvfp4": 18, "q5_1": 24, "q3_k": 20, "q4_k": 20, "q5_k": 24}[wl.expert_fmt]
        ablk = 18 if wl.expert_fmt == "nvfp4" else 36     # the experts' activation blocks
        nb_L, nb_H, nb_I = wl.L // 32, wl.H // 32, wl.I // 32
        gu_w = act * 2 * wl.I * nb_L * eblk
        dn_w = act * wl.L * nb_I * eblk
        du_w = (wl.L * nb_H + wl.H * nb_L) * blk
        rt_w = wl.E * wl.L * 4
        P = wl.T * wl.k
        tokens = args.steps * wl.T * world
        value = tokens / (dev_ms / 1e3)
        hbm_peak, peak_kind = peaks()
        step_s = dev_ms / 1e3 / args.steps
        layer_bytes = gu_w + dn_w + du_w + rt_w
        # activations the layer must read or write once: x, y, and the Q8_1 rows between the steps
        x_bytes = wl.T * wl.H * (2 if wl.x_dtype == "bf16" else 4)
        act_bytes = x_bytes + wl.T * wl.H * 4 + wl.T * nb_L * (36 + ablk) + P * nb_I * ablk
        if launches_per_step == 1:
            lay_ms = kern_ms[0]
            gu_ms = dn_ms = None
            lb = layer_bytes + act_bytes
            achieved = lb / (lay_ms / 1e3) / 1e9
            roof = {"bound": "hbm", "kernel": KERNEL_NAMES["layer"][1], "achieved": achieved, "peak": hbm_peak,
                    "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm_peak,
                    "traffic": traffic_for("layer", wl.name), "algorithmic_bytes_per_launch": lb}
        else:
            gu_ms = kern_ms[KERNELS.index("gate_up")]
            dn_ms = kern_ms[KERNELS.index("down")]
        if launches_per_step == 1:
            pass
        elif launches_per_step == 11:
            # block-scaled fp4 tensor cores: gate/up is a contraction, against the measured fp4 rate
            gu_ops = 2.0 * (2 * wl.I) * P * wl.L
            tpk, tkind = tensor_peak_fp4()
            achieved = gu_ops / (gu_ms / 1e3) / 1e12
            # HBM: the codes and the scale atoms of every routed expert, z's and h's packed rows
            gu_io = act * 2 * wl.I * wl.L * (0.5 + 1.0 / 16) + P * wl.L * (0.5 + 1.0 / 16) + P * wl.I * (0.5 + 1.0 / 16)
            t_tensor = gu_ops / (tpk * 1e12)
            t_hbm = gu_io / (hbm_peak * 1e9)
            t_meas = gu_ms / 1e3
            roof = {"bound": "tensor", "kernel": KERNEL_NAMES["gate_up"][11], "achieved": achieved, "peak": tpk,
                    "peak_kind": tkind, "unit": "TFLOP/s (fp4)",
                    "frac": achieved / tpk, "traffic": traffic_for("gate_up_nv", wl.name),
                    "algorithmic_ops_per_launch": gu_ops, "algorithmic_bytes_per_launch": gu_io,
                    "fractions": {"tensor": t_tensor / t_meas, "hbm": t_hbm / t_meas,
                                  "max_bound": max(t_tensor, t_hbm) / t_meas,
                                  "bound_us": {"tensor": t_tensor * 1e6, "hbm": t_hbm * 1e6}}}
        elif launches_per_step == 10:
            # tensor-core path: gate/up is a contraction, on int8 or on fp16-widened codes (the
            # peak of the MMA kind that ran, measured here)
            gu_ops = 2.0 * (2 * wl.I) * P * wl.L
            f16 = use_f16(args, wl)
            tpk, tkind = tensor_peak_f16() if f16 else tensor_peak_int8()
            achieved = gu_ops / (gu_ms / 1e3) / 1e12
            roof = {"bound": "tensor", "kernel": KERNEL_NAMES["gate_up"][10].format(kind="f16" if f16 else "i8"),
                    "achieved": achieved, "peak": tpk, "peak_kind": tkind,
                    "unit": "TFLOP/s (fp16 operands)" if f16 else "TOPS (int8)", "frac": achieved / tpk,
                    "traffic": traffic_for("gate_up_tc", wl.name), "algorithmic_ops_per_launch": gu_ops,
                    "algorithmic_bytes_per_launch": gu_w}
            # the launch's three bounds: tensor ops, HBM bytes (fp16 codes: the
            # weights' code bytes twice), and the fp32 epilogue (per 32-value
            # block of every output element one scale product and one fused
            # multiply-add, plus with int8 accumulators the int-to-float
            # subtract, as packed pairs: 1.0 or 1.5 fma.rn.f32x2-rate
            # instructions per element-block)
            gu_codes = float(wl.E) * (2 * wl.I) * wl.L
            gu_io = gu_w + (gu_codes if f16 else 0.0) + wl.T * nb_L * 36 + P * nb_I * 36
            elem_blocks = float(P) * (2 * wl.I) * nb_L
            f2r = f32x2_rate()
            t_tensor = gu_ops / (tpk * 1e12)
            t_hbm = gu_io / (hbm_peak * 1e9)
            t_epi = elem_blocks * (1.0 if f16 else 1.5) / f2r
            t_meas = gu_ms / 1e3
            roof["fractions"] = {
                "tensor": t_tensor / t_meas, "hbm": t_hbm / t_meas, "epilogue": t_epi / t_meas,
                "max_bound": max(t_tensor, t_hbm, t_epi) / t_meas,
                "bound_us": {"tensor": t_tensor * 1e6, "hbm": t_hbm * 1e6, "epilogue": t_epi * 1e6},
                "f32x2_instr_per_s": f2r, "hbm_bytes_per_launch": gu_io, "element_blocks_per_launch": elem_blocks,
                "note": "each fraction = that bound's time / the launch's event-timed time; the epilogue bound "
                        "uses the measured fma.rn.f32x2 instruction rate"}
        else:
            gu_bytes = gu_w + wl.T * nb_L * ablk + P * nb_I * ablk       # weights + zq + hq
            achieved = gu_bytes / (gu_ms / 1e3) / 1e9
            afmt = "NVFP4" if wl.expert_fmt == "nvfp4" else "Q8_1"
            efmt = wl.expert_fmt.upper()
            roof = {"bound": "hbm",
                    "kernel": KERNEL_NAMES["gate_up"][launches_per_step].format(fmt=efmt, afmt=afmt),
                    "achieved": achieved,
                    "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm_peak,
                    "traffic": traffic_for("gate_up", wl.name), "algorithmic_bytes_per_launch": gu_bytes}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dev_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16" if (use_f16(args, wl) and launches_per_step in (10, 11)) else "int8",
            "data": "synthetic (seeded counter-hash normals; random-init weights of the layer's shape)",
            "config": {"workload": "%s: %s" % (wl.name, workload_desc(wl)),
                       "global_batch": wl.T * world, "parallelism": "replicas" if world > 1 else "1 GPU",
                       "layer_copies": args.copies, "inputs": S,
                       "tc_operands": ("fp16-widened codes (kind::f16)" if use_f16(args, wl) else "int8 codes")
                       if launches_per_step in (10, 11) else None,
                       "l2": "inputs larger than L2: %d layer copies x ~%.0f MB touched per step rotate, "
                             "%.0f MB between reuses of a layer (L2 126 MB)"
                             % (args.copies, layer_bytes / 1e6, (args.copies - 1) * layer_bytes / 1e6),
                       "cuda_graph": "%d steps per graph%s; every graph captured and replayed once before "
                                     "the timed region" % (
                           G, ", one cooperative launch per step" if launches_per_step == 1
                           else ", programmatic dependent launch")},
            "long_run": long_run,
            "expert_weight_gbs": None if gu_ms is None else (gu_w + dn_w) / ((gu_ms + dn_ms) / 1e3) / 1e9,
            "expert_weight_frac": None if gu_ms is None else (gu_w + dn_w) / ((gu_ms + dn_ms) / 1e3) / 1e9 / hbm_peak,
            "layer_weight_gbs": layer_bytes / step_s / 1e9,
            "layer_weight_frac": layer_bytes / step_s / 1e9 / hbm_peak,
            "kernel_ms": dict(zip(KERNELS, kern_ms)),
            "distinct_experts_per_step": act,
            "roofline": roof,
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": xs[0].numel() * xs[0].element_size(),
                    "d2h_bytes_per_step": wl.T * wl.H * 4},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu:
            line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds, "cuda")
        print(json.dumps(line), flush=True)
    graphs.clear()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_stack(args):
    """The resident stack: each step runs one batch of T new tokens through all
    of the workload's layers on one fp32 residual stream (elq_moe_stack)."""
    import torch
    import torch.distributed as dist

    from quantized_latent_moe_b200 import build, elq, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    elq.lib()
    wl = synth.WORKLOADS[args.workload]
    fmt = elq.FMT[wl.fmt]
    stream = torch.cuda.current_stream()
    layers = []
    for l in range(wl.layers):
        li = l + 1000 * rank
        dw = synth.dense_weights(wl, li, device=dev)
        rb = dw["router_bias"]
        ly = elq.Layer.allocate(wl.H, wl.L, wl.E, wl.k, wl.I, fmt, fmt, dw["router_w"],
                                None if rb is None else rb.to(dev), device=dev)
        ly.set_dense(dw["D"], dw["U"])
        for e0 in range(0, wl.E, 32):
            ws_ = [synth.expert_weights(wl, e, li, device=dev) for e in range(e0, min(wl.E, e0 + 32))]
            ly.set_experts(e0, torch.stack([w[0] for w in ws_]), torch.stack([w[1] for w in ws_]),
                           torch.stack([w[2] for w in ws_]))
            del ws_
        layers.append(ly)
        del dw
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    S = min(args.inputs, 16)
    xs = [synth.make_x(wl, step=s + 1000 * rank, device=dev) for s in range(S)]
    h = torch.empty(wl.T, wl.H, dtype=torch.float32, device=dev)
    ws = layers[0].stack_workspace(wl.T)
    lws = ws[:layers[0].workspace_bytes(wl.T)]        # its first part is the layer workspace
    for ly in layers:
        ly.share_workspace(wl.T, lws)

    def step(i):
        elq.moe_stack(layers, xs[i % S], h, ws)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    assert elq.workspace_status(ws) == 0
    G = 4
    graphs = GraphSet(G, step, period=S)
    pos = graphs.run(args.warmup)
    graphs.prepare(args.steps, pos)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = None if args.no_clocks else Clocks(local)
    time.sleep(0.3)
    t_wall0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record(stream)
    pos = graphs.run(args.steps, pos)
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    dev_ms = e0.elapsed_time(e1)
    # end to end: pinned tokens in, the residual stream out, every step
    x_host = [x.cpu().pin_memory() for x in xs[:4]]
    h_host = torch.empty(wl.T, wl.H, dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(xs[0])
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(args.steps):
        x_dev.copy_(x_host[i % len(x_host)], non_blocking=True)
        elq.moe_stack(layers, x_dev, h, ws)
        h_host.copy_(h, non_blocking=True)
        stream.synchronize()
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1)
    # per-kernel times of one layer at this T (first layer, eager, behind a GPU sleep)
    nk = layers[0].kernel_count(wl.T)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)]
    for ev in evs:
        ev.record(stream)
    torch.cuda.synchronize()
    per = [[] for _ in range(nk)]
    for r in range(16):
        torch.cuda._sleep(2_000_000)
        elq.moe_layer_profiled(layers[r % len(layers)], xs[r % S], h, evs, lws)
        torch.cuda.synchronize()
        for j in range(nk):
            per[j].append(evs[j].elapsed_time(evs[j + 1]))
    t_wall1 = time.time()
    clocks = {"sampled": False} if clk is None else clk.stop(t_wall0, t_wall1)
    kern_ms = [statistics.mean(v) for v in per]
    # routed experts of every layer on one step (layer by layer on the same residual stream)
    n_act = []
    h.copy_(xs[0].float())
    for ly in layers:
        hl = h.clone()
        elq.moe_stack([ly], hl, h, ws)
        torch.cuda.synchronize()
        n_act.append(int(elq.workspace_view(ly, wl.T, "n_act", lws).item()))
    dev_ms, e2e_ms = max_over_ranks([dev_ms, e2e_ms], world, dev)
    if rank == 0:
        blk = 34 if wl.fmt == "q8_0" else 18
        nb_L, nb_H, nb_I = wl.L // 32, wl.H // 32, wl.I // 32
        per_layer_dense = (wl.L * nb_H + wl.H * nb_L) * blk + wl.E * wl.L * 4
        expert_bytes = [a * (2 * wl.I * nb_L + wl.L * nb_I) * blk for a in n_act]
        step_bytes = sum(expert_bytes) + wl.layers * per_layer_dense
        tokens = args.steps * wl.T * world
        value = tokens / (dev_ms / 1e3)
        hbm_peak, peak_kind = peaks()
        step_s = dev_ms / 1e3 / args.steps
        names = {5: KERNELS_SMALL_T, 6: KERNELS_LARGE_T, 10: KERNELS_TC}[nk]
        gu_ms = kern_ms[names.index("gate_up")]
        P = wl.T * wl.k
        gu_bytes = n_act[0] * 2 * wl.I * nb_L * blk + wl.T * nb_L * 36 + P * nb_I * 36
        achieved = gu_bytes / (gu_ms / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dev_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic (seeded counter-hash normals; random-init weights of the layer's shape)",
            "config": {"workload": "%s: %d layers on one fp32 residual stream, %s"
                                   % (wl.name, wl.layers, workload_desc(wl)),
                       "global_batch": wl.T * world, "parallelism": "replicas" if world > 1 else "1 GPU",
                       "inputs": S, "l2": "inputs larger than L2: %.1f GB of weights touched per step"
                                         % (step_bytes / 1e9),
                       "cuda_graph": "%d steps per graph; every graph captured and replayed once before "
                                     "the timed region" % G},
            "layer_weight_gbs": step_bytes / step_s / 1e9,
            "layer_weight_frac": step_bytes / step_s / 1e9 / hbm_peak,
            "kernel_ms": dict(zip(names, kern_ms)),
            "distinct_experts_per_layer": statistics.mean(n_act),
            "roofline": {"bound": "hbm", "kernel": ("k_tcgemm gate/up (tcgen05 kind::i8, +SwiGLU), T=%d" if nk == 10
                                                   else "k_wgemv<" + wl.fmt.upper() + "> gate/up (+SwiGLU, Q8_1), T=%d")
                                                  % wl.T,
                         "achieved": achieved, "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": None, "algorithmic_bytes_per_launch": gu_bytes},
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": xs[0].numel() * xs[0].element_size(),
                    "d2h_bytes_per_step": wl.T * wl.H * 4},
            "gpu_launches": (1 + wl.layers * (1 + nk)) * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu:
            cb = cpu_baseline(wl, args.cpu_seconds, "cuda")
            cb["value"] /= wl.layers
            cb["sample"] += "; tokens/s of the whole stack = one layer's rate / %d layers" % wl.layers
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)
    graphs.clear()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def spawn_ranks(n):
    """`bench.py --gpus N` run directly (no torchrun around it): relaunch this
    command as N ranks, one per GPU, under torch.distributed.run on this node;
    rank 0 prints the line.  Returns the launcher's exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(n),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        raise SystemExit("bench.py: --gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    from quantized_latent_moe_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    if args.steps is None:
        args.steps = wl.steps if wl.layers > 1 else 4096
    if args.warmup is None:
        args.warmup = 4 if wl.layers > 1 else 64
    if args.impl == "reference":
        if int(os.environ.get("WORLD_SIZE", "1")) > 1 and int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference(args)
        return
    if wl.layers > 1:
        run_stack(args)
    else:
        run_elq(args)


if __name__ == "__main__":
    main()
