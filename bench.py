#!/usr/bin/env python
"""Benchmark of the compressed-KV decode step (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch of synthetic input,
for every layer of the workload: append the new token's K and V (encode,
T = 1, at the last cache slot) and run split-K decode attention over the
whole compressed context (query rotation, scores from codes, online softmax,
value accumulation in the rotated domain, combine, inverse rotation), in one
kvq_decode_step launch per layer.  The layers of a step are one CUDA graph.

Headline workload: the Mistral-7B-shaped 32-layer decode step (B 8, 32
query / 8 KV heads, d 128, 32768 cached tokens, layers 0-3 at L 256/256, the
rest at L_K 128 / L_V 64): 14.03 GB of packed codes per step, far larger than
L2, so every step streams its cache from HBM.

  value  decode-attention effective HBM GB/s = algorithmic bytes of the step
         (packed K/V codes + fp16 params read, q read, output written, the
         appended token's fp16 read and codes written) / device time,
         summed over ranks (weak scaling: every rank runs its own replica)
  e2e    the same through kvq_decode_step_host, the C-ABI call with host
         buffers: per layer and step q and the new K/V are copied from pinned
         host memory and the output copied back, on the stream, inside the
         timed region
  roofline / roofline_fp32
         the decode kernel against the measured HBM copy bandwidth, and
         against the FP32 pipe (2 d (G + 1) FMA-pipe operations per cached
         token and KV head)
  decode_tinyllama, decode_llama_layer
         the TinyLlama-shaped 22-layer step (d 64, G 8, 65536 tokens) and the
         Llama-7B-shaped single layer (the latency case), measured the same way
  encode the prefill workload in full: K and V of 32 layers x 16 x 8192
         tokens x 8 KV heads encoded (tokens/s, GB/s), then dequantized back
         to fp16

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "mistral7b_32layers_b8_hq32_hkv8_d128_ctx32768"
TINYLLAMA = "tinyllama_22layers_b4_hq32_hkv4_d64_ctx65536"
LLAMA_LAYER = "llama7b_layer_b1_hq32_hkv8_d128_ctx4096"
PREFILL = "prefill_32layers_b16_t8192_hkv8_d128"
METRIC = "decode-attn effective HBM GB/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0    # B200 HBM3e, nominal (the measured copy is the roofline)
SM_COUNT_B200 = 148
FP32_LANES_PER_SM = 128     # FP32 FMA lanes per SM (4 sub-partitions x 32)
SM_MAX_MHZ = 1965.0


def fp32_peak_tflops(sm_mhz, sm_count=SM_COUNT_B200):
    """FP32 FMA-pipe peak, counting an FMA as two flops."""
    return 2.0 * FP32_LANES_PER_SM * sm_count * sm_mhz * 1e6 / 1e12


def decode_flops_per_token_head(d, G):
    """FP32-pipe work of decode attention per cached token and KV head, in
    flops with every pipe operation counted as an FMA (two flops): each pair
    is scaled by its norm once for K and once for V (2 d multiplies), then
    every one of the G query heads takes d FMAs for its score and d FMAs for
    its value accumulation, 2 d (G + 1) operations in all."""
    return 2 * 2 * d * (G + 1)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="wall time of the bounded oracle sample (cpu_baseline)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="headline workload only (no TinyLlama / Llama-layer steps, no prefill)")
    p.add_argument("--case", default=None,
                   choices=["decode_layer", "step_layer", "encode_layer", "dequant_layer",
                            "shard_layer"],
                   help="run one kernel case only (for profiler captures): the decode (or the "
                        "append + decode step) of --layer of --workload, or the prefill encode "
                        "(or dequant) of 8 batch entries of one layer; --steps launches after 3 "
                        "warm-up launches.  shard_layer: the context-sharded decode of --layer "
                        "with --parts ranks emulated on this GPU (each holding 1/parts of every "
                        "sequence: its split partials, then the merge of all parts)")
    p.add_argument("--parts", type=int, default=2,
                   help="shard_layer case: ranks the context is spread over")
    p.add_argument("--L", type=int, default=None,
                   help="with --case: codebook size for K and V instead of the workload's "
                        "(sizes outside the fast kernels' set select the general kernels)")
    p.add_argument("--layer", type=int, default=0)
    p.add_argument("--tensor", default="k", choices=["k", "v"],
                   help="encode_layer / dequant_layer case: the layer's K (8-bit linear norms) "
                        "or V (4-bit log)")
    return p.parse_args()


# ----------------------------------------------------------------- bytes --

def row_bytes_total(kvq, d, L, mode):
    c = kvq.codec(d, L, mode)
    return sum(kvq.kvq_row_bytes(c, w) for w in range(3))


def step_bytes(kvq, w, out_bytes=2):
    """(bytes per step, bytes per decode launch of each layer)."""
    per_layer = []
    total = 0
    for layer in range(w.layers):
        rk = row_bytes_total(kvq, w.d, w.L_K[layer], w.mode_K)
        rv = row_bytes_total(kvq, w.d, w.L_V[layer], w.mode_V)
        dec = w.B * w.H_kv * w.ctx * (rk + rv) + w.B * w.H_q * w.d * (2 + out_bytes)
        app = w.B * w.H_kv * (2 * w.d * 2 + rk + rv)
        per_layer.append(dec)
        total += dec + app
    return total, per_layer


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profile_traffic(kernel_tag):
    """DRAM bytes per launch from a committed ncu summary, or None if none
    exists or the kernel source changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.txt")
    if not os.path.exists(path):
        return None
    meta = {}
    for line in open(path):
        if ":" in line and not line.startswith(" "):
            k, v = line.split(":", 1)
            meta[k.strip()] = v.strip()
    src = os.path.join(ROOT, "decode_attention_rand_b200", "csrc", meta.get("source", ""))
    if not os.path.exists(src) or "source_sha256" not in meta:
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if h != meta["source_sha256"]:
        return None
    try:
        return float(meta["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- clocks --

REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """SM clock, power and clock-event reasons of this process's GPU, sampled
    every 10 ms through NVML in a thread (nvidia-smi at 100 ms where NVML is
    not importable)."""

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.samples = []  # (time, sm_mhz, sm_max_mhz, reasons tuple)
        self.stop_ev = threading.Event()
        self.thread = None
        self.proc = None

    def start(self):
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByPciBusId(self.bus_id.upper()) if self.bus_id \
                else N.nvmlDeviceGetHandleByIndex(0)
            self.thread = threading.Thread(target=self._nvml, args=(N, h), daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            fields = ("pci.bus_id,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                      "clocks_event_reasons.hw_thermal_slowdown,"
                      "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._smi, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _nvml(self, N, h):
        bits = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap}
        mx = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
        while not self.stop_ev.is_set():
            try:
                sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                r = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.time(), float(sm), float(mx),
                                     tuple(n for n in REASONS if r & bits[n])))
            except Exception:
                pass
            self.stop_ev.wait(0.01)

    def _smi(self):
        for line in self.proc.stdout:
            p = [x.strip() for x in line.split(",")]
            if len(p) < 7:
                continue
            if self.bus_id and not p[0].lower().endswith(self.bus_id[-12:]):
                continue
            try:
                self.samples.append((time.time(), float(p[1]), float(p[2]),
                                     tuple(n for n, v in zip(REASONS, p[3:7])
                                           if v.lower() == "active")))
            except ValueError:
                pass

    def stop(self):
        self.stop_ev.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        sel = [s for s in self.samples if t0 <= s[0] <= t1]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(s[1] for s in sel),
                "sm_max_mhz": max(s[2] for s in sel),
                "reasons": sorted({n for s in sel for n in s[3]}), "samples": len(sel)}


# ------------------------------------------------------------ GPU state --

class DecodeStep:
    """Device-resident caches of a workload and the launch sequence of one
    step (one kvq_decode_step per layer).  Caches smaller than twice the L2
    size are replicated and rotated so that every step reads from HBM."""

    def __init__(self, w, device, l2_bytes):
        import torch
        from decode_attention_rand_b200 import kvq, synth
        self.w, self.kvq, self.torch = w, kvq, torch
        self.device = device
        total, per_layer = step_bytes(kvq, w)
        cache_bytes = sum(per_layer)
        self.nbuf = max(1, math.ceil(2 * l2_bytes / cache_bytes))
        sm = torch.cuda.get_device_properties(device).multi_processor_count
        self.S = kvq.kvq_decode_num_splits(w.B, w.H_kv, w.ctx, sm)
        self.ws = kvq.DecodeWorkspace(w.B, w.H_q, w.d, self.S, device)
        self.ctx = torch.full((w.B,), w.ctx, dtype=torch.int32, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.tau = 1.0 / math.sqrt(w.d)
        self.cap = (w.ctx + 15) // 16 * 16
        self.layers = []
        for layer in range(w.layers):
            sk, sv = synth.layer_signs(w, layer)
            skd = torch.from_numpy(sk).to(device)
            svd = torch.from_numpy(sv).to(device)
            kc = kvq.codec(w.d, w.L_K[layer], w.mode_K)
            vc = kvq.codec(w.d, w.L_V[layer], w.mode_V)
            bufs = []
            for kind, c, s in ((synth.KIND_K, kc, skd), (synth.KIND_V, vc, svd)):
                p = kvq.alloc_plane(c, w.B, w.H_kv, self.cap, device)
                x = synth.kv(w, layer, kind, device=device)
                kvq.encode(c, s, x, p, 0)
                del x
                bufs.append(p)
            planes = [tuple(bufs)]
            for _ in range(1, self.nbuf):
                planes.append(tuple(kvq.Plane(p.codec, p.B, p.H_kv, p.capacity, p.angles.clone(),
                                              p.norms.clone(), p.params.clone()) for p in bufs))
            q0 = synth.queries(w, layer, device=device)
            k0 = synth.kv(w, layer, synth.KIND_K, device=device, T=1, salt=7)
            v0 = synth.kv(w, layer, synth.KIND_V, device=device, T=1, salt=7)
            # the step's inputs (q, new K, new V) in one buffer: one copy per
            # layer and token when they come from the host
            nq, nk = q0.numel(), k0.numel()
            io = torch.empty(nq + 2 * nk, dtype=torch.float16, device=device)
            q, knew, vnew = (io[:nq].view_as(q0), io[nq:nq + nk].view_as(k0),
                             io[nq + nk:].view_as(v0))
            q.copy_(q0)
            knew.copy_(k0)
            vnew.copy_(v0)
            out = torch.empty((w.B, w.H_q, w.d), dtype=torch.float16, device=device)
            L = dict(kc=kc, vc=vc, skd=skd, svd=svd, planes=planes, io=io, q=q, knew=knew,
                     vnew=vnew, out=out, cK=[p[0].c() for p in planes],
                     cV=[p[1].c() for p in planes])
            # append the new K and V at position ctx - 1, then attend: one kernel,
            # or an append launch and the decode (the library decides per codec
            # and launch shape)
            L["calls"] = [kvq.DecodeStepCall(q, knew, vnew, kc, vc, skd, svd, L["cK"][b],
                                             L["cV"][b], self.ctx, w.B, w.H_q, w.H_kv, w.ctx,
                                             self.tau, self.S, self.ws.buf, self.ws.nbytes,
                                             self.err, out, kvq.OUT_FP16)
                          for b in range(self.nbuf)]
            self.layers.append(L)
        torch.cuda.synchronize(device)
        self.calls_per_step = w.layers  # one kvq_decode_step call per layer
        self.bytes_per_step, self.bytes_per_launch = total, per_layer
        self.cache_bytes = cache_bytes * self.nbuf

    def step(self, i, ev=None, stream=None):
        b = i % self.nbuf
        st = stream.cuda_stream if stream is not None else self.torch.cuda.current_stream().cuda_stream
        for li, L in enumerate(self.layers):
            if ev is not None:
                ev[li][0].record()
            L["calls"][b](st)  # kvq_decode_step, arguments marshalled at setup
            if ev is not None:
                ev[li][1].record()

    def release(self):
        self.layers = []
        self.ws = None
        self.torch.cuda.synchronize(self.device)
        self.torch.cuda.empty_cache()


def time_graph(state, K, W, dist_ctx):
    """Device time of exactly K steps replayed from CUDA graphs, plus
    per-launch durations from events captured in a separate graph.

    The timed graphs hold the steps' kernels only: an event node between two
    launches would cut the programmatic dependency that lets each decode's
    setup overlap the previous launch."""
    import torch
    stream = torch.cuda.Stream()
    for i in range(W):
        state.step(i)
    torch.cuda.synchronize()
    per_graph = max(1, math.ceil(256 / max(1, state.calls_per_step)))
    unit = max(1, min(K, state.nbuf * max(1, math.ceil(per_graph / state.nbuf))))
    n_full, rem = divmod(K, unit)
    g_unit = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_unit, stream=stream):
        for i in range(unit):
            state.step(i, stream=torch.cuda.current_stream())
    g_rem = None
    if rem:
        g_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rem, stream=stream):
            for i in range(rem):
                state.step(n_full * unit + i, stream=torch.cuda.current_stream())
    # external events become event-record nodes of the graph, so each decode
    # launch is timed inside the replay
    n_ev = max(1, min(unit, 4 if state.calls_per_step > 1 else 16))
    evs = [[[torch.cuda.Event(enable_timing=True, external=True),
             torch.cuda.Event(enable_timing=True, external=True)]
            for _ in state.layers] for _ in range(n_ev)]
    g_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ev, stream=stream):
        for i in range(n_ev):
            state.step(i, evs[i], stream=torch.cuda.current_stream())
    # one untimed replay uploads the graphs (extra warm-up)
    g_unit.replay()
    if g_rem:
        g_rem.replay()
    g_ev.replay()
    torch.cuda.synchronize()
    barrier(dist_ctx)
    t_wall0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream()
    start.record(cur)
    for _ in range(n_full):
        g_unit.replay()
    if g_rem:
        g_rem.replay()
    end.record(cur)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(dist_ctx)
    ms = start.elapsed_time(end)
    per_layer = [[] for _ in state.layers]
    for _ in range(2):
        g_ev.replay()
        torch.cuda.synchronize()
        for i in range(n_ev):
            for li in range(len(state.layers)):
                per_layer[li].append(evs[i][li][0].elapsed_time(evs[i][li][1]))
    del g_unit, g_rem, g_ev
    return ms, [statistics.fmean(x) for x in per_layer], (t_wall0, t_wall1)


def kernel_launches_per_step(state):
    """Kernels of one step, counted from a CUDA graph of it (kernel nodes of
    the captured, never replayed, graph)."""
    import torch
    from cuda.bindings import runtime as rt
    g = torch.cuda.CUDAGraph(keep_graph=True)
    stream = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=stream):
        state.step(0, stream=torch.cuda.current_stream())
    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    count = sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)
    del g
    return count


def time_e2e(state, K, dist_ctx):
    """The step through the C-ABI call with host buffers: per layer and step,
    kvq_decode_step_host copies q and the new K/V from pinned host memory (one
    buffer per layer) to the GPU and the attention output back, on the
    stream, inside the timed region."""
    import torch
    kvq, w = state.kvq, state.w
    hin = [L["io"].cpu().pin_memory() for L in state.layers]  # q | new K | new V
    ho = [torch.empty_like(L["out"], device="cpu").pin_memory() for L in state.layers]
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in ho)
    cur = torch.cuda.current_stream()
    calls = [[kvq.DecodeStepHostCall(hin[li], L["io"], ho[li], L["out"], L["kc"], L["vc"],
                                     L["skd"], L["svd"], L["cK"][b], L["cV"][b], state.ctx, w.B,
                                     w.H_q, w.H_kv, w.ctx, state.tau, state.S, state.ws.buf,
                                     state.ws.nbytes, state.err, kvq.OUT_FP16)
              for b in range(state.nbuf)] for li, L in enumerate(state.layers)]
    st = cur.cuda_stream

    def one(i):
        b = i % state.nbuf
        for per_layer in calls:
            per_layer[b](st)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    n = max(1, min(K, 4000 // max(1, w.layers)))
    barrier(dist_ctx)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(cur)
    for i in range(n):
        one(i)
    end.record(cur)
    torch.cuda.synchronize()
    barrier(dist_ctx)
    return start.elapsed_time(end), n, h2d, d2h


def decode_report(state, ms, K, per_launch_ms, hbm_peak, peak_kind, sm_mhz, sm_count,
                  traffic=None):
    """Throughput and roofline figures of a timed decode workload."""
    w = state.w
    calls = K * state.calls_per_step
    # per layer: the decode kernel, with the append fused in or hidden behind
    # its first tiles; the roofline takes the whole layer's time (conservative)
    us_launch = ms / calls * 1e3
    bytes_launch = statistics.fmean(state.bytes_per_launch)
    gbs = bytes_launch / (us_launch / 1e6) / 1e9
    flops = w.B * w.H_kv * w.ctx * decode_flops_per_token_head(w.d, w.G)
    fp_peak = fp32_peak_tflops(sm_mhz, sm_count)
    tfs = flops / (us_launch / 1e6) / 1e12
    early = [i for i in range(w.layers) if (w.L_K[i], w.L_V[i]) != (w.L_K[-1], w.L_V[-1])]
    late = [i for i in range(w.layers) if i not in early]
    by_kind = {}
    for name, idx in (("early_boost_layers", early), ("other_layers", late)):
        if idx:
            t = statistics.fmean(per_launch_ms[i] for i in idx)
            b = statistics.fmean(state.bytes_per_launch[i] for i in idx)
            by_kind[name] = {"layers": len(idx), "L_K": w.L_K[idx[0]], "L_V": w.L_V[idx[0]],
                             "us_per_launch_event_bracketed": t * 1e3,
                             "gb_per_s": b / (t / 1e3) / 1e9,
                             "hbm_frac": b / (t / 1e3) / 1e9 / hbm_peak}
    return {
        "gb_per_s": state.bytes_per_step * K / (ms / 1e3) / 1e9,
        "ms_per_step": ms / K,
        "per_token_latency_ms": ms / K,
        "bytes_per_step": state.bytes_per_step,
        "num_splits": state.S,
        "roofline": {
            "kernel": "decode_kernel (split-K decode attention with the split combine; "
                      "kvq_decode_step runs it per layer with the new token's append fused in, "
                      "or after an append_kernel launch it hides; time per layer)",
            "bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
            "frac": gbs / hbm_peak, "peak_kind": f"{peak_kind} copy bandwidth",
            "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
            "traffic": traffic, "bytes_per_launch": bytes_launch, "us_per_launch": us_launch,
        },
        "roofline_fp32": {
            "achieved": tfs, "peak": fp_peak, "unit": "TFLOP/s", "frac": tfs / fp_peak,
            "flops_per_launch": flops,
            "peak_kind": f"FP32 FMA pipe, derived: {FP32_LANES_PER_SM} lanes/SM x {sm_count} "
                         f"SMs x 2 flop x {sm_mhz:.0f} MHz (sampled)",
        },
        "launch_kinds": by_kind,
    }


def time_prefill(device, hbm_peak, reps=3):
    """The prefill workload in full: kvq_encode of K and V of all 32 layers
    (16 x 8192 tokens x 8 KV heads each), then kvq_dequant of all of them;
    CUDA events around whole passes."""
    import torch
    from decode_attention_rand_b200 import kvq, synth
    w = synth.WORKLOADS[PREFILL]
    items = []
    for layer in range(w.layers):
        sk, sv = synth.layer_signs(w, layer)
        for kind, L, mode, s in ((synth.KIND_K, w.L_K[layer], w.mode_K, sk),
                                 (synth.KIND_V, w.L_V[layer], w.mode_V, sv)):
            c = kvq.codec(w.d, L, mode)
            p = kvq.alloc_plane(c, w.B, w.H_kv, w.ctx, device)
            x = synth.kv(w, layer, kind, device=device)
            items.append((c, p, x, torch.from_numpy(s).to(device)))
    # one fp16 destination per tensor kind, reused by every layer's dequant
    ys = [torch.empty_like(items[0][2]), torch.empty_like(items[1][2])]
    n_vec = len(items) * w.B * w.H_kv * w.ctx
    rows = sum(w.B * w.H_kv * w.ctx * row_bytes_total(kvq, w.d, c.L, c.norm_mode)
               for c, p, x, s in items)
    fp16 = sum(x.numel() * 2 for c, p, x, s in items)
    for c, p, x, s in items:  # warm-up pass
        kvq.encode(c, s, x, p, 0)
    for i, (c, p, x, s) in enumerate(items):
        kvq.dequant(c, s, p, w.ctx, out=ys[i % 2])
    torch.cuda.synchronize()
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record()
    for _ in range(reps):
        for c, p, x, s in items:
            kvq.encode(c, s, x, p, 0)
    e1.record()
    for _ in range(reps):
        for i, (c, p, x, s) in enumerate(items):
            kvq.dequant(c, s, p, w.ctx, out=ys[i % 2])
    e2.record()
    torch.cuda.synchronize()
    enc_s = e0.elapsed_time(e1) / 1e3 / reps
    dq_s = e1.elapsed_time(e2) / 1e3 / reps
    tokens = w.layers * w.B * w.ctx
    out = {
        "workload": f"{w.name}: K and V of {w.layers} layers, {n_vec} head vectors per pass",
        "tokens_per_s": tokens / enc_s,
        "head_vectors_per_s": n_vec / enc_s,
        "encode_gb_per_s": (fp16 + rows) / enc_s / 1e9,
        "encode_frac": (fp16 + rows) / enc_s / 1e9 / hbm_peak,
        "encode_frac_of_nominal_8tbs": (fp16 + rows) / enc_s / 1e9 / NOMINAL_HBM_GBS,
        "dequant_gb_per_s": (fp16 + rows) / dq_s / 1e9,
        "dequant_frac": (fp16 + rows) / dq_s / 1e9 / hbm_peak,
        "dequant_frac_of_nominal_8tbs": (fp16 + rows) / dq_s / 1e9 / NOMINAL_HBM_GBS,
        "ms_per_pass_encode": enc_s * 1e3,
        "ms_per_pass_dequant": dq_s * 1e3,
        "bytes_per_pass": fp16 + rows,
        "launches_per_pass": len(items),
    }
    del items, ys
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_case(args):
    """One kernel case on cuda:0, for profiler captures of a single launch."""
    import torch
    from decode_attention_rand_b200 import build as kbuild
    from decode_attention_rand_b200 import kvq, synth
    kbuild.build()
    kvq.lib()
    device = torch.device("cuda", 0)
    steps = max(1, min(args.steps, 20))
    if args.case in ("decode_layer", "step_layer"):
        w = synth.WORKLOADS[args.workload]
        layer = args.layer
        sk, sv = synth.layer_signs(w, layer)
        skd, svd = torch.from_numpy(sk).to(device), torch.from_numpy(sv).to(device)
        kc = kvq.codec(w.d, args.L or w.L_K[layer], w.mode_K)
        vc = kvq.codec(w.d, args.L or w.L_V[layer], w.mode_V)
        planes = []
        for kind, c, sg in ((synth.KIND_K, kc, skd), (synth.KIND_V, vc, svd)):
            p = kvq.alloc_plane(c, w.B, w.H_kv, w.ctx, device)
            x = synth.kv(w, layer, kind, device=device)
            kvq.encode(c, sg, x, p, 0)
            del x
            planes.append(p)
        q = synth.queries(w, layer, device=device)
        ctx = torch.full((w.B,), w.ctx, dtype=torch.int32, device=device)
        out = torch.empty((w.B, w.H_q, w.d), dtype=torch.float16, device=device)
        sm = torch.cuda.get_device_properties(device).multi_processor_count
        S = kvq.kvq_decode_num_splits(w.B, w.H_kv, w.ctx, sm)
        ws = kvq.DecodeWorkspace(w.B, w.H_q, w.d, S, device)

        if args.case == "decode_layer":
            def run():
                kvq.decode_attn(q, kc, vc, skd, svd, planes[0], planes[1], ctx, w.ctx, None,
                                num_splits=S, workspace=ws, out=out, out_dtype=kvq.OUT_FP16)
            what = f"decode {w.name} layer {layer}, {S} splits"
        else:
            # every launch appends the same new token at position ctx - 1
            kn = synth.kv(w, layer, synth.KIND_K, device=device, T=1, salt=7)[:, :, 0].contiguous()
            vn = synth.kv(w, layer, synth.KIND_V, device=device, T=1, salt=7)[:, :, 0].contiguous()

            def run():
                kvq.decode_step(q, kn, vn, kc, vc, skd, svd, planes[0], planes[1], ctx, w.ctx,
                                None, num_splits=S, workspace=ws, out=out,
                                out_dtype=kvq.OUT_FP16)
            what = f"append + decode step {w.name} layer {layer}, {S} splits"
        if args.L:
            what += f", L_K = L_V = {args.L}"
    elif args.case == "shard_layer":
        # context-sharded decode with the ranks emulated one after another on
        # this GPU: part r holds tokens [r ctx / N, (r + 1) ctx / N) of every
        # sequence in planes of its own and writes its split partials into
        # row r of the stacked buffer the merge reads
        w = synth.WORKLOADS[args.workload]
        layer, N = args.layer, max(1, args.parts)
        sk, sv = synth.layer_signs(w, layer)
        skd, svd = torch.from_numpy(sk).to(device), torch.from_numpy(sv).to(device)
        kc = kvq.codec(w.d, args.L or w.L_K[layer], w.mode_K)
        vc = kvq.codec(w.d, args.L or w.L_V[layer], w.mode_V)
        bounds = [(r * w.ctx // N, (r + 1) * w.ctx // N) for r in range(N)]
        planes = []
        for lo, hi in bounds:
            cap = max(16, (hi - lo + 15) // 16 * 16)
            pr = []
            for kind, c, sg in ((synth.KIND_K, kc, skd), (synth.KIND_V, vc, svd)):
                pl = kvq.alloc_plane(c, w.B, w.H_kv, cap, device)
                x = synth.kv(w, layer, kind, device=device)[:, :, lo:hi].contiguous()
                kvq.encode(c, sg, x, pl, 0)
                del x
                pr.append(pl)
            planes.append(pr)
        torch.cuda.empty_cache()
        q = synth.queries(w, layer, device=device)
        out = torch.empty((w.B, w.H_q, w.d), dtype=torch.float16, device=device)
        sm = torch.cuda.get_device_properties(device).multi_processor_count
        max_part = max(hi - lo for lo, hi in bounds)
        S = kvq.kvq_decode_num_splits(w.B, w.H_kv, max_part, sm)
        nbytes = kvq.kvq_decode_workspace_bytes(w.B, w.H_q, w.d, S)
        parts = torch.zeros((N, nbytes), dtype=torch.uint8, device=device)
        ctxs = [torch.full((w.B,), hi - lo, dtype=torch.int32, device=device) for lo, hi in bounds]
        tau = 1.0 / math.sqrt(w.d)

        def merge():
            kvq.kvq_decode_merge_partials(parts, N, w.B, w.H_q, w.d, S, svd, out, kvq.OUT_FP16)

        def run():
            for r, (lo, hi) in enumerate(bounds):
                kvq.kvq_decode_attn_partials(q, kc, vc, skd, svd, planes[r][0].c(),
                                             planes[r][1].c(), ctxs[r], w.B, w.H_q, w.H_kv,
                                             hi - lo, tau, S, parts[r], nbytes)
            merge()
        what = (f"context-sharded decode {w.name} layer {layer}: {N} parts of {max_part} tokens, "
                f"{S} splits each, then the merge")
    else:
        w = synth.WORKLOADS[PREFILL]
        sk, sv = synth.layer_signs(w, 0)
        isk = args.tensor == "k"
        c = (kvq.codec(w.d, args.L or w.L_K[0], w.mode_K) if isk
             else kvq.codec(w.d, args.L or w.L_V[0], w.mode_V))
        nb = 8
        p = kvq.alloc_plane(c, nb, w.H_kv, w.ctx, device)
        x = synth.kv(w, 0, synth.KIND_K if isk else synth.KIND_V, device=device, b_range=(0, nb))
        skd = torch.from_numpy(sk if isk else sv).to(device)

        if args.case == "encode_layer":
            def run():
                kvq.encode(c, skd, x, p, 0)
            what = f"encode {w.name} layer 0 {'K' if isk else 'V'}, batch entries 0..{nb - 1}"
        else:
            kvq.encode(c, skd, x, p, 0)
            y = torch.empty_like(x)

            def run():
                kvq.dequant(c, skd, p, w.ctx, 0, out=y)
            what = f"dequant {w.name} layer 0 {'K' if isk else 'V'}, batch entries 0..{nb - 1}"
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    res = {"case": what, "us_per_launch": e0.elapsed_time(e1) * 1e3 / steps}
    if args.case == "shard_layer":
        # the merge alone, replayed from a CUDA graph (a launch of a few
        # microseconds would otherwise be timed at the host's call rate), and
        # the bytes it reads (every part's partials) and writes
        graph, side = torch.cuda.CUDAGraph(), torch.cuda.Stream()
        with torch.cuda.graph(graph, stream=side):
            for _ in range(steps):
                merge()
        graph.replay()
        torch.cuda.synchronize()
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        res["merge_us"] = e0.elapsed_time(e1) * 1e3 / steps
        del graph
        res["merge_bytes"] = N * nbytes + out.numel() * out.element_size()
    print(json.dumps(res), flush=True)
    return 0


# --------------------------------------------------------------- oracle --

class OracleSteps:
    """The fp64 oracle on the host, on bounded samples of the step.

    One oracle step is one (layer, batch, KV-head) unit of the workload:
    append the new K and V token (encode), dequantize the unit's cached K and
    V codes over a context slice and attend its G query heads (textbook
    attention).  The slice is the whole context unless a per-step time
    budget asks for less.  Inputs are the synthetic tensors, encoded by the
    oracle itself before timing starts."""

    def __init__(self, w):
        import numpy as np
        import oracle as O
        self.w, self.O, self.np = w, O, np
        self.threads = O.default_threads()
        self.units = [(l, b, h) for l in range(w.layers) for b in range(w.B) for h in range(w.H_kv)]
        # row sizes from the oracle's own layout: this arm loads nothing but oracle/
        self.rows = {l: (sum(O.row_bytes(w.d, w.L_K[l], w.mode_K, k) for k in range(3)),
                         sum(O.row_bytes(w.d, w.L_V[l], w.mode_V, k) for k in range(3)))
                     for l in range(w.layers)}
        self.prepared = {}
        self.slice_len = w.ctx

    def _prepare(self, unit, slice_len):
        from decode_attention_rand_b200 import synth
        O, w, np = self.O, self.w, self.np
        l, b, h = unit
        sk, sv = synth.layer_signs(w, l)
        K = synth.kv(w, l, synth.KIND_K, T=slice_len, b_range=(b, b + 1))[0, h].numpy()
        V = synth.kv(w, l, synth.KIND_V, T=slice_len, b_range=(b, b + 1))[0, h].numpy()
        q = synth.queries(w, l)[b, h * w.G:(h + 1) * w.G].numpy().astype(np.float64)
        kc = O.encode(K, sk, w.L_K[l], w.mode_K, threads=self.threads)
        vc = O.encode(V, sv, w.L_V[l], w.mode_V, threads=self.threads)
        return (sk, sv, np.ascontiguousarray(K[-1:]), np.ascontiguousarray(V[-1:]), q, kc, vc)

    def _one(self, unit, data):
        O, w = self.O, self.w
        sk, sv, kn, vn, q, kc, vc = data
        l = unit[0]
        t0 = time.perf_counter()
        O.encode(kn, sk, w.L_K[l], w.mode_K, threads=1)
        O.encode(vn, sv, w.L_V[l], w.mode_V, threads=1)
        kh = O.dequant(kc, sk, threads=self.threads)
        vh = O.dequant(vc, sv, threads=self.threads)
        O.attend(q, kh, vh, 1.0 / math.sqrt(w.d))
        dt = time.perf_counter() - t0
        rk, rv = self.rows[l]
        nbytes = kc.n * (rk + rv) + w.G * w.d * 4 + 2 * w.d * 2 + rk + rv
        return nbytes, dt

    def calibrate(self, per_step_s):
        """Pick the context slice so that one step takes about per_step_s
        (timed first on a 2048-token slice, then scaled)."""
        probe = min(self.w.ctx, 2048)
        data = self._prepare(self.units[0], probe)
        _, t_probe = self._one(self.units[0], data)
        t_full = t_probe * self.w.ctx / probe
        if per_step_s is not None and t_full > per_step_s:
            sl = int(self.w.ctx * per_step_s / t_full) // 16 * 16
            self.slice_len = max(16, min(self.w.ctx, sl))
        self.prepared = {}
        return t_full

    def run(self, n_steps):
        rng = self.np.random.default_rng(0)
        picks = [self.units[0]] + [self.units[int(rng.integers(0, len(self.units)))]
                                   for _ in range(3)]
        for u in picks:
            if u not in self.prepared:
                self.prepared[u] = self._prepare(u, self.slice_len)
        done, secs = 0, 0.0
        for i in range(n_steps):
            u = picks[i % len(picks)]
            b, dt = self._one(u, self.prepared[u])
            done += b
            secs += dt
        return done, secs

    def describe(self, n_steps):
        w = self.w
        return (f"{n_steps} steps of one (layer, batch, KV-head) unit each with a "
                f"{self.slice_len}-token context slice (the full step has {len(self.units)} units "
                f"x {w.ctx} tokens), fp64 oracle, {self.threads} threads")


def cpu_baseline(w, seconds):
    ors = OracleSteps(w)
    ors.calibrate(seconds / 4)
    t0 = time.perf_counter()
    done, secs = ors.run(1)
    n = max(1, int(seconds / max(time.perf_counter() - t0, 1e-6)))
    done, secs = ors.run(n)
    return {"value": done / secs / 1e9, "unit": "GB/s", "cores": ors.threads, "kind": "oracle",
            "sample": ors.describe(n)}


# ------------------------------------------------------------- ranks ----

def init_dist(gpus):
    """One process per GPU from the torchrun environment: NCCL over the
    GPUs, or gloo on the host cores where there is no GPU (the CPU tests of
    the multi-rank path)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return dict(world=world, rank=rank, local=local, dist=dist, backend=backend)
    return dict(world=1, rank=0, local=0, dist=None, backend=None)


def barrier(ctx):
    if ctx["dist"] is not None:
        ctx["dist"].barrier()


def max_over_ranks(ctx, value):
    if ctx["dist"] is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64,
                     device="cuda" if ctx["backend"] == "nccl" else "cpu")
    ctx["dist"].all_reduce(t, op=ctx["dist"].ReduceOp.MAX)
    return float(t.item())


def workload_config(w) -> dict:
    """The workload part of the JSON line's config, shared by both arms."""
    return {"workload": w.name, "layers": w.layers, "batch": w.B, "H_q": w.H_q, "H_kv": w.H_kv,
            "head_dim": w.d, "ctx": w.ctx, "L_K": sorted(set(w.L_K)), "L_V": sorted(set(w.L_V)),
            "norms": "K lin8, V log4"}


def run_reference(args, w):
    """The reference arm: the fp64 oracle on the host cores, K timed steps of
    a bounded sample each, the whole run kept to a few minutes."""
    ors = OracleSteps(w)
    budget = max(5.0, min(150.0, 2.0 * (args.steps + args.warmup)))  # seconds, whole run
    ors.calibrate(budget / max(1, args.steps + args.warmup))
    ors.run(args.warmup)
    done, secs = ors.run(args.steps)
    gbs = done / secs / 1e9
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": ors.threads, "kind": "oracle",
                         "sample": ors.describe(args.steps)},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def measure(name, device, l2, K, W, ctx, hbm_peak, peak_kind, sm_count, sampler, e2e=False,
            traffic=None):
    """Build one decode workload, time K graphed steps (and the e2e path),
    and return its report plus the timed window and the state's launch count."""
    from decode_attention_rand_b200 import synth
    w = synth.WORKLOADS[name]
    state = DecodeStep(w, device, l2)
    ms, per_launch, (tw0, tw1) = time_graph(state, K, W, ctx)
    ms = max_over_ranks(ctx, ms)
    clocks = sampler.summary(tw0, tw1)
    rep = decode_report(state, ms, K, per_launch, hbm_peak, peak_kind,
                        clocks.get("sm_mhz") or SM_MAX_MHZ, sm_count, traffic)
    rep["workload"] = w.name
    rep["clocks"] = clocks
    rep["l2"] = (f"inputs larger than L2: {state.cache_bytes / 1e9:.2f} GB of codes read per "
                 f"cycle of {state.nbuf} step(s) (L2 {l2 / 2**20:.0f} MiB)")
    if e2e:
        e_ms, e_n, h2d, d2h = time_e2e(state, K, ctx)
        e_ms = max_over_ranks(ctx, e_ms)
        rep["e2e"] = {"value": ctx["world"] * state.bytes_per_step * e_n / (e_ms / 1e3) / 1e9,
                      "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "steps": e_n, "transfer": "cudaMemcpyAsync in and out on the stream per call"}
    err = int(state.err.item())
    launches = kernel_launches_per_step(state) * K
    state.release()
    if err != 0:
        raise RuntimeError(f"{name}: device error word {err}")
    return rep, launches


def main():
    args = parse()
    if args.case:
        return run_case(args)
    from decode_attention_rand_b200 import synth
    w = synth.WORKLOADS[args.workload]
    ctx = init_dist(args.gpus)
    if args.impl == "reference":
        # rank 0 alone times the oracle; the other ranks leave without work
        if ctx["rank"] == 0:
            run_reference(args, w)
        if ctx["dist"] is not None:
            ctx["dist"].destroy_process_group()
        return 0
    import torch
    from decode_attention_rand_b200 import build as kbuild
    from decode_attention_rand_b200 import kvq
    if ctx["rank"] == 0:
        kbuild.build()
    barrier(ctx)
    kvq.lib()
    device = torch.device("cuda", ctx["local"])
    torch.cuda.set_device(device)
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    bus = None
    try:
        bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    except Exception:
        pass
    hbm_peak, peak_kind = peaks()
    sampler = ClockSampler(bus)
    sampler.start()
    sm_count = props.multi_processor_count
    K, W = args.steps, max(args.warmup, 0)

    head, launches = measure(w.name, device, l2, K, W, ctx, hbm_peak, peak_kind, sm_count,
                             sampler, e2e=True, traffic=headline_traffic(w.name))
    extra = {}
    if not args.no_extra:
        for key, name in (("decode_tinyllama", TINYLLAMA), ("decode_llama_layer", LLAMA_LAYER)):
            if name != w.name:
                extra[key], _ = measure(name, device, l2, K, W, ctx, hbm_peak, peak_kind,
                                        sm_count, sampler)
        extra["encode"] = time_prefill(device, hbm_peak)
    sampler.stop()

    if ctx["rank"] != 0:
        if ctx["dist"] is not None:
            ctx["dist"].destroy_process_group()
        return 0
    world = ctx["world"]
    line = {
        "metric": METRIC, "value": world * head["gb_per_s"], "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            **workload_config(w), "num_splits": head["num_splits"], "out": "fp16",
            "l2": head["l2"],
            "timing": "CUDA graph replay of whole steps, CUDA events, max over ranks",
            "bytes_per_step": head["bytes_per_step"],
        },
        "roofline": head["roofline"],
        "roofline_fp32": head["roofline_fp32"],
        "launch_kinds": head["launch_kinds"],
        "per_token_latency_ms": {w.name: head["per_token_latency_ms"]},
        "e2e": head["e2e"],
        "gpu_launches": launches,
        "clocks": head["clocks"],
    }
    for key, rep in extra.items():
        line[key] = rep
        if "per_token_latency_ms" in rep:
            line["per_token_latency_ms"][rep["workload"]] = rep["per_token_latency_ms"]
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)
    if ctx["dist"] is not None:
        ctx["dist"].destroy_process_group()
    return 0


def headline_traffic(name):
    """DRAM bytes per decode launch of a workload, from the committed ncu
    summaries of its layer kinds (weighted by how many layers each kind has),
    or None when a summary is missing or stale."""
    from decode_attention_rand_b200 import synth
    w = synth.WORKLOADS[name]
    if name == DEFAULT_WORKLOAD:
        t0 = profile_traffic("decode_kernel_mistral7b_layer0")
        t4 = profile_traffic("decode_kernel_mistral7b_layer4")
        if t0 is None or t4 is None:
            return None
        n_early = sum(1 for i in range(w.layers) if w.L_K[i] == w.L_K[0])
        return (n_early * t0 + (w.layers - n_early) * t4) / w.layers
    return None


if __name__ == "__main__":
    sys.exit(main())
