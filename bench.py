#!/usr/bin/env python
"""Benchmark of the compressed-KV decode step (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch of synthetic input,
for every layer of the workload: append the new token's K and V (encode,
T = 1, at the last cache slot) and run split-K decode attention over the
whole compressed context (query rotation, scores from codes, online softmax,
value accumulation in the rotated domain, combine, inverse rotation), in one
kvq_decode_step launch per layer.

  value  decode-attention effective HBM GB/s = algorithmic bytes of the step
         (packed K/V codes + fp16 params read, q read, output written, the
         appended token's fp16 read and codes written) / device time,
         summed over ranks (weak scaling: every rank runs its own replica)
  e2e    the same through kvq_decode_step_host, the C-ABI call with host
         buffers: per layer and step q and the new K/V are copied from pinned
         host memory and the output copied back, on the stream, inside the
         timed region (e2e_zero_copy: the same call letting the kernel read
         and write the pinned host memory itself, without copies)
  encode prefill encode throughput on one layer of the prefill workload
         (tokens/s) and dequant GB/s, reported alongside

Default workload: the Llama-7B-shaped single-layer decode (B 1, 32 query /
8 KV heads, d 128, 4096 cached tokens, L_K 128, L_V 64).  Its caches are
rotated over enough copies to exceed twice the L2 size between reuses.

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

DEFAULT_WORKLOAD = "llama7b_layer_b1_hq32_hkv8_d128_ctx4096"
METRIC = "decode-attn effective HBM GB/s"
FALLBACK_HBM_GBS = 6650.0
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
    its value accumulation, 2 d (G + 1) operations in all.  A multiply fills
    an FMA lane slot, so this is the work that meets the FMA-pipe peak."""
    return 2 * 2 * d * (G + 1)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="wall time of the bounded oracle sample (cpu_baseline)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-encode", action="store_true")
    p.add_argument("--case", default=None, choices=["decode_layer", "encode_layer", "dequant_layer"],
                   help="run one kernel case only (for profiler captures): the decode of "
                        "--layer of --workload, or the prefill encode (or dequant) of 8 batch "
                        "entries of one layer; --steps launches after 3 warm-up launches")
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

class ClockSampler:
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            if self.bus_id and not parts[0].lower().endswith(self.bus_id[-12:]):
                continue
            self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        sel = [p for (t, p) in self.samples if t0 <= t <= t1] or [p for _, p in self.samples]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in sel if num(p[1]) is not None]
        mx = [num(p[2]) for p in sel if num(p[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for p in sel for n, v in zip(names, p[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(sel)}


# ------------------------------------------------------------ GPU state --

class DecodeStep:
    """Device-resident caches of a workload and the launch sequence of one step."""

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
            # one kernel: append the new K and V at position ctx - 1, then attend
            L["calls"] = [kvq.DecodeStepCall(q, knew, vnew, kc, vc, skd, svd, L["cK"][b],
                                             L["cV"][b], self.ctx, w.B, w.H_q, w.H_kv, w.ctx,
                                             self.tau, self.S, self.ws.buf, self.ws.nbytes,
                                             self.err, out, kvq.OUT_FP16)
                          for b in range(self.nbuf)]
            self.layers.append(L)
        torch.cuda.synchronize(device)
        self.kernels_per_step = w.layers  # one fused append + decode launch per layer

    def step(self, i, ev=None, stream=None):
        kvq, w = self.kvq, self.w
        b = i % self.nbuf
        st = stream.cuda_stream if stream is not None else self.torch.cuda.current_stream().cuda_stream
        for li, L in enumerate(self.layers):
            if ev is not None:
                ev[li][0].record()
            L["calls"][b](st)  # kvq_decode_step, arguments marshalled at setup
            if ev is not None:
                ev[li][1].record()


def time_graph(state, K, W, dist_ctx):
    """Device time of exactly K steps replayed from CUDA graphs, plus the
    average decode-launch duration from events captured in a separate graph.

    The timed graphs hold the steps' kernels only: an event node between the
    append and the decode would cut the programmatic dependency that lets the
    decode's setup overlap the append."""
    import torch
    stream = torch.cuda.Stream()
    for i in range(W):
        state.step(i)
    torch.cuda.synchronize()
    unit = max(1, min(K, state.nbuf * max(1, math.ceil(64 / state.nbuf))))
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
    n_ev = min(unit, 16)
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
    dec_ms = []
    for _ in range(4):
        g_ev.replay()
        torch.cuda.synchronize()
        dec_ms += [evs[i][li][0].elapsed_time(evs[i][li][1]) for i in range(n_ev)
                   for li in range(len(state.layers))]
    return ms, statistics.fmean(dec_ms), (t_wall0, t_wall1)


def time_e2e(state, K, dist_ctx, staged=False):
    """The step through the C-ABI call with host buffers: per layer and step,
    kvq_decode_step_host moves q and the new K/V from pinned memory (one
    buffer per layer) to the GPU and the attention output back: staged, by a
    copy in and a copy out on the stream; otherwise by the kernel's own
    loads and stores of the page-locked host memory."""
    import torch
    kvq, w = state.kvq, state.w
    hin = [L["io"].cpu().pin_memory() for L in state.layers]  # q | new K | new V
    ho = [torch.empty_like(L["out"], device="cpu").pin_memory() for L in state.layers]
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = sum(t.numel() * t.element_size() for t in ho)
    cur = torch.cuda.current_stream()
    # staged: device staging buffers, a copy in and a copy out on the stream
    # per call; otherwise the kernel reads the inputs from, and writes the
    # output to, the page-locked host buffers (transfers inside the launch)
    calls = [[kvq.DecodeStepHostCall(hin[li], L["io"] if staged else None, ho[li],
                                     L["out"] if staged else None, L["kc"], L["vc"],
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
    n = max(1, min(K, 2000 // max(1, w.layers)))
    barrier(dist_ctx)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(cur)
    for i in range(n):
        one(i)
    end.record(cur)
    torch.cuda.synchronize()
    barrier(dist_ctx)
    return start.elapsed_time(end), n, h2d, d2h


def time_encode(device, hbm_peak):
    """Prefill encode of one layer (K and V) and its dequant, device time."""
    import torch
    from decode_attention_rand_b200 import kvq, synth
    w = synth.WORKLOADS["prefill_32layers_b16_t8192_hkv8_d128"]
    sk, sv = synth.layer_signs(w, 0)
    items = []
    for kind, L, mode, s in ((synth.KIND_K, 128, 0, sk), (synth.KIND_V, 64, 1, sv)):
        c = kvq.codec(w.d, L, mode)
        p = kvq.alloc_plane(c, w.B, w.H_kv, w.ctx, device)
        x = synth.kv(w, 0, kind, device=device)
        y = torch.empty_like(x)
        items.append((c, p, x, y, torch.from_numpy(s).to(device)))
    n_vec = 2 * w.B * w.H_kv * w.ctx
    enc_bytes = sum(x.numel() * 2 + w.B * w.H_kv * w.ctx * row_bytes_total(kvq, w.d, c.L, c.norm_mode)
                    for c, p, x, y, s in items)
    reps = 20
    for c, p, x, y, s in items:
        kvq.encode(c, s, x, p, 0)
        kvq.dequant(c, s, p, w.ctx, out=y)
    torch.cuda.synchronize()
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record()
    for _ in range(reps):
        for c, p, x, y, s in items:
            kvq.encode(c, s, x, p, 0)
    e1.record()
    for _ in range(reps):
        for c, p, x, y, s in items:
            kvq.dequant(c, s, p, w.ctx, out=y)
    e2.record()
    torch.cuda.synchronize()
    enc_s = e0.elapsed_time(e1) / 1e3 / reps
    dq_s = e1.elapsed_time(e2) / 1e3 / reps
    tokens = w.B * w.ctx
    return {
        "workload": f"{w.name} (one layer: K and V, {n_vec} head vectors)",
        "tokens_per_s": tokens / enc_s,
        "head_vectors_per_s": n_vec / enc_s,
        "encode_gb_per_s": enc_bytes / enc_s / 1e9,
        "encode_frac": enc_bytes / enc_s / 1e9 / hbm_peak,
        "dequant_gb_per_s": enc_bytes / dq_s / 1e9,
        "dequant_frac": enc_bytes / dq_s / 1e9 / hbm_peak,
        "ms_per_layer_encode": enc_s * 1e3,
        "ms_per_layer_dequant": dq_s * 1e3,
    }


def time_decode_layers(device, hbm_peak, sm_mhz):
    """Decode-kernel time on single layers of the large decode workloads
    (eager launches, CUDA events; each layer's codes exceed L2)."""
    import torch
    from decode_attention_rand_b200 import kvq, synth
    sm = torch.cuda.get_device_properties(device).multi_processor_count
    fp_peak = fp32_peak_tflops(sm_mhz, sm)
    res = []
    for name, layer in (("mistral7b_32layers_b8_hq32_hkv8_d128_ctx32768", 4),
                        ("mistral7b_32layers_b8_hq32_hkv8_d128_ctx32768", 0),
                        ("tinyllama_22layers_b4_hq32_hkv4_d64_ctx65536", 2)):
        w = synth.WORKLOADS[name]
        sk, sv = synth.layer_signs(w, layer)
        skd, svd = torch.from_numpy(sk).to(device), torch.from_numpy(sv).to(device)
        kc = kvq.codec(w.d, w.L_K[layer], w.mode_K)
        vc = kvq.codec(w.d, w.L_V[layer], w.mode_V)
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
        S = kvq.kvq_decode_num_splits(w.B, w.H_kv, w.ctx, sm)
        ws = kvq.DecodeWorkspace(w.B, w.H_q, w.d, S, device)

        def run():
            kvq.decode_attn(q, kc, vc, skd, svd, planes[0], planes[1], ctx, w.ctx, None,
                            num_splits=S, workspace=ws, out=out, out_dtype=kvq.OUT_FP16)
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 20
        e0.record()
        for _ in range(n):
            run()
        e1.record()
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / 1e3 / n
        nb = (w.B * w.H_kv * w.ctx * (row_bytes_total(kvq, w.d, kc.L, kc.norm_mode) +
                                      row_bytes_total(kvq, w.d, vc.L, vc.norm_mode)) +
              w.B * w.H_q * w.d * 4)
        fl = w.B * w.H_kv * w.ctx * decode_flops_per_token_head(w.d, w.G)
        res.append({"workload": f"{name} layer {layer} (L_K {kc.L}, L_V {vc.L}, {S} splits)",
                    "us": t * 1e6, "gb_per_s": nb / t / 1e9, "hbm_frac": nb / t / 1e9 / hbm_peak,
                    "tflop_per_s": fl / t / 1e12, "fp32_frac": fl / t / 1e12 / fp_peak})
        del planes, q, ws
        torch.cuda.empty_cache()
    return res


def run_case(args):
    """One kernel case on cuda:0, for profiler captures of a single launch."""
    import torch
    from decode_attention_rand_b200 import build as kbuild
    from decode_attention_rand_b200 import kvq, synth
    kbuild.build()
    kvq.lib()
    device = torch.device("cuda", 0)
    steps = max(1, min(args.steps, 20))
    if args.case == "decode_layer":
        w = synth.WORKLOADS[args.workload]
        layer = args.layer
        sk, sv = synth.layer_signs(w, layer)
        skd, svd = torch.from_numpy(sk).to(device), torch.from_numpy(sv).to(device)
        kc = kvq.codec(w.d, w.L_K[layer], w.mode_K)
        vc = kvq.codec(w.d, w.L_V[layer], w.mode_V)
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

        def run():
            kvq.decode_attn(q, kc, vc, skd, svd, planes[0], planes[1], ctx, w.ctx, None,
                            num_splits=S, workspace=ws, out=out, out_dtype=kvq.OUT_FP16)
        what = f"decode {w.name} layer {layer}, {S} splits"
    else:
        w = synth.WORKLOADS["prefill_32layers_b16_t8192_hkv8_d128"]
        sk, sv = synth.layer_signs(w, 0)
        isk = args.tensor == "k"
        c = (kvq.codec(w.d, w.L_K[0], w.mode_K) if isk else kvq.codec(w.d, w.L_V[0], w.mode_V))
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
    print(json.dumps({"case": what, "us_per_launch": e0.elapsed_time(e1) * 1e3 / steps}), flush=True)
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
        """Pick the context slice so that one step takes about per_step_s."""
        data = self._prepare(self.units[0], self.w.ctx)
        _, t_full = self._one(self.units[0], data)
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
    t_full = ors.calibrate(None)
    n = max(1, int(seconds / max(t_full, 1e-6)))
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
    ors.calibrate(budget / (args.steps + args.warmup))
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

    state = DecodeStep(w, device, l2)
    total_bytes, per_layer = step_bytes(kvq, w)
    ms, dec_ms, (tw0, tw1) = time_graph(state, args.steps, args.warmup, ctx)
    ms = max_over_ranks(ctx, ms)
    e2e_ms, e2e_n, h2d, d2h = time_e2e(state, args.steps, ctx, staged=True)
    e2e_ms = max_over_ranks(ctx, e2e_ms)
    zc_ms, zc_n, _, _ = time_e2e(state, args.steps, ctx)
    zc_ms = max_over_ranks(ctx, zc_ms)
    enc = None if args.no_encode else time_encode(device, hbm_peak)
    big = None if args.no_encode else time_decode_layers(device, hbm_peak, SM_MAX_MHZ)
    t_end = time.time()
    sampler.stop()
    if int(state.err.item()) != 0:
        raise RuntimeError(f"device error word {int(state.err.item())}")

    if ctx["rank"] != 0:
        if ctx["dist"] is not None:
            ctx["dist"].destroy_process_group()
        return 0
    clocks = sampler.summary(tw0, tw1)
    world = ctx["world"]
    value = world * total_bytes * args.steps / (ms / 1e3) / 1e9
    e2e = world * total_bytes * e2e_n / (e2e_ms / 1e3) / 1e9
    e2e_zc = world * total_bytes * zc_n / (zc_ms / 1e3) / 1e9
    # the step is one kvq_decode_step launch per layer, so the timed region's
    # device time over its launches is the kernel's average launch duration;
    # dec_ms (event nodes around each launch, which add their own dispatch
    # gaps) is reported beside it
    dec_ms_isolated = dec_ms
    dec_ms = ms / (args.steps * w.layers)
    dec_bytes = statistics.fmean(per_layer)
    achieved = dec_bytes / (dec_ms / 1e3) / 1e9
    dec_flops = w.B * w.H_kv * w.ctx * decode_flops_per_token_head(w.d, w.G)
    sm_mhz = clocks.get("sm_mhz") or SM_MAX_MHZ
    fp_peak = fp32_peak_tflops(sm_mhz, props.multi_processor_count)
    fp_achieved = dec_flops / (dec_ms / 1e3) / 1e12
    traffic = profile_traffic("decode_kernel_llama7b_layer")
    # the binding roofline of the decode kernel: FP32 FMA pipe when the time
    # its flops need at peak exceeds the time its bytes need at HBM peak
    fp_bound = dec_flops / (fp_peak * 1e12) > dec_bytes / (hbm_peak * 1e9)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            **workload_config(w), "num_splits": state.S, "out": "fp16",
            "l2": f"inputs larger than L2: {state.nbuf} rotated cache copies "
                  f"({state.nbuf * sum(per_layer) / 2**20:.0f} MiB per cycle, L2 {l2 / 2**20:.0f} MiB)",
            "timing": "CUDA graph replay, CUDA events, max over ranks",
            "bytes_per_step": total_bytes,
        },
        "roofline": ({
            "kernel": "decode_kernel (one kvq_decode_step launch: append, splits and their combine)",
            "bound": "alu", "achieved": fp_achieved, "peak": fp_peak, "unit": "TFLOP/s",
            "frac": fp_achieved / fp_peak,
            "peak_kind": f"FP32 FMA pipe, derived: {FP32_LANES_PER_SM} lanes/SM x "
                         f"{props.multi_processor_count} SMs x 2 flop x {sm_mhz:.0f} MHz",
            "traffic": traffic, "flops_per_launch": dec_flops, "bytes_per_launch": dec_bytes,
            "us_per_launch": dec_ms * 1e3, "us_per_launch_event_bracketed": dec_ms_isolated * 1e3,
        } if fp_bound else {
            "kernel": "decode_kernel (one kvq_decode_step launch: append, splits and their combine)",
            "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "peak_kind": f"{peak_kind} copy bandwidth",
            "traffic": traffic, "bytes_per_launch": dec_bytes, "us_per_launch": dec_ms * 1e3,
            "us_per_launch_event_bracketed": dec_ms_isolated * 1e3,
        }),
        "roofline_hbm": {
            "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
            "peak_kind": f"{peak_kind} copy bandwidth", "traffic": traffic,
        },
        "e2e": {"value": e2e, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_n,
                "transfer": "cudaMemcpyAsync in and out on the stream per call"},
        "e2e_zero_copy": {"value": e2e_zc, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                          "d2h_bytes_per_step": d2h, "steps": zc_n,
                          "transfer": "kernel loads / stores of page-locked host memory"},
        "gpu_launches": state.kernels_per_step * args.steps,
        "clocks": clocks,
    }
    if enc:
        line["encode"] = enc
    if big:
        for r in big:
            r["fp32_frac"] = r["tflop_per_s"] / fp_peak
        line["decode_large_layers"] = big
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)
    if ctx["dist"] is not None:
        ctx["dist"].destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
