"""Codec quality and bit-rate report on synthetic data.

Two things a user picks codebook sizes with, neither needing a model:

  * the bit accounting of the "TurboAngle: Near-Lossless KV Cache Compression
    via Uniform Angle Quantization" abstract and its early-boost schedule:
    angle bits per element (log2 L per pair of elements, averaged over K and
    V), norm bits (8-bit K and 4-bit V norms per pair) and the fp16 per-vector
    parameters, per layer and averaged over a layer schedule, next to the bits
    the packed rows really take;
  * the error the codec puts into the cache and into attention: relative L2
    error of dequantized K and V (kvq_encode + kvq_dequant on the GPU) and of
    the decode-attention output read from the codes (kvq_decode_attn)
    against attention over the uncompressed fp16 cache, as the codebook sizes
    and the norm modes of K and V vary (the abstract's asymmetric choice is
    8-bit linear K norms with 4-bit log V norms; the sweep also runs the
    other three pairings).

Run ``python -m decode_attention_rand_b200.quality`` for the default sweep.
"""
from __future__ import annotations

import argparse
import json
import math

from . import kvq, synth


# ------------------------------------------------------------- bit rates --

def bits_per_element(d: int, L_K: int, L_V: int, mode_k: int = kvq.KVQ_NORM_LIN8,
                     mode_v: int = kvq.KVQ_NORM_LOG4) -> dict:
    """Nominal and stored bits per cached element of one layer (K and V
    averaged); by default 8-bit linear K norms and 4-bit log V norms.

    Nominal counts log2 L bits per pair for the angle, as the abstract's
    accounting does; stored is what the packed rows of include/kvq.h take
    (whole 32-bit angle words, byte-aligned norms and params)."""
    nbits = {kvq.KVQ_NORM_LIN8: 8, kvq.KVQ_NORM_LOG4: 4}
    pbits = {kvq.KVQ_NORM_LIN8: 16, kvq.KVQ_NORM_LOG4: 32}
    angle = (math.log2(L_K) + math.log2(L_V)) / 4.0
    norms = (nbits[mode_k] + nbits[mode_v]) / 4.0  # one norm code per pair
    params = (pbits[mode_k] + pbits[mode_v]) / (2.0 * d)  # fp16 parameters per vector
    kc = kvq.codec(d, L_K, mode_k)
    vc = kvq.codec(d, L_V, mode_v)
    stored = sum(kvq.kvq_row_bytes(kc, w) + kvq.kvq_row_bytes(vc, w) for w in range(3)) * 8 / (2.0 * d)
    return {"angle": angle, "norms": norms, "params": params,
            "total": angle + norms + params, "stored": stored}


def schedule_bits(w: synth.Workload) -> dict:
    """Bits per element averaged over the layers of a workload's schedule
    (early-boost layers weigh as much as any other layer)."""
    per = [bits_per_element(w.d, w.L_K[i], w.L_V[i]) for i in range(w.layers)]
    keys = per[0].keys()
    return {k: sum(p[k] for p in per) / len(per) for k in keys}


# ---------------------------------------------------------------- errors --

def _rel_l2_rows(a, b):
    a = a.double().reshape(-1, a.shape[-1])
    b = b.double().reshape(-1, b.shape[-1])
    return ((a - b).norm(dim=1) / b.norm(dim=1).clamp_min(1e-30))


MODES = {"lin8": kvq.KVQ_NORM_LIN8, "log4": kvq.KVQ_NORM_LOG4}


def codec_error(w: synth.Workload, layer: int, L_K: int, L_V: int, tokens: int | None = None,
                device="cuda", mode_k: int = kvq.KVQ_NORM_LIN8,
                mode_v: int = kvq.KVQ_NORM_LOG4) -> dict:
    """Relative L2 errors of the codec on one layer of a synthetic workload,
    truncated to `tokens` cached tokens: dequantized K and V per vector
    (mean and max) and the attention output per query head (mean and max)
    against fp64 attention over the uncompressed fp16 K and V."""
    import torch
    T = min(tokens or w.ctx, w.ctx)
    T16 = (T + 15) // 16 * 16
    sk, sv = synth.layer_signs(w, layer)
    skd, svd = torch.from_numpy(sk).to(device), torch.from_numpy(sv).to(device)
    kc = kvq.codec(w.d, L_K, mode_k)
    vc = kvq.codec(w.d, L_V, mode_v)
    k = synth.kv(w, layer, synth.KIND_K, device=device, T=T)
    v = synth.kv(w, layer, synth.KIND_V, device=device, T=T)
    K = kvq.alloc_plane(kc, w.B, w.H_kv, T16, device)
    V = kvq.alloc_plane(vc, w.B, w.H_kv, T16, device)
    kvq.encode(kc, skd, k, K, 0)
    kvq.encode(vc, svd, v, V, 0)
    kh = kvq.dequant(kc, skd, K, T)
    vh = kvq.dequant(vc, svd, V, T)
    ek, ev = _rel_l2_rows(kh, k), _rel_l2_rows(vh, v)
    names = {v_: k_ for k_, v_ in MODES.items()}
    res = {"L_K": L_K, "L_V": L_V, "tokens": T, "norms": f"K {names[mode_k]}, V {names[mode_v]}",
           "k_rel_l2_mean": ek.mean().item(), "k_rel_l2_max": ek.max().item(),
           "v_rel_l2_mean": ev.mean().item(), "v_rel_l2_max": ev.max().item(),
           "attn_rel_l2_mean": None, "attn_rel_l2_max": None,
           **{"bits_" + k_: v_ for k_, v_ in bits_per_element(w.d, L_K, L_V, mode_k,
                                                               mode_v).items()}}
    q = synth.queries(w, layer, device=device)
    ctx = torch.full((w.B,), T, dtype=torch.int32, device=device)
    tau = 1.0 / math.sqrt(w.d)
    out = kvq.decode_attn(q, kc, vc, skd, svd, K, V, ctx, T, tau)
    # attention over the uncompressed cache, fp64 (the yardstick, not a path)
    G = w.H_q // w.H_kv
    kk = k.double().repeat_interleave(G, dim=1)
    vv = v.double().repeat_interleave(G, dim=1)
    s = torch.einsum("bhd,bhtd->bht", q.double(), kk) * tau
    ref = torch.einsum("bht,bhtd->bhd", torch.softmax(s, dim=-1), vv)
    torch.cuda.synchronize()
    eo = _rel_l2_rows(out, ref)
    res["attn_rel_l2_mean"] = eo.mean().item()
    res["attn_rel_l2_max"] = eo.max().item()
    return res


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="llama7b_layer_b1_hq32_hkv8_d128_ctx4096",
                    choices=sorted(synth.WORKLOADS))
    ap.add_argument("--layer", type=int, default=0)
    ap.add_argument("--L", type=int, nargs="+", default=[16, 32, 64, 128, 256, 1024, 4096],
                    help="codebook sizes swept for K and V together")
    ap.add_argument("--tokens", type=int, default=2048, help="cached tokens per sequence")
    ap.add_argument("--norms", nargs="+", default=["lin8,log4", "log4,log4", "lin8,lin8",
                                                   "log4,lin8"],
                    help="norm modes swept, each 'K,V' (lin8 or log4)")
    ap.add_argument("--json", action="store_true")
    args = ap.parse_args(argv)
    w = synth.WORKLOADS[args.workload]
    kvq.lib()
    rows = []
    for nm in args.norms:
        mk, mv = (MODES[x] for x in nm.split(","))
        rows += [codec_error(w, args.layer, L, L, args.tokens, mode_k=mk, mode_v=mv)
                 for L in args.L]
    sched = {name: schedule_bits(ww) for name, ww in synth.WORKLOADS.items() if ww.kind == "decode"}
    if args.json:
        print(json.dumps({"errors": rows, "schedules": sched}))
        return 0
    print(f"{w.name}, layer {args.layer}, {rows[0]['tokens']} tokens")
    print(f"{'norms':>16} {'L_K=L_V':>8} {'bits/elt':>8} {'stored':>7} {'K err':>9} "
          f"{'V err':>9} {'attn err':>9} {'attn max':>9}")
    fmt = lambda x: f"{x:>9.2e}" if x is not None else f"{'-':>9}"
    for r in rows:
        print(f"{r['norms']:>16} {r['L_K']:>8} {r['bits_total']:>8.3f} {r['bits_stored']:>7.3f} "
              f"{fmt(r['k_rel_l2_mean'])} {fmt(r['v_rel_l2_mean'])} "
              f"{fmt(r['attn_rel_l2_mean'])} {fmt(r['attn_rel_l2_max'])}")
    print("\nlayer schedules (bits per element, averaged over layers):")
    for name, b in sched.items():
        print(f"  {name:48s} angle {b['angle']:.3f}  total {b['total']:.3f}  stored {b['stored']:.3f}")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
