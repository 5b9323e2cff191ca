"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the codec: it only draws inputs (fp16 K/V
head vectors, queries, the +-1 diagonal of each (layer, K|V)) with fixed
seeds, in the shapes and distributions of the workloads below.  No trained
weights or datasets are used; the synthetic tensors stand in for the KV
activations of the models whose shapes the workloads borrow (Llama-7B,
Mistral-7B, TinyLlama), and for the perplexity dataset of "TurboAngle:
Near-Lossless KV Cache Compression via Uniform Angle Quantization", Abstract.

Distributions (per workload):
  "tiny"      K ~ N(0,1) with channels 3 and 77 scaled x20; V ~ N(0,1)
  "llama"     K ~ N(0,1) * s_c, s_c ~ lognormal(0, 0.5) per (KV head,
              channel), plus 2 channels per KV head scaled x20; V ~ N(0,1)
  "tinyllama" K ~ N(0,1) with 1 channel per KV head scaled x30; V ~ N(0,1)
  queries     N(0,1)
Random channel choices and scales come from numpy's PCG64 seeded by
(seed, layer, kind); the bulk normals from a torch.Generator on the target
device, seeded the same way, so a tensor is reproducible per device.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

MASK64 = (1 << 64) - 1
KIND_K, KIND_V, KIND_Q = 0, 1, 2


def splitmix64(x: int) -> int:
    """One step of SplitMix64 (Steele, Lea and Flood, 2014), on Python ints."""
    x = (x + 0x9E3779B97F4A7C15) & MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def stream_seed(seed: int, layer: int, kind: int) -> int:
    """63-bit seed of the (seed, layer, kind) substream."""
    return splitmix64((seed << 32) + (layer << 2) + kind) >> 1


def signs(seed: int, layer: int, kind: int, d: int) -> np.ndarray:
    """The +-1 diagonal D of one (layer, K|V): s_j = +1 when the top bit of
    SplitMix64(base + j) is 0, base = stream_seed(seed, layer, kind)."""
    base = stream_seed(seed, layer, kind)
    out = np.empty(d, np.int8)
    for j in range(d):
        out[j] = -1 if (splitmix64(base + j) >> 63) else 1
    return out


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    B: int
    H_q: int
    H_kv: int
    d: int
    ctx: int
    L_K: tuple
    L_V: tuple
    k_dist: str
    seed: int = 0
    kind: str = "decode"  # "decode" or "prefill"
    note: str = ""
    mode_K: int = 0  # LIN8
    mode_V: int = 1  # LOG4

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv


def _per_layer(n, early, early_L, late_L):
    return tuple(early_L if i < early else late_L for i in range(n))


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_b1_hq4_hkv2_d128_ctx256", 1, 1, 4, 2, 128, 256, (128,), (128,), "tiny",
                 note="round trip + one decode step: the 256th token is appended, then attended"),
        Workload("llama7b_layer_b1_hq32_hkv8_d128_ctx4096", 1, 1, 32, 8, 128, 4096, (128,), (64,),
                 "llama", note="Llama-7B-shaped single layer decode step"),
        Workload("mistral7b_32layers_b8_hq32_hkv8_d128_ctx32768", 32, 8, 32, 8, 128, 32768,
                 _per_layer(32, 4, 256, 128), _per_layer(32, 4, 256, 64), "tiny",
                 note="Mistral-7B-shaped decode step with per-layer early-boost (layers 0-3)"),
        Workload("prefill_32layers_b16_t8192_hkv8_d128", 32, 16, 32, 8, 128, 8192,
                 (128,) * 32, (64,) * 32, "tiny", kind="prefill",
                 note="prefill encode throughput plus dequant back to fp16"),
        Workload("tinyllama_22layers_b4_hq32_hkv4_d64_ctx65536", 22, 4, 32, 4, 64, 65536,
                 _per_layer(22, 2, 256, 128), _per_layer(22, 2, 256, 32), "tinyllama",
                 note="TinyLlama-shaped long-context small-head decode step"),
    ]
}
WORKLOAD_ORDER = list(WORKLOADS)


def _np_rng(seed: int, layer: int, kind: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(stream_seed(seed, layer, kind) ^ 0x5EED))


def _torch_gen(device, seed: int, layer: int, kind: int, salt: int = 0):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((stream_seed(seed, layer, kind) + salt) & ((1 << 63) - 1))
    return g


def channel_scales(w: Workload, layer: int, kind: int) -> np.ndarray:
    """Per (KV head, channel) multiplier of the raw normals, float32 [H_kv, d]."""
    sc = np.ones((w.H_kv, w.d), np.float32)
    if kind != KIND_K:
        return sc
    rng = _np_rng(w.seed, layer, kind)
    if w.k_dist == "tiny":
        for c in (3, 77):
            if c < w.d:
                sc[:, c] = 20.0
    elif w.k_dist == "llama":
        sc *= rng.lognormal(0.0, 0.5, size=(w.H_kv, w.d)).astype(np.float32)
        for h in range(w.H_kv):
            for c in rng.choice(w.d, size=2, replace=False):
                sc[h, c] *= 20.0
    elif w.k_dist == "tinyllama":
        for h in range(w.H_kv):
            sc[h, rng.integers(0, w.d)] *= 30.0
    else:
        raise ValueError(w.k_dist)
    return sc


def kv(w: Workload, layer: int, kind: int, device="cpu", T: int | None = None,
       b_range=None, salt: int = 0):
    """fp16 K (kind 0) or V (kind 1) tensor [B', H_kv, T, d] on `device`.

    The normals of batch entry b come from their own generator, so any batch
    sub-range b_range=(b0, b1) reproduces the same values as the full tensor.
    """
    import torch
    T = w.ctx if T is None else T
    b0, b1 = (0, w.B) if b_range is None else b_range
    sc = torch.from_numpy(channel_scales(w, layer, kind)).to(device)
    out = torch.empty((b1 - b0, w.H_kv, T, w.d), dtype=torch.float16, device=device)
    for b in range(b0, b1):
        g = _torch_gen(device, w.seed, layer, kind, salt=salt * 1_000_003 + b + 1)
        x = torch.randn((w.H_kv, T, w.d), generator=g, device=device, dtype=torch.float32)
        x.mul_(sc[:, None, :])
        out[b - b0] = x.to(torch.float16)
    return out


def queries(w: Workload, layer: int, device="cpu", salt: int = 0):
    """fp16 queries [B, H_q, d], N(0,1)."""
    import torch
    g = _torch_gen(device, w.seed, layer, KIND_Q, salt=salt)
    return torch.randn((w.B, w.H_q, w.d), generator=g, device=device,
                       dtype=torch.float32).to(torch.float16)


def layer_signs(w: Workload, layer: int):
    """(signs_K, signs_V) int8 [d] of one layer."""
    return signs(w.seed, layer, KIND_K, w.d), signs(w.seed, layer, KIND_V, w.d)


@dataclass
class Shape:
    """A small ad-hoc shape for sweeps and edge cases."""
    B: int
    H_q: int
    H_kv: int
    d: int
    ctx: int
    L_K: int
    L_V: int
    k_dist: str = "tiny"
    seed: int = 0
    extra: dict = field(default_factory=dict)

    def workload(self) -> Workload:
        return Workload(f"adhoc_b{self.B}_hq{self.H_q}_hkv{self.H_kv}_d{self.d}_ctx{self.ctx}",
                        1, self.B, self.H_q, self.H_kv, self.d, self.ctx, (self.L_K,),
                        (self.L_V,), self.k_dist, seed=self.seed)
