"""kvq_decode_attn_noalloc, the decode entry point for callers that cannot
allocate device memory (for example a serving loop whose device memory all
belongs to its own pooling allocator, or a plain C program without an
allocator), checked through the C ABI against kvq_decode_attn, which takes a
caller-allocated workspace.

The no-allocation variant draws its scratch from an array built into the
library and shared by every call, so it is called twice in a row here: the
second call must not be disturbed by what the first left behind.  This file
is collected last so that a run stopping at the first failure has already
run every other test.
"""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from decode_attention_rand_b200 import build as kbuild
from decode_attention_rand_b200 import kvq, synth

pytestmark = pytest.mark.gpu
REL_L2_TOL = 2e-3  # the tolerance the parity tests use for attention outputs


@pytest.fixture(scope="module")
def ready():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    kbuild.build()
    kvq.lib()
    return torch.device("cuda:0")


def _layer(w, layer, dev):
    sk, sv = synth.layer_signs(w, layer)
    skd, svd = torch.from_numpy(sk).to(dev), torch.from_numpy(sv).to(dev)
    kc = kvq.codec(w.d, w.L_K[layer], kvq.KVQ_NORM_LIN8)
    vc = kvq.codec(w.d, w.L_V[layer], kvq.KVQ_NORM_LOG4)
    cap = (w.ctx + 15) // 16 * 16
    Kp, Vp = kvq.alloc_plane(kc, w.B, w.H_kv, cap, dev), kvq.alloc_plane(vc, w.B, w.H_kv, cap, dev)
    kvq.encode(kc, skd, synth.kv(w, layer, synth.KIND_K, device=dev), Kp, 0)
    kvq.encode(vc, svd, synth.kv(w, layer, synth.KIND_V, device=dev), Vp, 0)
    q = synth.queries(w, layer, device=dev)
    return kc, vc, skd, svd, Kp, Vp, q


def _rel_l2(a, b):
    a = a.double().reshape(-1, a.shape[-1])
    b = b.double().reshape(-1, b.shape[-1])
    return ((a - b).norm(dim=1) / b.norm(dim=1).clamp_min(1e-30)).max().item()


def _noalloc(w, kc, vc, skd, svd, Kp, Vp, q, ctx, tau, S, err, like):
    out = torch.full_like(like, float("nan"))
    kvq.kvq_decode_attn_noalloc(q, kc, vc, skd, svd, Kp.c(), Vp.c(), ctx, w.B, w.H_q, w.H_kv,
                                w.ctx, tau, S, err, out, kvq.OUT_FP32)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("name,ctx_lens,splits", [
    # 16 splits of 8 KV heads: one cluster per KV head, partials in shared memory
    ("llama7b_layer_b1_hq32_hkv8_d128_ctx4096", None, 16),
    # the default split count (18 here: last-CTA combine)
    ("llama7b_layer_b1_hq32_hkv8_d128_ctx4096", None, None),
    # 20 splits (more than a cluster takes): partials and completion counters
    # in the built-in scratch array, merged by the last CTA of each KV head
    ("llama7b_layer_b1_hq32_hkv8_d128_ctx4096", None, 20),
    ("tiny_b1_hq4_hkv2_d128_ctx256", [200], None),
])
def test_noalloc_matches_workspace_entry_point(ready, name, ctx_lens, splits):
    """Same kernel, same splits, same inputs: the output is bit-identical to
    kvq_decode_attn with a caller workspace, on two calls in a row."""
    dev = ready
    w = synth.WORKLOADS[name]
    kc, vc, skd, svd, Kp, Vp, q = _layer(w, 0, dev)
    ctx_vals = ctx_lens or [w.ctx] * w.B
    ctx = torch.tensor(ctx_vals, dtype=torch.int32, device=dev)
    sm = torch.cuda.get_device_properties(dev).multi_processor_count
    S = splits or kvq.kvq_decode_num_splits(w.B, w.H_kv, w.ctx, sm)
    tau = 1.0 / math.sqrt(w.d)
    ref = kvq.decode_attn(q, kc, vc, skd, svd, Kp, Vp, ctx, w.ctx, tau, num_splits=S,
                          out_dtype=kvq.OUT_FP32)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for call in range(2):
        out = _noalloc(w, kc, vc, skd, svd, Kp, Vp, q, ctx, tau, S, err, ref)
        assert torch.equal(out, ref), call
    assert int(err.item()) == 0
    assert _rel_l2(out, ref) <= REL_L2_TOL


def test_noalloc_scratch_reuse_across_calls(ready):
    """Calls in a row share the array and find the previous call's partials
    and counters there: 20 splits, then 7 splits over a shorter context (its
    counters are fewer and its partials land elsewhere), a call rejected for
    its size, 20 splits again with another query; each equals its
    workspace-entry-point twin."""
    dev = ready
    w = synth.WORKLOADS["llama7b_layer_b1_hq32_hkv8_d128_ctx4096"]
    kc, vc, skd, svd, Kp, Vp, q = _layer(w, 0, dev)
    tau = 1.0 / math.sqrt(w.d)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    q2 = torch.flip(q, dims=[1]).contiguous()
    plan = [(20, w.ctx, q), (7, 1500, q), (None, w.ctx, q), (20, w.ctx, q2)]
    for S, n, qq in plan:
        ctx = torch.tensor([n], dtype=torch.int32, device=dev)
        if S is None:
            out = torch.zeros((1, w.H_q, w.d), dtype=torch.float32, device=dev)
            with pytest.raises(kvq.KvqError):
                kvq.kvq_decode_attn_noalloc(qq, kc, vc, skd, svd, Kp.c(), Vp.c(), ctx, 1, w.H_q,
                                            w.H_kv, w.ctx, tau, 65535, err, out, kvq.OUT_FP32)
            continue
        ref = kvq.decode_attn(qq, kc, vc, skd, svd, Kp, Vp, ctx, w.ctx, tau, num_splits=S,
                              out_dtype=kvq.OUT_FP32)
        out = _noalloc(w, kc, vc, skd, svd, Kp, Vp, qq, ctx, tau, S, err, ref)
        assert torch.equal(out, ref), (S, n)
    assert int(err.item()) == 0


def test_noalloc_rejects_a_request_beyond_its_scratch(ready):
    dev = ready
    w = synth.WORKLOADS["tiny_b1_hq4_hkv2_d128_ctx256"]
    kc, vc, skd, svd, Kp, Vp, q = _layer(w, 0, dev)
    ctx = torch.tensor([w.ctx], dtype=torch.int32, device=dev)
    # a split count whose partials exceed the built-in scratch
    splits = 65535
    need = kvq.kvq_decode_workspace_bytes(1, w.H_q, w.d, splits)
    assert need > (4 << 20)
    out = torch.zeros((1, w.H_q, w.d), dtype=torch.float32, device=dev)
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attn_noalloc(q, kc, vc, skd, svd, Kp.c(), Vp.c(), ctx, 1, w.H_q, w.H_kv,
                                    w.ctx, 0.1, splits, None, out, kvq.OUT_FP32)
    assert e.value.status == kvq.KVQ_EINVAL
    assert "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert bool((out == 0).all())
