"""Context-sharded decode attention: the cached context of each sequence spread
over the ranks of a process group (one GPU each), merged once per step.

Each rank holds a range of every sequence's tokens in its own planes (its
`ctx_len` counts the tokens it holds) and runs kvq_decode_attn_partials over
them: per (batch entry, query head, split) a running maximum, a softmax
denominator and a rotated-domain accumulator, in its workspace.  The
workspaces are all-gathered (one exchange of B * H_q * splits * (d + 2)
floats per rank and step) and kvq_decode_merge_partials merges every rank's
splits into the attention output, the same merge the single-GPU decode
performs over its own splits.  Every rank ends with the full output.

This module is argument marshalling and the exchange; the arithmetic runs in
the library's kernels.
"""
from __future__ import annotations

import math

from . import kvq


def decode_attn_partials(q, kc, vc, signs_k, signs_v, K: "kvq.Plane", V: "kvq.Plane", ctx_len,
                         max_ctx: int, num_splits: int, softmax_scale: float | None = None,
                         workspace: "kvq.DecodeWorkspace | None" = None, err_word=None,
                         stream=None) -> "kvq.DecodeWorkspace":
    """This rank's partials (kvq_decode_attn_partials) in a workspace."""
    B, H_q, d = q.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if workspace is None or workspace.num_splits != num_splits:
        workspace = kvq.DecodeWorkspace(B, H_q, d, num_splits, q.device)
    kvq.kvq_decode_attn_partials(q, kc, vc, signs_k, signs_v, K.c(), V.c(), ctx_len, B, H_q,
                                 K.H_kv, max_ctx, softmax_scale, num_splits, workspace.buf,
                                 workspace.nbytes, err_word, stream)
    return workspace


def merge_partials(parts, B: int, H_q: int, d: int, num_splits: int, signs_v, out=None,
                   out_dtype: int = kvq.OUT_FP32, stream=None):
    """Attention output from `parts`, the workspaces of every rank stacked
    [n_parts][workspace bytes] (kvq_decode_merge_partials)."""
    import torch
    n_parts = parts.shape[0]
    if out is None:
        out = torch.empty((B, H_q, d), dtype=torch.float16 if out_dtype == kvq.OUT_FP16
                          else torch.float32, device=parts.device)
    kvq.kvq_decode_merge_partials(parts, n_parts, B, H_q, d, num_splits, signs_v, out, out_dtype,
                                  stream)
    return out


def gather_partials(buf, group=None):
    """Every rank's workspace bytes, stacked in rank order: [world][n]."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    bufs = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(bufs, buf, group=group)
    return torch.stack(bufs)


def context_sharded_decode(q, kc, vc, signs_k, signs_v, K: "kvq.Plane", V: "kvq.Plane",
                           ctx_len, max_ctx: int, num_splits: int,
                           softmax_scale: float | None = None, group=None,
                           out_dtype: int = kvq.OUT_FP32, err_word=None):
    """One decode step over a context sharded across the ranks of `group`:
    this rank's partials, the all-gather, the merge.  q, the codecs and the
    diagonals are the same on every rank; K, V, ctx_len and max_ctx describe
    the tokens this rank holds; num_splits is the same on every rank."""
    B, H_q, d = q.shape
    ws = decode_attn_partials(q, kc, vc, signs_k, signs_v, K, V, ctx_len, max_ctx, num_splits,
                              softmax_scale, err_word=err_word)
    parts = gather_partials(ws.buf[:ws.nbytes], group)
    return merge_partials(parts, B, H_q, d, num_splits, signs_v, out_dtype=out_dtype)
