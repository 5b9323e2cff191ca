"""Helpers shared by the parity tests.

``unpack_rows`` reads codes out of packed rows with plain numpy bit
arithmetic (it is used to compare the GPU's bytes with the oracle's codes and
shares nothing with either implementation).  ``compare_codes`` applies the
parity rule: angle and norm codes and fp16 parameters bit-exact, except where
the oracle flags a value within 1e-6 of a decision edge; mismatches must be
at most 1e-5 of all codes.
"""
from __future__ import annotations

import numpy as np

import oracle as O

REL_L2_TOL = 2e-3      # dequantized vectors and attention outputs
MISMATCH_BUDGET = 1e-5  # fraction of codes that may differ (all of them flagged)


def angle_bits(L: int) -> int:
    b = 1
    while (1 << b) < L:
        b += 1
    return b


def unpack_rows(angles: np.ndarray, norms: np.ndarray, params: np.ndarray, d: int, L: int,
                mode: int):
    """(angle codes [n,P], norm codes [n,P], param fp16 bits [n,1|2]) from rows."""
    P = d // 2
    b = angle_bits(L)
    n = angles.shape[0]
    words = angles.reshape(n, -1).view("<u4").astype(np.uint64)
    a = np.zeros((n, P), np.int64)
    for i in range(P):
        pos = i * b
        w, sh = pos // 32, pos % 32
        v = words[:, w] >> np.uint64(sh)
        if sh + b > 32:
            v |= words[:, w + 1] << np.uint64(32 - sh)
        a[:, i] = (v & np.uint64((1 << b) - 1)).astype(np.int64)
    if mode == O.MODE_LIN8:
        c = norms.reshape(n, P).astype(np.int64)
        p = params.reshape(n, 2).view("<u2").astype(np.int64).reshape(n, 1)
    else:
        nb = norms.reshape(n, P // 2).astype(np.int64)
        c = np.empty((n, P), np.int64)
        c[:, 0::2] = nb & 0xF
        c[:, 1::2] = nb >> 4
        p = params.reshape(n, 4).view("<u2").astype(np.int64).reshape(n, 2)
    return a, c, p


def compare_codes(gpu_rows, oracle_codes: "O.Codes", budget: float = MISMATCH_BUDGET):
    """Check GPU rows (angles, norms, params as uint8 [n, row]) against the
    oracle's codes of the same vectors; returns a stats dict."""
    d, L, mode = oracle_codes.d, oracle_codes.L, oracle_codes.mode
    ga, gc, gp = unpack_rows(*gpu_rows, d, L, mode)
    oa, oc, op = unpack_rows(oracle_codes.angles, oracle_codes.norms, oracle_codes.params, d, L,
                             mode)
    f = oracle_codes.flags
    pflag = (f[:, :1] & O.FLAG_PARAM) != 0
    bad_a = (ga != oa) & ((f & O.FLAG_ANGLE) == 0)
    bad_n = (gc != oc) & ((f & (O.FLAG_NORM | O.FLAG_PARAM)) == 0)
    bad_p = (gp != op) & ~pflag
    n_codes = ga.size * 2
    mism = int((ga != oa).sum() + (gc != oc).sum())
    stats = dict(vectors=ga.shape[0], codes=n_codes, mismatches=mism,
                 unflagged_angle=int(bad_a.sum()), unflagged_norm=int(bad_n.sum()),
                 unflagged_param=int(bad_p.sum()),
                 flagged=int((f != 0).sum()))
    assert stats["unflagged_angle"] == 0, stats
    assert stats["unflagged_norm"] == 0, stats
    assert stats["unflagged_param"] == 0, stats
    assert mism <= budget * n_codes, stats
    return stats


def rel_l2(got: np.ndarray, want: np.ndarray, axis=-1) -> np.ndarray:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    num = np.linalg.norm(got - want, axis=axis)
    den = np.linalg.norm(want, axis=axis)
    return num / np.maximum(den, 1e-300)


def plane_rows(plane, b_range=None, h_range=None, t_range=None):
    """Host copy of the rows of a kvq.Plane: (angles, norms, params), each
    uint8 [n, row] in (b, h, t) order over the given ranges."""
    out = []
    for w in range(3):
        r = plane.rows(w)
        if b_range is not None:
            r = r[b_range[0]:b_range[1]]
        if h_range is not None:
            r = r[:, h_range[0]:h_range[1]]
        if t_range is not None:
            r = r[:, :, t_range[0]:t_range[1]]
        out.append(np.ascontiguousarray(r.cpu().numpy().reshape(-1, r.shape[-1])))
    return tuple(out)


def paged_rows(plane, table, b: int, t0: int, t1: int):
    """Host copy of tokens t0 .. t1-1 of every KV head of sequence b of a
    kvq.PagedPlane, read through the page table `table` [B][max_pages]:
    (angles, norms, params), each uint8 [n, row] in (h, t) order."""
    import torch
    pt = plane.page_tokens
    t = torch.arange(t0, t1)
    pages = torch.as_tensor(np.asarray(table)[b], dtype=torch.long)[t // pt]
    dev = plane.rows(0).device
    pages, offs = pages.to(dev), (t % pt).to(dev)
    out = []
    for w in range(3):
        r = plane.rows(w)
        rows = [r[pages, h, offs] for h in range(plane.H_kv)]
        out.append(np.ascontiguousarray(torch.cat(rows).cpu().numpy()))
    return tuple(out)


def put_rows(plane, codes: "O.Codes", b, h, t0: int):
    """Write oracle-encoded rows (tokens t0.. of sequence (b, h)) into a plane."""
    import torch
    n = codes.n
    for w, arr in enumerate((codes.angles, codes.norms, codes.params)):
        dst = plane.rows(w)[b, h, t0:t0 + n]
        dst.copy_(torch.from_numpy(np.ascontiguousarray(arr)).to(dst.device))
